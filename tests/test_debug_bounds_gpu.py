"""The MOE_DEBUG_BOUNDS build on the GPU: the small parity cases, run through
libmoe_b200_debug.so (every index one kernel computes and another uses is
checked before the access), still match the oracle and leave the status word
at 0, i.e. no check fired on valid inputs. Runs the cases in a child process
that loads the debug library in place of the normal one. No input here is
built to drive an index out of range: the predicates themselves are tested on
the host (test_bounds_host.py)."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = ("tiny_f32_full_parity or f32_ragged or bf16_parity_all_paths or int8_parity_all_paths or "
         "fused_combine or token_tile_split_k or weight_stream_split_k or variants_bf16 or "
         "int8_tall_tiles or row_gather_parity or pair_tile_boundaries")


def test_parity_cases_through_the_debug_build():
    from mixture_experts_ffn_14_b200 import build as B

    if not os.path.exists(B.LIB_DEBUG):
        B.build(debug_bounds=True)
    env = dict(os.environ, MOE_B200_LIBRARY=os.path.basename(B.LIB_DEBUG))
    flags = subprocess.run([sys.executable, "-c", "import mixture_experts_ffn_14_b200 as m; print(m.moe_build_flags())"],
                           cwd=ROOT, env=env, capture_output=True, text=True)
    assert flags.stdout.strip() == "1", flags.stdout + flags.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_parity_gpu.py", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider", "-k", CASES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
