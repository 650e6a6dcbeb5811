"""Host-compiled checks of device logic (no GPU): the index predicates of the
MOE_DEBUG_BOUNDS build with in-range and out-of-range indices, and the
token-tile order of the expert GEMMs; and the debug build of the library loads
and reports its flag."""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixture_experts_ffn_14_b200", "csrc")


def test_bounds_predicates_on_host(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.fail("no host C++ compiler")
    exe = tmp_path / "bounds_check"
    subprocess.run([cxx, "-std=c++17", "-O1", "-Wall", "-Werror", "-I", CSRC,
                    os.path.join(ROOT, "tests", "bounds_host_check.cpp"), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "bounds predicates ok" in r.stdout


def test_tile_order_is_a_grouped_bijection(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.fail("no host C++ compiler")
    exe = tmp_path / "tile_order_check"
    subprocess.run([cxx, "-std=c++17", "-O2", "-Wall", "-Werror", "-I", CSRC,
                    os.path.join(ROOT, "tests", "tile_order_host_check.cpp"), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr
    assert "tile order ok" in r.stdout


def test_debug_build_loads_and_reports_its_flag():
    from mixture_experts_ffn_14_b200 import build as B

    lib = B.LIB_DEBUG
    if not os.path.exists(lib):
        B.build(debug_bounds=True)
    code = ("import mixture_experts_ffn_14_b200 as m; "
            "print(m.moe_build_flags(), m.moe_abi_version())")
    env = dict(os.environ, MOE_B200_LIBRARY=os.path.basename(lib))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["1", "2"]
    import mixture_experts_ffn_14_b200 as m
    assert m.moe_build_flags() == 0          # the normal build has no checks
