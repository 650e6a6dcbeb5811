"""Expert parallelism of the MoE sublayer over W GPUs, one process per GPU.

Grok-1 book ch. 1, section 1.6.3: the MoE layer shards the expert axis over
the devices of a (1, 8) mesh with shard_map, because which experts a token
needs is only known at run time. Here GPU r owns the n = 8 / W consecutive
experts r*n .. r*n + n - 1 (their weights only) and holds its own batch of
tokens. One forward:

  1. route and dispatch the local tokens (``moe_route_dispatch``): the permuted
     rows are sorted by (expert, token), hence grouped by owning GPU;
  2. exchange the per-expert row counts (an all-to-all of W x n integers; the
     counts are read back to the host once, as the split sizes of step 3);
  3. send every block of rows and its gates to the GPU that owns its experts
     (all-to-all with those split sizes);
  4. make the received rows expert-contiguous (``moe_gather_rows``: they arrive
     grouped by source GPU);
  5. run the local experts, gate applied (``moe_experts_forward``);
  6. undo step 4 and send every row back (all-to-all, split sizes reversed):
     each GPU gets its rows back in its own permuted order;
  7. sum each token's two rows (``moe_combine``).

Steps 1, 4, 5, 6 (the gather) and 7 run in the library's kernels; the
exchanges are the communication library's all-to-all (NCCL over NVLink under
torch.distributed, or gloo on the CPU). The host logic of the exchange (split
sizes, receive layout, the expert-major reordering) is in ``ExchangePlan`` and
``ep_forward``; the compute steps come from a ``LocalCompute`` object
(``LibraryCompute`` runs them on the GPU through the C ABI).
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Sequence

import numpy as np

E_TOTAL = 8


def experts_per_rank(world: int, E: int = E_TOTAL) -> int:
    if world < 1 or E % world != 0:
        raise ValueError(f"{E} experts do not split evenly over {world} GPUs")
    return E // world


def local_experts(rank: int, world: int, E: int = E_TOTAL) -> range:
    """Experts owned by GPU ``rank``."""
    n = experts_per_rank(world, E)
    return range(rank * n, rank * n + n)


def send_rows(counts: Sequence[int], world: int, E: int = E_TOTAL) -> list:
    """Rows this GPU sends to each GPU: the sum of its per-expert token-slot
    counts over the experts the destination owns."""
    n = experts_per_rank(world, E)
    c = [int(v) for v in counts]
    if len(c) != E:
        raise ValueError("counts must have one entry per expert")
    return [sum(c[r * n:(r + 1) * n]) for r in range(world)]


@dataclass
class ExchangePlan:
    """Layout of one exchange, seen from GPU ``rank``.

    recv_counts[s][j]: rows GPU s sends for local expert j. The receive buffer
    is source-major (all of GPU 0's rows, sorted by expert, then GPU 1's...);
    the experts run on expert-major rows (all rows of local expert 0, in source
    order, then expert 1...). ``to_expert_major[i]`` is the receive-buffer row
    of expert-major row i; ``to_source_major`` is its inverse."""

    rank: int
    world: int
    send_rows: list
    recv_counts: np.ndarray
    recv_rows: list
    expert_rows: list
    to_expert_major: np.ndarray
    to_source_major: np.ndarray

    @property
    def rows_in(self) -> int:
        return int(sum(self.recv_rows))


def make_plan(rank: int, world: int, counts: Sequence[int], recv_counts, E: int = E_TOTAL) -> ExchangePlan:
    """Plan of GPU ``rank`` from its own per-expert counts and the counts the
    other GPUs send it (``recv_counts`` [world, n])."""
    n = experts_per_rank(world, E)
    rc = np.asarray(recv_counts, dtype=np.int64).reshape(world, n)
    if (rc < 0).any():
        raise ValueError("negative row count")
    # Receive-buffer start of each (source, local expert) block, source-major.
    start = np.zeros((world, n), dtype=np.int64)
    at = 0
    for s in range(world):
        for j in range(n):
            start[s, j] = at
            at += rc[s, j]
    order = [np.arange(start[s, j], start[s, j] + rc[s, j], dtype=np.int64) for j in range(n) for s in range(world)]
    to_em = np.concatenate(order) if order else np.zeros(0, dtype=np.int64)
    inv = np.empty_like(to_em)
    inv[to_em] = np.arange(to_em.shape[0], dtype=np.int64)
    return ExchangePlan(rank=rank, world=world, send_rows=send_rows(counts, world, E), recv_counts=rc,
                        recv_rows=[int(v) for v in rc.sum(axis=1)], expert_rows=[int(v) for v in rc.sum(axis=0)],
                        to_expert_major=to_em, to_source_major=inv)


class LocalCompute:
    """The compute steps of one GPU's forward (see the module docstring).

    ``route_dispatch(x)`` returns a dict with at least ``counts`` (host list of
    8 ints), ``xp`` (permuted rows [2T, d]), ``gate_perm`` ([2T]) and whatever
    ``combine`` needs; ``gather_rows(src, index)`` returns src[index] (rows);
    ``experts(rows, expert_rows, gates)`` returns gate * FFN_e(row) for the
    expert-major rows [R, d] (fp32); ``combine(routed, y)`` returns out [T, d]
    from y [2T, d] in the routed permuted order."""

    def route_dispatch(self, x):
        raise NotImplementedError

    def gather_rows(self, src, index):
        raise NotImplementedError

    def experts(self, rows, expert_rows, gates):
        raise NotImplementedError

    def combine(self, routed, y):
        raise NotImplementedError

    def empty(self, shape, like):
        raise NotImplementedError


class DistExchange:
    """The exchanges over a torch.distributed process group (NCCL over NVLink
    between GPUs; gloo on the CPU): all-to-all with per-peer split sizes."""

    def __init__(self, group=None):
        import torch.distributed as dist

        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_to_all(self, out, inp, out_splits, in_splits):
        import torch.distributed as dist

        dist.all_to_all_single(out, inp, output_split_sizes=list(out_splits), input_split_sizes=list(in_splits),
                               group=self.group)
        return out


def exchange_counts(counts, exchange, E: int = E_TOTAL, device=None):
    """All-to-all of the per-expert counts: returns recv_counts [world, n]
    (host), row s = the counts GPU s holds for this GPU's experts."""
    import torch

    n = experts_per_rank(exchange.world, E)
    send = torch.tensor([int(v) for v in counts], dtype=torch.int64, device=device)
    recv = torch.empty(exchange.world * n, dtype=torch.int64, device=device)
    exchange.all_to_all(recv, send, [n] * exchange.world, [n] * exchange.world)
    return recv.cpu().numpy().reshape(exchange.world, n)


def ep_forward(x, compute: LocalCompute, exchange=None, E: int = E_TOTAL):
    """One expert-parallel forward of this GPU's tokens x [T, d]; every rank of
    the exchange calls it with its own batch (collective). ``exchange``: a
    ``DistExchange`` (default: the default process group). Returns out [T, d]."""
    import torch

    if exchange is None:
        exchange = DistExchange()
    routed = compute.route_dispatch(x)
    counts = routed["counts"]
    dev = routed["xp"].device
    recv_counts = exchange_counts(counts, exchange, E, device=dev)
    plan = make_plan(exchange.rank, exchange.world, counts, recv_counts, E)
    T2, d = routed["xp"].shape
    xrecv = compute.empty((plan.rows_in, d), routed["xp"])
    grecv = compute.empty((plan.rows_in,), routed["gate_perm"])
    exchange.all_to_all(xrecv, routed["xp"], plan.recv_rows, plan.send_rows)
    exchange.all_to_all(grecv, routed["gate_perm"], plan.recv_rows, plan.send_rows)
    idx = torch.as_tensor(plan.to_expert_major, dtype=torch.int32, device=dev)
    rows = compute.gather_rows(xrecv, idx)
    gates = compute.gather_rows(grecv.reshape(-1, 1), idx).reshape(-1)
    y_em = compute.experts(rows, plan.expert_rows, gates)
    inv = torch.as_tensor(plan.to_source_major, dtype=torch.int32, device=dev)
    y_src = compute.gather_rows(y_em, inv)
    y_back = compute.empty((T2, d), y_em)
    exchange.all_to_all(y_back, y_src, plan.send_rows, plan.recv_rows)
    return compute.combine(routed, y_back)


class LibraryCompute(LocalCompute):
    """The compute steps on this GPU through the library's C ABI. Holds the
    router weights (all experts' routing) and the weights of this GPU's
    experts only: w_gate, w_up [n, d, f], w_down [n, f, d] (and the int8
    scales [n, f], [n, f], [n, d])."""

    def __init__(self, w_router, w_gate, w_up, w_down, scales=None, router_bias=None, activation=0,
                 renormalize=False, path=0, down_splits=0):
        from . import _native as N

        self.N = N
        self.w_router, self.w_gate, self.w_up, self.w_down = w_router, w_gate, w_up, w_down
        self.scales, self.router_bias = scales, router_bias
        self.activation, self.renormalize = activation, renormalize
        self.path, self.down_splits = path, down_splits
        self.n = w_gate.shape[0]
        self._small = None

    def _check(self, st, what):
        from . import MoeError

        if st != self.N.MOE_OK:
            raise MoeError(st, what)

    def _status_ws(self, device):
        import torch

        if self._small is None or self._small.device != device:
            self._small = torch.empty(256, dtype=torch.uint8, device=device)
        return self._small

    def empty(self, shape, like):
        import torch

        return torch.empty(shape, dtype=like.dtype, device=like.device)

    def route_dispatch(self, x):
        import torch

        from . import _ptr, _stream, dtype_code

        T, d = x.shape
        dev = x.device
        dt = dtype_code(x, self.w_gate)
        xp_dtype = torch.float16 if dt == self.N.MOE_BF16_INT8W else x.dtype
        r = {
            "idx": torch.empty((T, 2), dtype=torch.int32, device=dev),
            "gates": torch.empty((T, 2), dtype=torch.float32, device=dev),
            "counts_dev": torch.empty(8, dtype=torch.int32, device=dev),
            "offsets": torch.empty(9, dtype=torch.int32, device=dev),
            "perm_token": torch.empty(2 * T, dtype=torch.int32, device=dev),
            "perm_slot": torch.empty(2 * T, dtype=torch.int32, device=dev),
            "slot_pos": torch.empty((T, 2), dtype=torch.int32, device=dev),
            "gate_perm": torch.empty(2 * T, dtype=torch.float32, device=dev),
            "xp": torch.empty((2 * T, d), dtype=xp_dtype, device=dev),
        }
        if T > 0:
            ws = torch.empty(self.N.lib().moe_route_workspace_size(T, d, dt), dtype=torch.uint8, device=dev)
            out = self.N.MoeRouted(*[_ptr(r[k]) for k in ("idx", "gates", "counts_dev", "offsets", "perm_token",
                                                           "perm_slot", "slot_pos", "gate_perm", "xp")])
            st = self.N.lib().moe_route_dispatch(_ptr(x), _ptr(self.w_router), _ptr(self.router_bias), T, d, dt,
                                                 int(bool(self.renormalize)), ctypes.byref(out), _ptr(ws),
                                                 ws.numel(), _stream(None))
            self._check(st, "moe_route_dispatch")
            r["counts"] = [int(v) for v in r["counts_dev"].cpu().tolist()]
        else:
            r["counts"] = [0] * 8
        r["T"], r["dtype"] = T, dt
        return r

    def gather_rows(self, src, index):
        import torch

        from . import _ptr, _stream

        n = index.shape[0]
        dst = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
        if n == 0:
            return dst
        row_bytes = src[0].numel() * src.element_size()
        ws = self._status_ws(src.device)
        st = self.N.lib().moe_gather_rows(_ptr(src), src.shape[0], _ptr(index), n, row_bytes, _ptr(dst), _ptr(ws),
                                          ws.numel(), _stream(None))
        self._check(st, "moe_gather_rows")
        return dst

    def experts(self, rows, expert_rows, gates):
        import torch

        from . import _options, _ptr, _scales, _stream

        R, d = rows.shape
        f = self.w_gate.shape[2]
        y = torch.empty((R, d), dtype=torch.float32, device=rows.device)
        if R == 0:
            return y
        dt = self._dtype()
        counts = torch.tensor(expert_rows, dtype=torch.int32, device=rows.device)
        size = self.N.lib().moe_experts_workspace_size(R, d, f, self.n, dt, self.path, self.down_splits)
        if size == 0:
            raise ValueError("moe_experts_forward: unsupported sizes")
        ws = torch.empty(size, dtype=torch.uint8, device=rows.device)
        sc = _scales(self.scales)
        a = self.N.MoeExpertRows(_ptr(rows), _ptr(counts), _ptr(gates), _ptr(self.w_gate), _ptr(self.w_up),
                                 _ptr(self.w_down), ctypes.pointer(sc) if sc is not None else None, _ptr(y),
                                 R, d, f, self.n, dt)
        opts, _ = _options(self.activation, None, self.path, self.down_splits, None, False, None, None, 1e-5)
        st = self.N.lib().moe_experts_forward(ctypes.byref(a), ctypes.byref(opts), _ptr(ws), ws.numel(),
                                              _stream(None))
        self._check(st, "moe_experts_forward")
        return y

    def _dtype(self):
        import torch

        if self.w_gate.dtype == torch.int8:
            return self.N.MOE_BF16_INT8W
        return self.N.MOE_F32 if self.w_gate.dtype == torch.float32 else self.N.MOE_BF16

    def combine(self, routed, y):
        import torch

        from . import _ptr, _stream

        T = routed["T"]
        d = y.shape[1]
        out_dtype = torch.float32 if routed["dtype"] == self.N.MOE_F32 else torch.bfloat16
        out = torch.empty((T, d), dtype=out_dtype, device=y.device)
        if T == 0:
            return out
        ws = self._status_ws(y.device)
        st = self.N.lib().moe_combine(_ptr(y), _ptr(routed["slot_pos"]), T, d, routed["dtype"], None, None, 1e-5,
                                      _ptr(out), _ptr(ws), ws.numel(), _stream(None))
        self._check(st, "moe_combine")
        return out
