"""Python binding of libcc, the B200 collective-primitives library (C ABI, include/cc.h).

Argument marshalling only: every function here turns torch tensors into the raw device
pointers, sizes and the current CUDA stream that the C entry point of the same name takes,
calls it, and raises CCError on a non-OK status. All computation happens in libcc's CUDA
kernels. There is no CPU path: the first call without a built libcc.so raises, and passing
a tensor that is not on the current CUDA device raises before any call.

    import collective_communication_primitives_rank_b200 as cc
    cc.cc_allreduce(send_tensors, recv_tensors, op="sum", algo="ring", scale=1.0)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcc.so")

_LIB = None

CC_OK, CC_ERR_INVALID_ARG, CC_ERR_UNSUPPORTED, CC_ERR_CUDA, CC_ERR_TIMEOUT = range(5)
CC_F32, CC_BF16, CC_I32 = 0, 1, 2
CC_SUM, CC_MAX, CC_MIN, CC_PROD = 0, 1, 2, 3
CC_ALGO_RING, CC_ALGO_TREE = 0, 1
MAX_RANKS = 64
# `scale` value that asks the library for the average over the ranks (it multiplies by
# fl(1/N) itself); the bucket calls pass it when scale is None
CC_SCALE_MEAN = float("nan")


def _scale(scale) -> float:
    return CC_SCALE_MEAN if scale is None else float(scale)

_vp, _sz, _i, _f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_PP = ctypes.POINTER(ctypes.c_void_p)
_I32P = ctypes.POINTER(ctypes.c_int32)
_SZP = ctypes.POINTER(ctypes.c_size_t)

_SIGS = {
    "cc_status_string": (ctypes.c_char_p, [_i]),
    "cc_version": (_i, []),
    "cc_chunk": (_i, [_sz, _i, _i, _SZP, _SZP]),
    "cc_async_status": (_i, [_i, _vp]),
    "cc_selftest_bounded_wait": (_i, [ctypes.c_uint, _vp]),
    "cc_allreduce": (_i, [_PP, _PP, _i, _sz, _i, _i, _i, _i, _f, _vp]),
    "cc_reduce_scatter": (_i, [_PP, _PP, _i, _sz, _i, _i, _i, _i, _f, _vp]),
    "cc_allreduce_stepped": (_i, [_PP, _PP, _i, _sz, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "cc_allreduce_hierarchical": (_i, [_PP, _PP, _i, _i, _sz, _i, _i, _i, _f, _vp]),
    "cc_allreduce_multiring": (_i, [_PP, _PP, _i, _i, _sz, _i, _i, _i, _f, _vp]),
    "cc_allgather": (_i, [_PP, _PP, _i, _sz, _i, _vp]),
    "cc_broadcast": (_i, [_vp, _PP, _i, _i, _sz, _i, _vp]),
    "cc_reduce": (_i, [_PP, _vp, _i, _i, _sz, _i, _i, _i, _f, _vp]),
    "cc_scatter": (_i, [_vp, _PP, _i, _i, _sz, _i, _vp]),
    "cc_gather": (_i, [_PP, _vp, _i, _i, _sz, _i, _vp]),
    "cc_route_topk": (_i, [_PP, _PP, _i, _i, _i, _i, _vp]),
    "cc_alltoallv_workspace_size": (_sz, [_i, _i, _i, _i]),
    "cc_alltoallv": (_i, [_PP, _PP, _i, _sz, _PP, _i, _i, _i, _sz, _i, _vp, _sz, _vp]),
    "cc_alltoallv_recv_counts": (_i, [_vp, _i, _vp, _vp]),
    "cc_alltoallv_plan": (_i, [_PP, _i, _i, _i, _i, _vp, _sz, _vp]),
    "cc_alltoallv_run": (_i, [_PP, _PP, _i, _sz, _PP, _i, _i, _i, _sz, _i, _vp, _sz, _vp]),
    "cc_alltoallv_noalloc": (_i, [_PP, _PP, _i, _sz, _PP, _i, _i, _i, _sz, _i, _vp, _vp]),
    "cc_bucket_assign": (_i, [_SZP, _i, _sz, _sz, _I32P, _I32P, _I32P]),
    "cc_bucket_flatten": (_i, [_PP, _SZP, _i, _vp, _i, _vp]),
    "cc_bucket_unflatten": (_i, [_vp, _PP, _SZP, _i, _i, _vp]),
    "cc_bucket_allreduce": (_i, [_PP, _PP, _i, _i, _SZP, _sz, _i, _f, _vp]),
    "cc_bucket_allreduce_host": (_i, [_PP, _PP, _PP, _PP, _i, _i, _SZP, _sz, _i, _f, _i, _vp]),
    "cc_bucket_allreduce_buckets": (_i, [_PP, _PP, _i, _i, _SZP, _sz, _i, _i, _i, _f, _vp]),
    "cc_allreduce_slice": (_i, [_PP, _PP, _i, _i, _sz, _i, _i, _i, _i, _f, _vp]),
    "cc_reduce_scatter_slice": (_i, [_PP, _vp, _i, _i, _sz, _i, _i, _i, _f, _vp]),
    "cc_allgather_slice": (_i, [_vp, _PP, _i, _i, _sz, _i, _vp]),
    "cc_ipc_handle_bytes": (_sz, []),
    "cc_ipc_export": (_i, [_vp, ctypes.c_char_p, _SZP]),
    "cc_ipc_open": (_i, [ctypes.c_char_p, _sz, _PP]),
    "cc_ipc_close": (_i, [_vp]),
}


def get_lib() -> ctypes.CDLL:
    """Load libcc.so (once) and declare every entry point's signature."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libcc.so not found at {LIB_PATH}; build it with "
                "`python -m collective_communication_primitives_rank_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


class _Lib:
    def __getattr__(self, name):
        return getattr(get_lib(), name)


lib = _Lib()


class CCError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.cc_status_string(status).decode()}")


def _check(status: int, where: str) -> None:
    if status != CC_OK:
        raise CCError(status, where)


_OPS = {"sum": CC_SUM, "max": CC_MAX, "min": CC_MIN, "prod": CC_PROD}
_ALGOS = {"ring": CC_ALGO_RING, "tree": CC_ALGO_TREE}


def _torch():
    import torch
    return torch


def dtype_code(t) -> int:
    torch = _torch()
    m = {torch.float32: CC_F32, torch.bfloat16: CC_BF16, torch.int32: CC_I32}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _dev_ptr(t) -> int:
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("libcc takes CUDA tensors only")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, current device is cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError("libcc takes contiguous tensors")
    return t.data_ptr()


def _ptrs(tensors: Sequence) -> ctypes.Array:
    return (ctypes.c_void_p * len(tensors))(*[_dev_ptr(t) for t in tensors])


def _stream(stream) -> Optional[int]:
    if stream is None:
        return _torch().cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _sizes(vals) -> ctypes.Array:
    return (ctypes.c_size_t * len(vals))(*[int(v) for v in vals])


def cc_async_status(reset: bool = False, stream=None) -> int:
    """Synchronizes the stream and returns CC_OK or CC_ERR_TIMEOUT (a device-side bounded
    wait gave up since the last reset)."""
    return int(lib.cc_async_status(1 if reset else 0, _stream(stream)))


def cc_chunk(count: int, nranks: int, c: int) -> tuple[int, int]:
    """(start, length) of ring chunk c (the library's chunk rule)."""
    a, n = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.cc_chunk(count, nranks, c, ctypes.byref(a), ctypes.byref(n)), "cc_chunk")
    return a.value, n.value


def _same(tensors, numel: int, dtype, what: str) -> None:
    for t in tensors:
        if t.numel() != numel or t.dtype != dtype:
            raise ValueError(f"{what}: every tensor must have {numel} elements of {dtype}")


def _ranks(tensors, what: str) -> int:
    n = len(tensors)
    if not 1 <= n <= MAX_RANKS:
        raise ValueError(f"{what}: 1..{MAX_RANKS} ranks, got {n}")
    return n


# ---- collectives -------------------------------------------------------------------------------

def cc_allreduce(send, recv, *, op="sum", algo="ring", scale=1.0, stream=None) -> None:
    """recv[r] = reduction of send[0..N-1] in `algo`'s fold order, times scale."""
    n = _ranks(send, "cc_allreduce")
    _same(send, send[0].numel(), send[0].dtype, "cc_allreduce send")
    _same(recv, send[0].numel(), recv[0].dtype, "cc_allreduce recv")
    if len(recv) != n:
        raise ValueError("cc_allreduce: one output per rank")
    _check(lib.cc_allreduce(_ptrs(send), _ptrs(recv), n, send[0].numel(), dtype_code(send[0]),
                            dtype_code(recv[0]), _OPS[op], _ALGOS[algo], _scale(scale), _stream(stream)),
           "cc_allreduce")


def cc_allreduce_hierarchical(send, recv, ranks_per_node: int, *, op="sum", scale=1.0, stream=None) -> None:
    """recv[r] = what the intra-node RS -> inter-node ring AR -> intra-node AG schedule leaves."""
    n = _ranks(send, "cc_allreduce_hierarchical")
    _same(send, send[0].numel(), send[0].dtype, "cc_allreduce_hierarchical send")
    _same(recv, send[0].numel(), recv[0].dtype, "cc_allreduce_hierarchical recv")
    if len(recv) != n:
        raise ValueError("cc_allreduce_hierarchical: one output per rank")
    _check(lib.cc_allreduce_hierarchical(_ptrs(send), _ptrs(recv), n, int(ranks_per_node), send[0].numel(),
                                         dtype_code(send[0]), dtype_code(recv[0]), _OPS[op], _scale(scale),
                                         _stream(stream)), "cc_allreduce_hierarchical")


def cc_allreduce_multiring(send, recv, nrings: int, *, op="sum", scale=1.0, stream=None) -> None:
    """recv[r] = what nrings rings side by side leave (part k of the buffer on ring k, odd
    rings in the opposite direction), times scale."""
    n = _ranks(send, "cc_allreduce_multiring")
    _same(send, send[0].numel(), send[0].dtype, "cc_allreduce_multiring send")
    _same(recv, send[0].numel(), recv[0].dtype, "cc_allreduce_multiring recv")
    if len(recv) != n:
        raise ValueError("cc_allreduce_multiring: one output per rank")
    _check(lib.cc_allreduce_multiring(_ptrs(send), _ptrs(recv), n, int(nrings), send[0].numel(), dtype_code(send[0]),
                                      dtype_code(recv[0]), _OPS[op], _scale(scale), _stream(stream)),
           "cc_allreduce_multiring")


def cc_allreduce_stepped(send, recv, workspace, *, op="sum", algo="ring", scale=1.0, stream=None) -> None:
    """cc_allreduce's result, computed by executing the schedule step by step (grid barrier
    between steps). `workspace`: a CUDA tensor of at least 256 bytes."""
    n = _ranks(send, "cc_allreduce_stepped")
    _same(send, send[0].numel(), send[0].dtype, "cc_allreduce_stepped send")
    _same(recv, send[0].numel(), recv[0].dtype, "cc_allreduce_stepped recv")
    if len(recv) != n:
        raise ValueError("cc_allreduce_stepped: one output per rank")
    _check(lib.cc_allreduce_stepped(_ptrs(send), _ptrs(recv), n, send[0].numel(), dtype_code(send[0]),
                                    dtype_code(recv[0]), _OPS[op], _ALGOS[algo], _scale(scale), _dev_ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "cc_allreduce_stepped")


def cc_reduce_scatter(send, recv, *, op="sum", algo="ring", scale=1.0, stream=None) -> None:
    """recv[c] = chunk c of the ring reduction of send[0..N-1]."""
    n = _ranks(send, "cc_reduce_scatter")
    _same(send, send[0].numel(), send[0].dtype, "cc_reduce_scatter send")
    if len(recv) != n:
        raise ValueError("cc_reduce_scatter: one output per rank")
    for c in range(n):
        _same([recv[c]], cc_chunk(send[0].numel(), n, c)[1], recv[0].dtype, f"cc_reduce_scatter recv[{c}]")
    _check(lib.cc_reduce_scatter(_ptrs(send), _ptrs(recv), n, send[0].numel(), dtype_code(send[0]),
                                 dtype_code(recv[0]), _OPS[op], _ALGOS[algo], _scale(scale), _stream(stream)),
           "cc_reduce_scatter")


def cc_allgather(send, recv, *, stream=None) -> None:
    """recv[r] = concatenation of send[0..N-1] (send[c] is chunk c of recv's length)."""
    n = _ranks(send, "cc_allgather")
    _same(recv, recv[0].numel(), recv[0].dtype, "cc_allgather recv")
    if len(recv) != n:
        raise ValueError("cc_allgather: one output per rank")
    for c in range(n):
        _same([send[c]], cc_chunk(recv[0].numel(), n, c)[1], recv[0].dtype, f"cc_allgather send[{c}]")
    _check(lib.cc_allgather(_ptrs(send), _ptrs(recv), len(send), recv[0].numel(), dtype_code(recv[0]),
                            _stream(stream)), "cc_allgather")


def cc_broadcast(src, recv, root: int = 0, *, stream=None) -> None:
    _ranks(recv, "cc_broadcast")
    _same(recv, src.numel(), src.dtype, "cc_broadcast recv")
    _check(lib.cc_broadcast(_dev_ptr(src), _ptrs(recv), len(recv), root, src.numel(), dtype_code(src),
                            _stream(stream)), "cc_broadcast")


def cc_reduce(send, recv_root, root: int = 0, *, op="sum", scale=1.0, stream=None) -> None:
    _ranks(send, "cc_reduce")
    _same(send, send[0].numel(), send[0].dtype, "cc_reduce send")
    _same([recv_root], send[0].numel(), recv_root.dtype, "cc_reduce recv_root")
    _check(lib.cc_reduce(_ptrs(send), _dev_ptr(recv_root), len(send), root, send[0].numel(), dtype_code(send[0]),
                         dtype_code(recv_root), _OPS[op], _scale(scale), _stream(stream)), "cc_reduce")


def cc_scatter(src, recv, root: int = 0, *, stream=None) -> None:
    n = _ranks(recv, "cc_scatter")
    for c in range(n):
        _same([recv[c]], cc_chunk(src.numel(), n, c)[1], src.dtype, f"cc_scatter recv[{c}]")
    _check(lib.cc_scatter(_dev_ptr(src), _ptrs(recv), len(recv), root, src.numel(), dtype_code(src),
                          _stream(stream)), "cc_scatter")


def cc_gather(send, recv_root, root: int = 0, *, stream=None) -> None:
    n = _ranks(send, "cc_gather")
    for c in range(n):
        _same([send[c]], cc_chunk(recv_root.numel(), n, c)[1], recv_root.dtype, f"cc_gather send[{c}]")
    _check(lib.cc_gather(_ptrs(send), _dev_ptr(recv_root), len(send), root, recv_root.numel(),
                         dtype_code(recv_root), _stream(stream)), "cc_gather")


# ---- MoE -----------------------------------------------------------------------------------------

def cc_route_topk(logits, expert_ids, *, stream=None) -> None:
    """expert_ids[r][t] = top-k expert ids of logits[r][t] (larger first, ties to lower id)."""
    torch = _torch()
    _ranks(logits, "cc_route_topk")
    tokens, experts = logits[0].shape
    _same(logits, tokens * experts, torch.float32, "cc_route_topk logits")
    _same(expert_ids, tokens * expert_ids[0].shape[1], torch.int32, "cc_route_topk expert_ids")
    if len(expert_ids) != len(logits):
        raise ValueError("cc_route_topk: one id tensor per rank")
    _check(lib.cc_route_topk(_ptrs(logits), _ptrs(expert_ids), len(logits), tokens, experts,
                             expert_ids[0].shape[1], _stream(stream)), "cc_route_topk")


def cc_alltoallv_workspace_size(nranks: int, tokens: int, topk: int, experts_per_rank: int) -> int:
    return int(lib.cc_alltoallv_workspace_size(nranks, tokens, topk, experts_per_rank))


def cc_alltoallv(send, recv, expert_ids, experts_per_rank: int, workspace, *, direction: int = 0,
                 row_bytes: Optional[int] = None, recv_capacity_rows: Optional[int] = None, stream=None) -> None:
    """direction 0: dispatch token rows to expert ranks; 1: combine them back.

    Dispatch: send[s] is [tokens, hidden]; recv[d] holds up to recv_capacity_rows rows.
    Combine: send[d] is rank d's dispatch output; recv[s] is [tokens, topk, hidden]."""
    _alltoallv(lib.cc_alltoallv, "cc_alltoallv", send, recv, expert_ids, experts_per_rank, workspace,
               direction, row_bytes, recv_capacity_rows, stream)


def _alltoallv(fn, name, send, recv, expert_ids, experts_per_rank, workspace, direction, row_bytes,
               recv_capacity_rows, stream) -> None:
    torch = _torch()
    n = _ranks(send, name)
    if len(recv) != n or len(expert_ids) != n:
        raise ValueError(f"{name}: one send, recv and id tensor per rank")
    tokens, topk = expert_ids[0].shape
    _same(expert_ids, tokens * topk, torch.int32, f"{name} expert_ids")
    tok = send if direction == 0 else recv
    if row_bytes is None:
        row_bytes = tok[0].numel() * tok[0].element_size() // max(1, tokens * (1 if direction == 0 else topk))
    rows_side = recv if direction == 0 else send
    cap = min(t.numel() * t.element_size() for t in rows_side) // row_bytes
    recv_capacity_rows = cap if recv_capacity_rows is None else min(cap, recv_capacity_rows)
    need = tokens * row_bytes * (1 if direction == 0 else topk)
    for t in tok:
        if t.numel() * t.element_size() < need:
            raise ValueError(f"{name}: token buffer smaller than tokens x row_bytes (x topk for combine)")
    if workspace.numel() * workspace.element_size() < cc_alltoallv_workspace_size(n, tokens, topk, experts_per_rank):
        raise ValueError(f"{name}: workspace too small")
    _check(fn(_ptrs(send), _ptrs(recv), len(send), row_bytes, _ptrs(expert_ids), tokens, topk, experts_per_rank,
              recv_capacity_rows, direction, _dev_ptr(workspace), workspace.numel() * workspace.element_size(),
              _stream(stream)), name)


def cc_alltoallv_plan(expert_ids, experts_per_rank: int, workspace, *, stream=None) -> None:
    """Builds in `workspace` the routing tables of expert_ids (one [tokens, topk] int32 tensor per
    rank), for any number of cc_alltoallv_run calls, dispatch or combine, over that routing."""
    torch = _torch()
    n = len(expert_ids)
    if n < 1:
        raise ValueError("cc_alltoallv_plan: no ranks")
    tokens, topk = expert_ids[0].shape
    _same(expert_ids, tokens * topk, torch.int32, "cc_alltoallv_plan expert_ids")
    if workspace.numel() * workspace.element_size() < cc_alltoallv_workspace_size(n, tokens, topk, experts_per_rank):
        raise ValueError("cc_alltoallv_plan: workspace too small")
    _check(lib.cc_alltoallv_plan(_ptrs(expert_ids), n, tokens, topk, experts_per_rank, _dev_ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "cc_alltoallv_plan")


def cc_alltoallv_run(send, recv, expert_ids, experts_per_rank: int, workspace, *, direction: int = 0,
                     row_bytes: Optional[int] = None, recv_capacity_rows: Optional[int] = None,
                     stream=None) -> None:
    """The row copy of cc_alltoallv alone, over the tables the last cc_alltoallv_plan (or
    cc_alltoallv) left in `workspace` for these same expert_ids; arguments as cc_alltoallv."""
    _alltoallv(lib.cc_alltoallv_run, "cc_alltoallv_run", send, recv, expert_ids, experts_per_rank, workspace,
               direction, row_bytes, recv_capacity_rows, stream)


def cc_alltoallv_recv_counts(workspace, nranks: int, out, *, stream=None) -> None:
    """Stream-ordered copy of the per-destination received row counts into `out` (int32;
    a CUDA tensor or a pinned host tensor)."""
    torch = _torch()
    if out.dtype != torch.int32 or out.numel() < nranks:
        raise ValueError("cc_alltoallv_recv_counts: out must hold nranks int32")
    if not out.is_cuda and not out.is_pinned():
        raise ValueError("cc_alltoallv_recv_counts: a host output must be pinned")
    ptr = out.data_ptr()
    _check(lib.cc_alltoallv_recv_counts(_dev_ptr(workspace), nranks, ptr, _stream(stream)),
           "cc_alltoallv_recv_counts")


# ---- DDP buckets ----------------------------------------------------------------------------------

def cc_bucket_assign(numels: Sequence[int], elem_bytes: int = 4, cap_bytes: int = 25 * 1024 * 1024):
    """Host call: returns the tensor ids of each bucket, buckets in launch order."""
    n = len(numels)
    order = (ctypes.c_int32 * max(1, n))()
    start = (ctypes.c_int32 * (n + 1))()
    nb = ctypes.c_int32()
    _check(lib.cc_bucket_assign(_sizes(numels) if n else None, n, elem_bytes, cap_bytes, order, start,
                                ctypes.byref(nb)), "cc_bucket_assign")
    return [[order[k] for k in range(start[b], start[b + 1])] for b in range(nb.value)]


def cc_bucket_flatten(tensors, bucket, *, stream=None) -> None:
    if sum(t.numel() for t in tensors) > bucket.numel() or any(t.dtype != bucket.dtype for t in tensors):
        raise ValueError("cc_bucket_flatten: bucket too small or dtype mismatch")
    _check(lib.cc_bucket_flatten(_ptrs(tensors), _sizes([t.numel() for t in tensors]), len(tensors),
                                 _dev_ptr(bucket), dtype_code(bucket), _stream(stream)), "cc_bucket_flatten")


def cc_bucket_unflatten(bucket, tensors, *, stream=None) -> None:
    if sum(t.numel() for t in tensors) > bucket.numel() or any(t.dtype != bucket.dtype for t in tensors):
        raise ValueError("cc_bucket_unflatten: bucket too small or dtype mismatch")
    _check(lib.cc_bucket_unflatten(_dev_ptr(bucket), _ptrs(tensors), _sizes([t.numel() for t in tensors]),
                                   len(tensors), dtype_code(bucket), _stream(stream)), "cc_bucket_unflatten")


def cc_bucket_allreduce(grads, out, *, cap_bytes: int = 25 * 1024 * 1024, algo="ring", scale=None,
                        stream=None) -> None:
    """grads[r][i] / out[r][i]: rank r's tensor i (registration order). One fused pass."""
    torch = _torch()
    n, nt = _ranks(grads, "cc_bucket_allreduce"), len(grads[0])
    if len(out) != n or any(len(row) != nt for row in list(grads) + list(out)):
        raise ValueError("cc_bucket_allreduce: grads and out must both be [nranks][ntensors]")
    for i in range(nt):
        _same([grads[r][i] for r in range(n)] + [out[r][i] for r in range(n)], grads[0][i].numel(),
              torch.float32, f"cc_bucket_allreduce tensor {i}")
    flat_in = [t for row in grads for t in row]
    flat_out = [t for row in out for t in row]
    _check(lib.cc_bucket_allreduce(_ptrs(flat_in), _ptrs(flat_out), n, nt, _sizes([t.numel() for t in grads[0]]),
                                   cap_bytes, _ALGOS[algo], _scale(scale), _stream(stream)), "cc_bucket_allreduce")


class BucketAllreducePlan:
    """cc_bucket_allreduce with the marshalling done once: the tensor tables are checked
    and turned into pointer arrays at construction, and run() is a bare C call. The
    tensors must stay alive (and keep their storage) while the plan is used."""

    def __init__(self, grads, out, *, cap_bytes: int = 25 * 1024 * 1024, algo="ring", scale=None):
        torch = _torch()
        n, nt = _ranks(grads, "BucketAllreducePlan"), len(grads[0])
        if len(out) != n or any(len(row) != nt for row in list(grads) + list(out)):
            raise ValueError("BucketAllreducePlan: grads and out must both be [nranks][ntensors]")
        for i in range(nt):
            _same([grads[r][i] for r in range(n)] + [out[r][i] for r in range(n)], grads[0][i].numel(),
                  torch.float32, f"BucketAllreducePlan tensor {i}")
        self._keep = (grads, out)
        self.n, self.nt = n, nt
        self._in = _ptrs([t for row in grads for t in row])
        self._out = _ptrs([t for row in out for t in row])
        self._numels = _sizes([t.numel() for t in grads[0]])
        self.cap_bytes = int(cap_bytes)
        self.algo = _ALGOS[algo]
        self.scale = _scale(scale)
        self._fn = get_lib().cc_bucket_allreduce

    def run(self, stream=None) -> None:
        st = self._fn(self._in, self._out, self.n, self.nt, self._numels, self.cap_bytes, self.algo, self.scale,
                      _stream(stream))
        if st != CC_OK:
            raise CCError(st, "cc_bucket_allreduce")

    def run_buckets(self, first: int, count: int = 1, stream=None) -> None:
        """Only buckets [first, first + count) of the plan's assignment (for overlap with
        backward: launch each bucket on a side stream once its gradients exist)."""
        st = get_lib().cc_bucket_allreduce_buckets(self._in, self._out, self.n, self.nt, self._numels, self.cap_bytes,
                                                   int(first), int(count), self.algo, self.scale, _stream(stream))
        if st != CC_OK:
            raise CCError(st, "cc_bucket_allreduce_buckets")


def _packed(*grids) -> int:
    """1 when, in every table, each rank's tensors are views of one storage (one allocation),
    the promise that lets cc_bucket_allreduce_host merge copies across tensors."""
    for grid in grids:
        for row in grid:
            if len({t.untyped_storage().data_ptr() for t in row}) > 1:
                return 0
    return 1


class BucketAllreduceHostPlan:
    """cc_bucket_allreduce_host with the marshalling done once (see BucketAllreducePlan)."""

    def __init__(self, host_grads, host_out, dev_grads, dev_out, *, cap_bytes: int = 25 * 1024 * 1024,
                 algo="ring", scale=None):
        torch = _torch()
        n, nt = _ranks(host_grads, "BucketAllreduceHostPlan"), len(host_grads[0])
        for grid in (host_out, dev_grads, dev_out):
            if len(grid) != n or any(len(row) != nt for row in grid):
                raise ValueError("BucketAllreduceHostPlan: all four tables must be [nranks][ntensors]")
        for i in range(nt):
            ts = [g[r][i] for g in (host_grads, host_out, dev_grads, dev_out) for r in range(n)]
            _same(ts, host_grads[0][i].numel(), torch.float32, f"BucketAllreduceHostPlan tensor {i}")
        for grid in (host_grads, host_out):
            for row in grid:
                for t in row:
                    if t.is_cuda or not t.is_contiguous():
                        raise ValueError("BucketAllreduceHostPlan: host tables hold contiguous CPU tensors")
        self._keep = (host_grads, host_out, dev_grads, dev_out)
        self.n, self.nt = n, nt
        hp = lambda grid: (ctypes.c_void_p * (n * nt))(*[t.data_ptr() for row in grid for t in row])
        self._hin, self._hout = hp(host_grads), hp(host_out)
        self._din = _ptrs([t for row in dev_grads for t in row])
        self._dout = _ptrs([t for row in dev_out for t in row])
        self._numels = _sizes([t.numel() for t in host_grads[0]])
        self.cap_bytes, self.algo = int(cap_bytes), _ALGOS[algo]
        self.scale = _scale(scale)
        self.packed = _packed(host_grads, host_out, dev_grads, dev_out)
        self._fn = get_lib().cc_bucket_allreduce_host

    def run(self, stream=None) -> None:
        st = self._fn(self._hin, self._hout, self._din, self._dout, self.n, self.nt, self._numels, self.cap_bytes,
                      self.algo, self.scale, self.packed, _stream(stream))
        if st != CC_OK:
            raise CCError(st, "cc_bucket_allreduce_host")


def cc_bucket_allreduce_host(host_grads, host_out, dev_grads, dev_out, *, cap_bytes: int = 25 * 1024 * 1024,
                             algo="ring", scale=None, stream=None) -> None:
    """The fused DDP step on host-resident gradients: host -> device copies, the fused
    allreduce, device -> host copies, all on one stream. host_* are CPU tensors (pin them
    for asynchronous copies); dev_* are CUDA staging tensors of the same shapes."""
    torch = _torch()
    n, nt = _ranks(host_grads, "cc_bucket_allreduce_host"), len(host_grads[0])
    for grid in (host_out, dev_grads, dev_out):
        if len(grid) != n or any(len(row) != nt for row in grid):
            raise ValueError("cc_bucket_allreduce_host: all four tables must be [nranks][ntensors]")
    for i in range(nt):
        ts = [g[r][i] for g in (host_grads, host_out, dev_grads, dev_out) for r in range(n)]
        _same(ts, host_grads[0][i].numel(), torch.float32, f"cc_bucket_allreduce_host tensor {i}")
    for r in range(n):
        for i in range(nt):
            if host_grads[r][i].is_cuda or host_out[r][i].is_cuda:
                raise ValueError("cc_bucket_allreduce_host: host tables must hold CPU tensors")
            if not (host_grads[r][i].is_contiguous() and host_out[r][i].is_contiguous()):
                raise ValueError("cc_bucket_allreduce_host: contiguous tensors only")
    hp = lambda grid: (ctypes.c_void_p * (n * nt))(*[t.data_ptr() for row in grid for t in row])
    _check(lib.cc_bucket_allreduce_host(hp(host_grads), hp(host_out),
                                        _ptrs([t for row in dev_grads for t in row]),
                                        _ptrs([t for row in dev_out for t in row]), n, nt,
                                        _sizes([t.numel() for t in host_grads[0]]), cap_bytes, _ALGOS[algo],
                                        _scale(scale), _packed(host_grads, host_out, dev_grads, dev_out),
                                        _stream(stream)), "cc_bucket_allreduce_host")


# ---- one rank per process: slices over peer-mapped buffers -----------------------------------

class PeerGroup:
    """Every rank's copy of some device tensors, mapped into this process.

    Each process of the torch.distributed group `group` (one per GPU; any backend) passes its
    own tensors, in the same order and of the same sizes on every rank. Their CUDA IPC
    handles are exchanged over the group, and the other ranks' allocations are opened with
    cc_ipc_open. buffers(i) is the list of the N ranks' copies of tensor i: this rank's
    tensor at its own index, device pointers (ints) of the peers' elsewhere, which the slice
    calls take. close() unmaps the peers; the tensors must stay alive until every rank has
    closed its group."""

    def __init__(self, tensors, group=None):
        dist = _torch().distributed
        self.rank = dist.get_rank(group)
        self.nranks = dist.get_world_size(group)
        self._tensors = list(tensors)
        hb = int(lib.cc_ipc_handle_bytes())
        mine = []
        for t in self._tensors:
            h = ctypes.create_string_buffer(hb)
            off = ctypes.c_size_t()
            _check(lib.cc_ipc_export(_dev_ptr(t), h, ctypes.byref(off)), "cc_ipc_export")
            mine.append((h.raw, off.value, t.numel(), str(t.dtype)))
        every = [None] * self.nranks
        dist.all_gather_object(every, mine, group=group)
        self._opened = []
        self._bufs = []
        try:
            for i, t in enumerate(self._tensors):
                row = []
                for r in range(self.nranks):
                    if r == self.rank:
                        row.append(t)
                        continue
                    h, off, numel, dt = every[r][i]
                    if numel != t.numel() or dt != str(t.dtype):
                        raise ValueError(f"PeerGroup: tensor {i} differs on rank {r} ({numel} x {dt})")
                    p = ctypes.c_void_p()
                    _check(lib.cc_ipc_open(h, off, ctypes.byref(p)), "cc_ipc_open")
                    self._opened.append(p.value)
                    row.append(p.value)
                self._bufs.append(row)
        except Exception:
            self.close()
            raise

    def buffers(self, i: int) -> list:
        return list(self._bufs[i])

    def close(self) -> None:
        while self._opened:
            lib.cc_ipc_close(self._opened.pop())


def _slice_ptrs(bufs, rank: int, what: str):
    """(pointer array, this rank's tensor) of N buffers: tensors of this process or peer
    device pointers (ints); the entry at `rank` must be a tensor."""
    torch = _torch()
    n = _ranks(bufs, what)
    if not 0 <= rank < n:
        raise ValueError(f"{what}: rank {rank} outside 0..{n - 1}")
    own = bufs[rank]
    if not isinstance(own, torch.Tensor):
        raise ValueError(f"{what}: entry {rank} (this rank) must be a tensor")
    vals = []
    for b in bufs:
        if isinstance(b, torch.Tensor):
            if b.numel() != own.numel() or b.dtype != own.dtype:
                raise ValueError(f"{what}: every buffer must have {own.numel()} elements of {own.dtype}")
            vals.append(_dev_ptr(b))
        else:
            vals.append(int(b))
    return (ctypes.c_void_p * n)(*vals), own


def cc_allreduce_slice(send, recv, rank: int, *, op="sum", algo="ring", scale=1.0, stream=None) -> None:
    """Rank `rank`'s share of cc_allreduce over N ranks' buffers (see PeerGroup): folds chunk
    `rank` from every send buffer and writes it into every recv buffer. After all N ranks
    have run it (ordered by the caller's barriers), every recv equals cc_allreduce's."""
    sp, s0 = _slice_ptrs(send, rank, "cc_allreduce_slice send")
    rp, r0 = _slice_ptrs(recv, rank, "cc_allreduce_slice recv")
    if len(recv) != len(send) or r0.numel() != s0.numel():
        raise ValueError("cc_allreduce_slice: one output per rank, as long as the input")
    _check(lib.cc_allreduce_slice(sp, rp, len(send), rank, s0.numel(), dtype_code(s0), dtype_code(r0), _OPS[op],
                                  _ALGOS[algo], _scale(scale), _stream(stream)), "cc_allreduce_slice")


def cc_reduce_scatter_slice(send, shard, rank: int, *, op="sum", scale=1.0, stream=None) -> None:
    """Rank `rank`'s share of cc_reduce_scatter: folds chunk `rank` of every send buffer into
    this rank's shard (a tensor of this process)."""
    sp, s0 = _slice_ptrs(send, rank, "cc_reduce_scatter_slice send")
    n = len(send)
    _same([shard], cc_chunk(s0.numel(), n, rank)[1], shard.dtype, "cc_reduce_scatter_slice shard")
    _check(lib.cc_reduce_scatter_slice(sp, _dev_ptr(shard), n, rank, s0.numel(), dtype_code(s0),
                                       dtype_code(shard), _OPS[op], _scale(scale), _stream(stream)),
           "cc_reduce_scatter_slice")


def cc_allgather_slice(shard, recv, rank: int, *, stream=None) -> None:
    """Rank `rank`'s share of cc_allgather: copies this rank's shard into chunk `rank` of
    every recv buffer."""
    rp, r0 = _slice_ptrs(recv, rank, "cc_allgather_slice recv")
    n = len(recv)
    _same([shard], cc_chunk(r0.numel(), n, rank)[1], r0.dtype, "cc_allgather_slice shard")
    _check(lib.cc_allgather_slice(_dev_ptr(shard), rp, n, rank, r0.numel(), dtype_code(r0), _stream(stream)),
           "cc_allgather_slice")


class PeerAllreduce:
    """Allreduce of one tensor per process across a torch.distributed group, one pass over
    NVLink: each rank folds its own chunk from all peers' inputs and writes it into all
    peers' outputs (cc_allreduce_slice). run() orders the ranks with a stream
    synchronisation and a group barrier before and after the slice."""

    def __init__(self, send, recv, group=None, *, op="sum", algo="ring", scale=1.0):
        self.group = group
        self.peers = PeerGroup([send, recv], group)
        self.op, self.algo, self.scale = op, algo, scale

    def run(self, stream=None) -> None:
        torch = _torch()
        s = stream if stream is not None else torch.cuda.current_stream()
        s.synchronize()
        torch.distributed.barrier(group=self.group)
        cc_allreduce_slice(self.peers.buffers(0), self.peers.buffers(1), self.peers.rank, op=self.op,
                           algo=self.algo, scale=self.scale, stream=s)
        s.synchronize()
        torch.distributed.barrier(group=self.group)

    def close(self) -> None:
        self.peers.close()


def raw_call(name: str, *args) -> int:
    """Call a C entry point with already-marshalled arguments (tests of the ABI itself)."""
    return getattr(lib, name)(*args)
