"""The C ABI on the CPU: the library loads, exports every entry point include/cc.h declares,
rejects bad arguments before touching the GPU, and its host-only calls (chunk rule,
bucket assignment, workspace sizes) agree with the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from oracle import ddp
from oracle import layout as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cc.h")

cc = pytest.importorskip("collective_communication_primitives_rank_b200")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(cc.LIB_PATH):
        from collective_communication_primitives_rank_b200 import build
        build.build()
    return cc.get_lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^CC_API\s+[\w\s\*]+?\b(cc_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for want in ["cc_allreduce", "cc_reduce_scatter", "cc_allgather", "cc_broadcast", "cc_alltoallv",
                 "cc_bucket_flatten", "cc_bucket_unflatten", "cc_bucket_allreduce", "cc_reduce", "cc_scatter",
                 "cc_gather", "cc_route_topk", "cc_status_string", "cc_chunk"]:
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in cc._SIGS, f"binding lacks a signature for {name}"


def test_status_strings(lib):
    assert [lib.cc_status_string(i) for i in range(5)] == [
        b"CC_OK", b"CC_ERR_INVALID_ARG", b"CC_ERR_UNSUPPORTED", b"CC_ERR_CUDA", b"CC_ERR_TIMEOUT"]


@pytest.mark.parametrize("count,n", [(0, 1), (10, 4), (7, 8), (4096, 4), (1001, 64), (300_000_000, 8)])
def test_chunk_rule_matches_oracle(count, n):
    want = L.chunk_bounds(count, n)
    for c in range(n):
        a, ln = cc.cc_chunk(count, n, c)
        assert (a, a + ln) == want[c]


def test_bucket_assignment_matches_oracle(lib):
    nums = [synth.numel(s) for _, s in synth.transformer_grad_shapes()]
    assert cc.cc_bucket_assign(nums) == ddp.assign_buckets(nums)
    for cap in (40, 100, 1000):
        small = [5, 17, 3, 30, 1, 8, 0, 12]
        assert cc.cc_bucket_assign(small, 4, cap) == ddp.assign_buckets(small, 4, cap)
    assert cc.cc_bucket_assign([]) == []


def _pp(vals):
    return (ctypes.c_void_p * len(vals))(*vals)


FAKE = [0x10000 * (i + 1) for i in range(65)]  # never dereferenced: every call below must fail validation


@pytest.mark.parametrize("args,status", [
    (dict(nranks=0), cc.CC_ERR_INVALID_ARG),
    (dict(nranks=65), cc.CC_ERR_INVALID_ARG),
    (dict(in_t=cc.CC_F32, out_t=cc.CC_I32), cc.CC_ERR_INVALID_ARG),
    (dict(in_t=cc.CC_I32, out_t=cc.CC_F32), cc.CC_ERR_INVALID_ARG),
    (dict(in_t=cc.CC_BF16, out_t=cc.CC_BF16), cc.CC_ERR_INVALID_ARG),
    (dict(in_t=cc.CC_I32, out_t=cc.CC_I32, scale=0.5), cc.CC_ERR_INVALID_ARG),
    (dict(op=7), cc.CC_ERR_INVALID_ARG),
    (dict(algo=5), cc.CC_ERR_INVALID_ARG),
    (dict(in_t=cc.CC_I32, out_t=cc.CC_I32, scale=cc.CC_SCALE_MEAN), cc.CC_ERR_INVALID_ARG),  # no int mean
    (dict(null_at=2), cc.CC_ERR_INVALID_ARG),
    (dict(count=0), cc.CC_OK),
])
def test_allreduce_argument_validation(lib, args, status):
    n = args.get("nranks", 4)
    send = FAKE[:max(n, 1)]
    if "null_at" in args:
        send = list(send)
        send[args["null_at"]] = 0
    recv = FAKE[1:max(n, 1) + 1]
    st = lib.cc_allreduce(_pp(send), _pp(recv), n, args.get("count", 100), args.get("in_t", cc.CC_F32),
                          args.get("out_t", cc.CC_F32), args.get("op", cc.CC_SUM), args.get("algo", 0),
                          args.get("scale", 1.0), None)
    assert st == status


def test_in_place_with_widening_is_rejected(lib):
    p = _pp(FAKE[:4])
    assert lib.cc_allreduce(p, p, 4, 10, cc.CC_BF16, cc.CC_F32, cc.CC_SUM, 0, 1.0, None) == cc.CC_ERR_INVALID_ARG


def test_tree_reduce_scatter_is_unsupported(lib):
    st = lib.cc_reduce_scatter(_pp(FAKE[:4]), _pp(FAKE[4:8]), 4, 100, cc.CC_F32, cc.CC_F32, cc.CC_SUM,
                               cc.CC_ALGO_TREE, 1.0, None)
    assert st == cc.CC_ERR_UNSUPPORTED


def test_other_entry_points_validate(lib):
    p4 = _pp(FAKE[:4])
    assert lib.cc_broadcast(FAKE[0], p4, 4, 4, 10, cc.CC_F32, None) == cc.CC_ERR_INVALID_ARG  # root out of range
    assert lib.cc_reduce(p4, None, 4, 0, 10, cc.CC_F32, cc.CC_F32, cc.CC_SUM, 1.0, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_allgather(p4, p4, 4, 10, 9, None) == cc.CC_ERR_INVALID_ARG  # dtype
    assert lib.cc_route_topk(p4, p4, 4, 10, 64, 9, None) == cc.CC_ERR_INVALID_ARG  # topk > 8
    ws = lib.cc_alltoallv_workspace_size(8, 8192, 2, 8)
    assert ws > 0
    # misaligned workspace, bad row size, too small workspace, bad direction
    assert lib.cc_alltoallv(p4, p4, 4, 64, p4, 10, 2, 2, 100, 0, FAKE[0] + 8, ws, ws, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_alltoallv(p4, p4, 4, 60, p4, 10, 2, 2, 100, 0, FAKE[0], ws, ws, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_alltoallv(p4, p4, 4, 64, p4, 10, 2, 2, 100, 0, FAKE[0], 16, 16, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_alltoallv(p4, p4, 4, 64, p4, 10, 2, 2, 100, 2, FAKE[0], ws, ws, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_alltoallv_workspace_size(65, 10, 2, 2) == 0
    # the plan / run halves check what cc_alltoallv checks
    assert lib.cc_alltoallv_plan(p4, 4, 10, 9, 2, FAKE[0], ws, None) == cc.CC_ERR_INVALID_ARG      # topk > 8
    assert lib.cc_alltoallv_plan(None, 4, 10, 2, 2, FAKE[0], ws, None) == cc.CC_ERR_INVALID_ARG    # no ids
    assert lib.cc_alltoallv_plan(p4, 4, 10, 2, 2, FAKE[0] + 8, ws, None) == cc.CC_ERR_INVALID_ARG  # misaligned
    assert lib.cc_alltoallv_plan(p4, 4, 10, 2, 2, FAKE[0], 16, None) == cc.CC_ERR_INVALID_ARG      # too small
    assert lib.cc_alltoallv_run(p4, p4, 4, 60, p4, 10, 2, 2, 100, 0, FAKE[0], ws, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_alltoallv_run(p4, p4, 4, 64, p4, 10, 2, 2, 100, 2, FAKE[0], ws, None) == cc.CC_ERR_INVALID_ARG
    assert lib.cc_alltoallv_run(p4, p4, 4, 64, p4, 10, 2, 2, 100, 0, FAKE[0], 16, None) == cc.CC_ERR_INVALID_ARG
    sizes = (ctypes.c_size_t * 2)(10, 10)
    assert lib.cc_bucket_allreduce(p4, p4, 2, 2, sizes, 0, 0, 0.5, None) == cc.CC_ERR_INVALID_ARG  # cap 0
    assert lib.cc_bucket_allreduce(p4, p4, 2, 0, sizes, 100, 0, 0.5, None) == cc.CC_OK  # nothing to do


def test_binding_refuses_cpu_tensors():
    import torch
    x = [torch.zeros(8) for _ in range(2)]
    with pytest.raises(ValueError):
        cc.cc_allreduce(x, x)


def test_packed_detection_for_the_host_pipeline():
    # the host-buffer DDP step may merge copies across tensors only when, in every table, each
    # rank's tensors are views of one storage (one allocation)
    import torch
    flat = [torch.zeros(100) for _ in range(2)]
    views = [[f[0:30], f[30:100]] for f in flat]
    assert cc._packed(views, views) == 1
    separate = [[torch.zeros(30), torch.zeros(70)] for _ in range(2)]
    assert cc._packed(views, separate) == 0
    mixed = [[flat[0][0:30], torch.zeros(70)], [flat[1][0:30], flat[1][30:100]]]
    assert cc._packed(mixed) == 0


def test_multiring_ring_count_is_validated(lib):
    p = _pp(FAKE[:4])
    for k in (0, 65, -1):
        assert lib.cc_allreduce_multiring(p, p, 4, k, 10, cc.CC_F32, cc.CC_F32, cc.CC_SUM, 1.0, None) == \
            cc.CC_ERR_INVALID_ARG
    assert lib.cc_allreduce_multiring(p, p, 4, 2, 0, cc.CC_F32, cc.CC_F32, cc.CC_SUM, 1.0, None) == cc.CC_OK
