"""cc_alltoallv_noalloc: the alltoallv entry point for callers that cannot allocate device
memory (its routing scratch is a fixed array inside the library instead of a caller
workspace). It must give exactly what cc_alltoallv gives, call after call, although every
call reuses the same scratch array. Called here through the C ABI directly.

This file sorts last so that a run stopping at the first failure has run everything else
first; it also passes on its own in a fresh process (the first call sets the array up)."""
import ctypes

import numpy as np
import pytest

import synth
from oracle import moe

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)
import collective_communication_primitives_rank_b200 as cc  # noqa: E402


def _case(n, tokens, hidden, epr, seed):
    ids = [moe.route_topk(synth.normal_f32(seed, r, tokens * n * epr, stream=3).reshape(tokens, n * epr), 2)
           for r in range(n)]
    toks = [synth.to_bf16_bits(synth.normal_f32(seed, r, tokens * hidden, stream=4)).view(np.int16).reshape(tokens, hidden)
            for r in range(n)]
    d_ids = [torch.from_numpy(i).cuda() for i in ids]
    d_tok = [torch.from_numpy(t).cuda().view(torch.bfloat16) for t in toks]
    return d_ids, d_tok


def _pp(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def _noalloc(send, recv, ids, epr, cap, direction, counts):
    n = len(send)
    tokens, topk = ids[0].shape
    row_bytes = send[0].shape[-1] * 2
    st = cc.lib.cc_alltoallv_noalloc(_pp(send), _pp(recv), n, row_bytes, _pp(ids), tokens, topk, epr, cap,
                                     direction, counts.data_ptr() if counts is not None else None,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == cc.CC_OK, cc.lib.cc_status_string(st)


@pytest.mark.parametrize("shape", [[(8, 512, 64, 8, 1), (4, 300, 8, 2, 2)], [(8, 8192, 64, 8, 3), (2, 50, 16, 3, 4)]])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(shape):
    for n, tokens, hidden, epr, seed in shape:  # two calls in a row, different shapes
        ids, tok = _case(n, tokens, hidden, epr, seed)
        cap = tokens * 2 * n
        # the existing entry point, with a caller workspace
        ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
        ref = [torch.zeros(cap, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        cc.cc_alltoallv(tok, ref, ids, epr, ws, direction=0)
        ref_cnt = torch.zeros(n, dtype=torch.int32, device="cuda")
        cc.cc_alltoallv_recv_counts(ws, n, ref_cnt)
        ref_back = [torch.zeros(tokens, 2, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        cc.cc_alltoallv(ref, ref_back, ids, epr, ws, direction=1)
        # the allocation-free entry point
        got = [torch.zeros(cap, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        cnt = torch.full((n,), -1, dtype=torch.int32, device="cuda")
        _noalloc(tok, got, ids, epr, cap, 0, cnt)
        back = [torch.zeros(tokens, 2, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        _noalloc(got, back, ids, epr, cap, 1, None)
        torch.cuda.synchronize()
        assert torch.equal(cnt, ref_cnt)
        for d in range(n):
            assert torch.equal(got[d].view(torch.int16), ref[d].view(torch.int16)), f"dispatch rank {d}"
            assert torch.equal(back[d].view(torch.int16), ref_back[d].view(torch.int16)), f"combine rank {d}"
            for k in range(2):
                assert torch.equal(back[d][:, k].view(torch.int16), tok[d].view(torch.int16))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    n, tokens, epr = 8, 1 << 15, 8  # needs far more than 1 MiB of routing scratch
    assert cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) > (1 << 20)
    t = [torch.zeros(16, 8, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    ids = [torch.zeros(tokens, 2, dtype=torch.int32, device="cuda") for _ in range(n)]
    st = cc.lib.cc_alltoallv_noalloc(_pp(t), _pp(t), n, 16, _pp(ids), tokens, 2, epr, 16, 0, None,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == cc.CC_ERR_INVALID_ARG


def test_noalloc_with_no_tokens_reports_zero_rows():
    """tokens = 0: nothing is copied; the receive counts come back as zeros (the scratch is
    cleared by the call, whatever an earlier call left there)."""
    n, epr = 4, 2
    ids, tok = _case(n, 64, 16, epr, 5)  # an earlier call leaves non-zero tables in the scratch
    got = [torch.zeros(64 * 2 * n, 16, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    _noalloc(tok, got, ids, epr, 64 * 2 * n, 0, None)
    empty_ids = [torch.zeros(1, 2, dtype=torch.int32, device="cuda") for _ in range(n)]
    cnt = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    st = cc.lib.cc_alltoallv_noalloc(_pp(tok), _pp(got), n, 32, _pp(empty_ids), 0, 2, epr, 16, 0, cnt.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == cc.CC_OK
    assert cnt.tolist() == [0] * n


def test_noalloc_accepts_the_largest_shape_that_fits_and_rejects_the_next():
    """The 1 MiB limit at its edge: the largest token count whose routing scratch fits gives
    exactly cc_alltoallv's result; one token more is rejected before anything runs."""
    n, epr, hidden = 8, 8, 8
    size = lambda t: cc.cc_alltoallv_workspace_size(n, t, 2, epr)
    lo, hi = 1, 1 << 16
    assert size(lo) <= (1 << 20) < size(hi)
    while hi - lo > 1:  # the size grows with the token count
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if size(mid) <= (1 << 20) else (lo, mid)
    ids, tok = _case(n, lo, hidden, epr, 6)
    cap = lo * 2 * n
    ws = torch.empty(size(lo) // 4 + 64, dtype=torch.int32, device="cuda")
    ref = [torch.zeros(cap, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    cc.cc_alltoallv(tok, ref, ids, epr, ws, direction=0)
    got = [torch.zeros(cap, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    _noalloc(tok, got, ids, epr, cap, 0, None)
    torch.cuda.synchronize()
    for d in range(n):
        assert torch.equal(got[d].view(torch.int16), ref[d].view(torch.int16)), f"dispatch rank {d}"
    ids2, tok2 = _case(n, hi, hidden, epr, 7)  # buffers sized for the larger shape
    out2 = [torch.zeros(hi * 2, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    st = cc.lib.cc_alltoallv_noalloc(_pp(tok2), _pp(out2), n, hidden * 2, _pp(ids2), hi, 2, epr, hi * 2, 0, None,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == cc.CC_ERR_INVALID_ARG
