"""GPU parity for the MoE alltoallv path and the DDP bucket path, against the oracle."""
import numpy as np
import pytest

import synth
from oracle import collectives as C
from oracle import ddp, moe

from .helpers import Guarded, bits, to_dev, to_host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)
import collective_communication_primitives_rank_b200 as cc  # noqa: E402


def _logits(seed, n, tokens, experts):
    return [synth.normal_f32(seed, r, tokens * experts, stream=3).reshape(tokens, experts) for r in range(n)]


@pytest.mark.parametrize("n,tokens,experts,topk", [(8, 1000, 64, 2), (2, 33, 5, 1), (4, 257, 1024, 8), (1, 7, 3, 3)])
def test_route_topk_matches_oracle(n, tokens, experts, topk):
    lg = _logits(1, n, tokens, experts)
    lg[0][0, :4] = np.float32(1.5)     # ties: lower id first
    lg[0][1, :] = np.float32(0.0)
    lg[0][1, experts - 1] = np.float32(-0.0)
    ids = [torch.full((tokens, topk), -7, dtype=torch.int32, device="cuda") for _ in range(n)]
    cc.cc_route_topk([to_dev(x) for x in lg], ids)
    torch.cuda.synchronize()
    for r in range(n):
        assert np.array_equal(to_host(ids[r]), moe.route_topk(lg[r], topk))


def _moe_case(n, tokens, hidden, epr, seed=2):
    lg = _logits(seed, n, tokens, n * epr)
    ids = [moe.route_topk(x, 2) for x in lg]
    toks = [synth.to_bf16_bits(synth.normal_f32(seed, r, tokens * hidden, stream=4)).reshape(tokens, hidden)
            for r in range(n)]
    return ids, toks


# (4, 3000, 16, 256): 24 tiles x 1024 experts per source, more counts than the table kernel scans
# in shared memory, so the per-source prefix runs on its global-memory path
# (16, 300, 16, 64): 16 x 1024 totals, more than one CTA stages, so cc_alltoallv takes the
# separate table and copy launches instead of the single cooperative one
@pytest.mark.parametrize("n,tokens,hidden,epr", [(8, 300, 64, 8), (4, 1000, 8, 2), (3, 17, 16, 1), (1, 50, 8, 4),
                                                 (8, 2048, 4096, 8), (4, 3000, 16, 256), (2, 20000, 8, 4),
                                                 (5, 16384, 16, 6), (16, 300, 16, 64)])
def test_alltoallv_dispatch_and_combine_match_oracle(n, tokens, hidden, epr):
    ids, toks = _moe_case(n, tokens, hidden, epr)
    want, _ = moe.dispatch(toks, ids, epr)
    cap = max(w.shape[0] for w in want) + 5
    d_ids = [to_dev(i) for i in ids]
    d_tok = [to_dev(t) for t in toks]
    recv = [Guarded(cap * hidden, torch.bfloat16, shape=(cap, hidden)) for _ in range(n)]
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv(d_tok, [g.t for g in recv], d_ids, epr, ws, direction=0)
    counts = torch.zeros(n, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv_recv_counts(ws, n, counts)
    back = [Guarded(tokens * 2 * hidden, torch.bfloat16, shape=(tokens, 2, hidden)) for _ in range(n)]
    cc.cc_alltoallv([g.t for g in recv], [g.t for g in back], d_ids, epr, ws, direction=1)
    torch.cuda.synchronize()
    assert to_host(counts).tolist() == [w.shape[0] for w in want]
    combined, _ = moe.combine(want, ids, epr)
    for d in range(n):
        got = to_host(recv[d].t)[:want[d].shape[0]]
        assert np.array_equal(got, want[d]), f"dispatch rank {d}"
        recv[d].check()
    for s in range(n):
        assert np.array_equal(to_host(back[s].t), combined[s]), f"combine rank {s}"
        back[s].check()


@pytest.mark.parametrize("n,tokens,hidden,epr", [(8, 300, 64, 8), (3, 17, 16, 1), (4, 3000, 16, 256),
                                                 (16, 300, 16, 64)])
def test_alltoallv_plan_then_runs_match_oracle(n, tokens, hidden, epr):
    """One plan serves a dispatch and its combine, twice over; after the ids change, a new plan
    gives the new routing (the second routing is a different seed, same shape)."""
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    for seed in (3, 11):
        ids, toks = _moe_case(n, tokens, hidden, epr, seed=seed)
        want, _ = moe.dispatch(toks, ids, epr)
        combined, _ = moe.combine(want, ids, epr)
        cap = max(w.shape[0] for w in want) + 5
        d_ids = [to_dev(i) for i in ids]
        d_tok = [to_dev(t) for t in toks]
        cc.cc_alltoallv_plan(d_ids, epr, ws)
        counts = torch.zeros(n, dtype=torch.int32, device="cuda")
        cc.cc_alltoallv_recv_counts(ws, n, counts)
        for _ in range(2):
            recv = [Guarded(cap * hidden, torch.bfloat16, shape=(cap, hidden)) for _ in range(n)]
            back = [Guarded(tokens * 2 * hidden, torch.bfloat16, shape=(tokens, 2, hidden)) for _ in range(n)]
            cc.cc_alltoallv_run(d_tok, [g.t for g in recv], d_ids, epr, ws, direction=0)
            cc.cc_alltoallv_run([g.t for g in recv], [g.t for g in back], d_ids, epr, ws, direction=1)
            torch.cuda.synchronize()
            assert to_host(counts).tolist() == [w.shape[0] for w in want]
            for d in range(n):
                assert np.array_equal(to_host(recv[d].t)[:want[d].shape[0]], want[d]), f"dispatch rank {d}"
                recv[d].check()
            for s in range(n):
                assert np.array_equal(to_host(back[s].t), combined[s]), f"combine rank {s}"
                back[s].check()


@pytest.mark.parametrize("n,epr", [(4, 2), (8, 32), (16, 64), (64, 16)])
def test_alltoallv_without_tokens_reports_zero_rows(n, epr):
    """tokens = 0 at every size of the N x E totals (up to 64 ranks x 1024 experts): nothing
    is copied and the receive counts are zeros, whatever an earlier plan left in the workspace."""
    ids, _ = _moe_case(n, 40, 8, epr, seed=6)
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, 40, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv_plan([to_dev(i) for i in ids], epr, ws)
    ids1 = [torch.zeros(1, 2, dtype=torch.int32, device="cuda") for _ in range(n)]  # tokens = 0 below
    tok = [torch.zeros(1, 16, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    out = [torch.full((4, 16), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    st = cc.lib.cc_alltoallv(cc._ptrs(tok), cc._ptrs(out), n, 32, cc._ptrs(ids1), 0, 2, epr, 4, 0, ws.data_ptr(),
                             ws.numel() * 4, torch.cuda.current_stream().cuda_stream)
    assert st == cc.CC_OK
    counts = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv_recv_counts(ws, n, counts)
    torch.cuda.synchronize()
    assert counts.tolist() == [0] * n
    assert all(bool((o == 3.0).all()) for o in out)


def test_alltoallv_run_reads_rows_written_just_before_it():
    """A run launched right after the kernel that writes its send rows sees those rows: the
    rows are rewritten on the device between plan and run, with no host sync in between."""
    n, tokens, hidden, epr = 4, 4096, 2048, 4
    ids, toks = _moe_case(n, tokens, hidden, epr, seed=5)
    want, _ = moe.dispatch(toks, ids, epr)
    cap = max(w.shape[0] for w in want)
    d_ids = [to_dev(i) for i in ids]
    d_tok = [to_dev(t) for t in toks]
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    recv = [torch.empty(cap, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    stale = [torch.zeros_like(t) for t in d_tok]
    cc.cc_alltoallv_plan(d_ids, epr, ws)
    for s in range(n):
        stale[s].copy_(d_tok[s])          # device writes of the send rows, stream-ordered before the run
    cc.cc_alltoallv_run(stale, recv, d_ids, epr, ws, direction=0)
    torch.cuda.synchronize()
    for d in range(n):
        assert np.array_equal(to_host(recv[d])[:want[d].shape[0]], want[d]), f"dispatch rank {d}"


@pytest.mark.parametrize("n,tokens,epr", [(4, 700, 3), (2, 20000, 4), (4, 3000, 256), (16, 300, 64)])
def test_alltoallv_out_of_range_ids_route_nowhere(n, tokens, epr):
    """Ids below 0 or at / past N * experts_per_rank are sent to no rank (the oracle's send
    lists hold no such row); combine leaves their slots as they were."""
    hidden = 8
    ids, toks = _moe_case(n, tokens, hidden, epr, seed=13)
    E = n * epr
    rng = np.random.default_rng(4)
    for r in range(n):
        flat = ids[r].reshape(-1).copy()
        pick = rng.choice(flat.size, size=flat.size // 7, replace=False)
        flat[pick] = rng.choice(np.array([-1, -5, E, E + 3, 2 ** 31 - 1], dtype=np.int32), size=pick.size)
        ids[r] = flat.reshape(ids[r].shape)
    want, _ = moe.dispatch(toks, ids, epr)
    combined, _ = moe.combine(want, ids, epr)
    cap = max(w.shape[0] for w in want) + 2
    d_ids = [to_dev(i) for i in ids]
    recv = [Guarded(cap * hidden, torch.bfloat16, shape=(cap, hidden)) for _ in range(n)]
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv([to_dev(t) for t in toks], [g.t for g in recv], d_ids, epr, ws, direction=0)
    counts = torch.zeros(n, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv_recv_counts(ws, n, counts)
    back = [torch.full((tokens, 2, hidden), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    cc.cc_alltoallv([g.t for g in recv], back, d_ids, epr, ws, direction=1)
    torch.cuda.synchronize()
    assert to_host(counts).tolist() == [w.shape[0] for w in want]
    seven = to_host(torch.full((1,), 7.0, dtype=torch.bfloat16))[0]
    for d in range(n):
        assert np.array_equal(to_host(recv[d].t)[:want[d].shape[0]], want[d]), f"dispatch rank {d}"
        recv[d].check()
    for s in range(n):
        got = to_host(back[s])
        bad = (ids[s] < 0) | (ids[s] >= E)
        assert np.array_equal(got[~bad], combined[s][~bad]), f"combine rank {s}"
        assert (got[bad] == seven).all(), f"combine rank {s}: an unrouted slot was written"


def test_alltoallv_capacity_drops_overflow_rows_only():
    n, tokens, hidden, epr = 4, 200, 8, 2
    ids, toks = _moe_case(n, tokens, hidden, epr, seed=9)
    want, _ = moe.dispatch(toks, ids, epr)
    cap = min(w.shape[0] for w in want) - 3
    recv = [Guarded(cap * hidden, torch.bfloat16, shape=(cap, hidden)) for _ in range(n)]
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv([to_dev(t) for t in toks], [g.t for g in recv], [to_dev(i) for i in ids], epr, ws)
    counts = torch.zeros(n, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv_recv_counts(ws, n, counts)
    torch.cuda.synchronize()
    assert to_host(counts).tolist() == [w.shape[0] for w in want]
    for d in range(n):
        assert np.array_equal(to_host(recv[d].t), want[d][:cap])
        recv[d].check()


# ---- DDP buckets ----------------------------------------------------------------------------------------

def _small_model(n, seed=1, layers=2, d=64, ffn=256, vocab=500):
    shapes = synth.transformer_grad_shapes(layers, d, ffn, vocab)
    grads = [[synth.normal_f32(seed, r, synth.numel(s), 1e-3, stream=i).reshape(s)
              for i, (_, s) in enumerate(shapes)] for r in range(n)]
    return shapes, grads


@pytest.mark.parametrize("algo", ["ring", "tree"])
@pytest.mark.parametrize("n,cap", [(8, 40_000), (3, 100_000), (8, 25 * 1024 * 1024), (16, 7_000)])
def test_fused_bucket_allreduce_matches_oracle(algo, n, cap):
    shapes, grads = _small_model(n)
    want, _ = ddp.ddp_allreduce(grads, cap_bytes=cap, algo=algo)
    d_in = [[to_dev(g) for g in row] for row in grads]
    out = [[Guarded(g.size, torch.float32, shape=g.shape) for g in row] for row in grads]
    cc.cc_bucket_allreduce(d_in, [[o.t for o in row] for row in out], cap_bytes=cap, algo=algo)
    cc.cc_bucket_allreduce(d_in, d_in, cap_bytes=cap, algo=algo)  # in place
    torch.cuda.synchronize()
    for r in range(n):
        for i in range(len(shapes)):
            assert np.array_equal(bits(to_host(out[r][i].t)), bits(want[r][i])), f"rank {r} tensor {i}"
            assert np.array_equal(bits(to_host(d_in[r][i])), bits(want[r][i])), f"in place rank {r} tensor {i}"
            out[r][i].check()


def test_bucket_plan_matches_direct_call():
    n, cap = 8, 30_000
    shapes, grads = _small_model(n, seed=6)
    want, _ = ddp.ddp_allreduce(grads, cap_bytes=cap)
    d_in = [[to_dev(g) for g in row] for row in grads]
    out = [[torch.empty_like(t) for t in row] for row in d_in]
    plan = cc.BucketAllreducePlan(d_in, out, cap_bytes=cap)
    for _ in range(2):
        plan.run()
    torch.cuda.synchronize()
    for r in range(n):
        for i in range(len(shapes)):
            assert np.array_equal(bits(to_host(out[r][i])), bits(want[r][i]))


@pytest.mark.parametrize("cap", [30_000, 25 * 1024 * 1024])
def test_host_buffer_pipeline_matches_oracle(cap):
    n = 8
    shapes, grads = _small_model(n, seed=7)
    want, _ = ddp.ddp_allreduce(grads, cap_bytes=cap)
    h_in = [[torch.from_numpy(g).pin_memory() for g in row] for row in grads]
    h_out = [[torch.empty(g.shape, dtype=torch.float32).pin_memory() for g in row] for row in grads]
    d_in = [[torch.empty(g.shape, device="cuda") for g in row] for row in grads]
    d_out = [[torch.empty(g.shape, device="cuda") for g in row] for row in grads]
    plan = cc.BucketAllreduceHostPlan(h_in, h_out, d_in, d_out, cap_bytes=cap)
    for _ in range(2):
        plan.run()
    torch.cuda.synchronize()
    for r in range(n):
        for i in range(len(shapes)):
            assert np.array_equal(bits(h_out[r][i].numpy()), bits(want[r][i])), f"rank {r} tensor {i}"


@pytest.mark.parametrize("cap", [30_000, 25 * 1024 * 1024])
def test_host_buffer_pipeline_packed_matches_oracle(cap):
    # each rank's tensors are views of one flat buffer per table: the pipeline merges a
    # stage's contiguous copies across tensors; ~13.5M elements per rank make two stages
    n = 8
    shapes, grads = _small_model(n, seed=9, layers=3, d=512, ffn=2048, vocab=8000)
    want, _ = ddp.ddp_allreduce(grads, cap_bytes=cap)
    sizes = [g.size for g in grads[0]]
    offs = np.concatenate([[0], np.cumsum(sizes)])

    def views(flat):
        return [flat[offs[i]:offs[i + 1]] for i in range(len(sizes))]

    h_flat = [torch.from_numpy(np.concatenate([g.ravel() for g in row])).pin_memory() for row in grads]
    ho_flat = [torch.full((int(offs[-1]),), float("nan")).pin_memory() for _ in range(n)]
    d_flat = [torch.empty(int(offs[-1]), device="cuda") for _ in range(n)]
    do_flat = [torch.empty(int(offs[-1]), device="cuda") for _ in range(n)]
    plan = cc.BucketAllreduceHostPlan([views(h) for h in h_flat], [views(h) for h in ho_flat],
                                      [views(d) for d in d_flat], [views(d) for d in do_flat], cap_bytes=cap)
    assert plan.packed == 1
    plan.run()
    torch.cuda.synchronize()
    for r in range(n):
        got = views(ho_flat[r])
        for i in range(len(shapes)):
            assert np.array_equal(bits(got[i].numpy()), bits(want[r][i].ravel())), f"rank {r} tensor {i}"


def test_flatten_allreduce_unflatten_equals_fused():
    n, cap = 8, 60_000
    shapes, grads = _small_model(n, seed=4)
    want, _ = ddp.ddp_allreduce(grads, cap_bytes=cap)
    buckets = cc.cc_bucket_assign([g.size for g in grads[0]], 4, cap)
    assert buckets == ddp.assign_buckets([g.size for g in grads[0]], 4, cap)
    d_in = [[to_dev(g) for g in row] for row in grads]
    outs = [[torch.empty_like(t) for t in row] for row in d_in]
    for members in buckets:
        size = sum(grads[0][i].size for i in members)
        flats = [Guarded(size, torch.float32) for _ in range(n)]
        for r in range(n):
            cc.cc_bucket_flatten([d_in[r][i] for i in members], flats[r].t)
        red = [torch.empty(size, device="cuda") for _ in range(n)]
        cc.cc_allreduce([f.t for f in flats], red, scale=1.0 / n)
        for r in range(n):
            cc.cc_bucket_unflatten(red[r], [outs[r][i] for i in members])
        torch.cuda.synchronize()
        for r in range(n):
            flats[r].check()
            assert np.array_equal(to_host(flats[r].t), ddp.flatten(grads[r], members))
    for r in range(n):
        for i in range(len(shapes)):
            assert np.array_equal(bits(to_host(outs[r][i])), bits(want[r][i]))


def test_bucket_overlap_with_a_simulated_backward():
    """Backward writes the gradients bucket by bucket on the compute stream; each bucket's
    allreduce is launched on a side stream as soon as its gradients exist (event wait), while
    backward goes on. The result equals the oracle's whole-step allreduce."""
    n, cap = 8, 30_000
    shapes, grads = _small_model(n, seed=11)
    want, _ = ddp.ddp_allreduce(grads, cap_bytes=cap)
    src = [[to_dev(g) for g in row] for row in grads]  # what backward will produce
    d_in = [[torch.zeros_like(t) for t in row] for row in src]
    out = [[torch.empty_like(t) for t in row] for row in src]
    plan = cc.BucketAllreducePlan(d_in, out, cap_bytes=cap)
    buckets = cc.cc_bucket_assign([g.size for g in grads[0]], 4, cap)
    compute, comm = torch.cuda.current_stream(), torch.cuda.Stream()
    for b, members in enumerate(buckets):
        for r in range(n):
            for i in members:
                d_in[r][i].copy_(src[r][i])  # "backward" produces bucket b's gradients
        ready = torch.cuda.Event()
        ready.record(compute)
        comm.wait_event(ready)
        plan.run_buckets(b, 1, stream=comm)
    compute.wait_stream(comm)
    torch.cuda.synchronize()
    for r in range(n):
        for i in range(len(shapes)):
            assert np.array_equal(bits(to_host(out[r][i])), bits(want[r][i])), f"rank {r} tensor {i}"
