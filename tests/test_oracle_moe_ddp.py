"""Oracle pins for the MoE alltoallv and the DDP bucket path."""
import numpy as np
import pytest

import synth
from oracle import collectives as C
from oracle import ddp, moe


def _routing(seed, n, tokens, experts):
    return [moe.route_topk(synth.normal_f32(seed, r, tokens * experts, stream=3).reshape(tokens, experts))
            for r in range(n)]


def test_top2_is_the_two_largest_with_ties_to_lower_id():
    logits = np.array([[0.5, 2.0, 2.0, -1.0], [3.0, 3.0, 3.0, 3.0], [-1, -2, -3, 7]], np.float32)
    assert moe.route_topk(logits).tolist() == [[1, 2], [0, 1], [3, 0]]


def test_top2_matches_brute_force():
    logits = synth.normal_f32(4, 0, 300 * 64).reshape(300, 64)
    ids = moe.route_topk(logits)
    for t in range(300):
        row = logits[t]
        best = max(range(64), key=lambda e: (row[e], -e))
        second = max((e for e in range(64) if e != best), key=lambda e: (row[e], -e))
        assert ids[t].tolist() == [best, second]


@pytest.mark.parametrize("n,tokens,experts_per_rank,hidden", [(8, 64, 8, 16), (4, 33, 2, 8), (1, 10, 4, 4), (3, 5, 1, 3)])
def test_dispatch_then_combine_is_identity_and_counts_conserve(n, tokens, experts_per_rank, hidden):
    E = n * experts_per_rank
    ids = _routing(2, n, tokens, E)
    toks = [synth.int32_uniform(3, r, tokens * hidden, -1000, 1000).reshape(tokens, hidden) for r in range(n)]
    recv, m1 = moe.dispatch(toks, ids, experts_per_rank)
    # per destination: every row routed to one of its experts arrives, exactly once
    table = moe.count_table(ids, E)
    for d in range(n):
        assert recv[d].shape[0] == table[:, d * experts_per_rank:(d + 1) * experts_per_rank].sum()
    assert sum(r.shape[0] for r in recv) == n * tokens * 2
    back, m2 = moe.combine(recv, ids, experts_per_rank)
    for s in range(n):
        for k in range(2):
            assert np.array_equal(back[s][:, k, :], toks[s])
    assert m1.sent == m2.recvd


def test_dispatch_block_order_is_local_expert_then_token_then_slot():
    n, tokens, epr = 2, 6, 2
    ids = [np.array([[1, 3], [0, 1], [3, 2], [1, 0], [2, 3], [0, 2]], np.int32),
           np.array([[2, 0], [3, 1], [0, 3], [1, 2], [3, 0], [2, 1]], np.int32)]
    toks = [np.arange(tokens, dtype=np.int32).reshape(tokens, 1) + 100 * s for s in range(n)]
    recv, _ = moe.dispatch(toks, ids, epr)
    # rank 0 holds experts 0, 1: from src 0, expert 0 rows (t1,k0),(t3,k1),(t5,k0) then
    # expert 1 rows (t0,k0),(t1,k1),(t3,k0); then src 1's block
    assert recv[0][:6, 0].tolist() == [1, 3, 5, 0, 1, 3]
    assert recv[0][6:, 0].tolist() == [100, 102, 104, 101, 103, 105]


def test_uniform_alltoall_is_the_transpose():
    """Lecture 09 §7.4 experiment 4, with rank i's j-th block routed to rank j."""
    n = 4
    ids = [np.array([[j, j] for j in range(n)], np.int32) for i in range(n)]
    toks = [np.array([[10 * i + j] for j in range(n)], np.int32) for i in range(n)]
    recv, _ = moe.dispatch(toks, ids, experts_per_rank=1)
    for j in range(n):
        assert recv[j][::2, 0].tolist() == [10 * i + j for i in range(n)]


# ---- DDP ------------------------------------------------------------------------------------------

def test_transformer_gradient_inventory():
    shapes = synth.transformer_grad_shapes()
    nums = [synth.numel(s) for _, s in shapes]
    assert len(nums) == 147 and sum(nums) == 109_632_000
    b = ddp.assign_buckets(nums)
    assert len(b) == 17
    assert sorted(i for m in b for i in m) == list(range(147))
    for m in b:
        size = sum(nums[i] for i in m) * 4
        assert size <= ddp.CAP_BYTES or len(m) == 1
    assert b[-1] == [0] and b[0][0] == 146  # embedding alone, last; lnf.b first


def test_bucket_assignment_small_cases():
    assert ddp.assign_buckets([10, 10, 10], 4, 80) == [[2, 1], [0]]
    assert ddp.assign_buckets([30, 1, 1], 4, 80) == [[2, 1], [0]]
    assert ddp.assign_buckets([1, 1, 1], 4, 12) == [[2, 1, 0]]
    assert ddp.assign_buckets([], 4, 12) == []


def test_ddp_average_is_ring_sum_times_one_eighth_and_close_to_fp64_mean():
    n = 8
    shapes = [(33, 8), (5,), (64,), (7, 7), (100,)]
    grads = [[synth.normal_f32(1, r, synth.numel(s), 1e-3, stream=i).reshape(s) for i, s in enumerate(shapes)]
             for r in range(n)]
    out, meshes = ddp.ddp_allreduce(grads, cap_bytes=600)
    buckets = ddp.assign_buckets([synth.numel(s) for s in shapes], 4, 600)
    for members in buckets:
        flats = [ddp.flatten(grads[r], members) for r in range(n)]
        s, _ = C.ring_allreduce(flats)
        want = s[0] * np.float32(0.125)
        got = np.concatenate([out[0][i].reshape(-1) for i in members])
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    for i, s in enumerate(shapes):
        x64 = np.stack([grads[r][i] for r in range(n)]).astype(np.float64)
        bound = (n - 1) * 2.0 ** -24 * np.abs(x64).sum(0) / n
        assert np.all(np.abs(out[3][i] - x64.mean(0)) <= bound + 1e-30)
