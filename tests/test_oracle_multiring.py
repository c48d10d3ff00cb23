"""Pins of the oracle's multi-ring allreduce (lecture 09 §5.3: several rings side by side, one
per NIC rail, for large cross-node messages). Reading: K rings, the message cut into K
contiguous parts by the chunk rule, ring k running the ring allreduce on part k, odd rings in
the opposite direction. Checked against an independent closed-form fold, brute-force int32
sums, the ring's per-rank byte count 2T(N-1)/N with the per-direction split, the reductions
to the plain ring (K = 1, or N = 2 where both directions fold the same pair), an fp64 bound,
sampling, and planted mistakes."""
import numpy as np
import pytest

import synth
from oracle import collectives as C


def _bits(a):
    return np.ascontiguousarray(a).view(np.uint32 if a.dtype == np.float32 else a.dtype)


def _spread_f32(seed, n, count):
    out = []
    for r in range(n):
        u = synth.uniform_f32(seed, r, count)
        e = synth.int32_uniform(seed, r, count, -20, 20, stream=1)
        out.append((u * np.exp2(e).astype(np.float32)).astype(np.float32))
    return out


def _split(length, parts, i):
    """[start, stop) of part i when `length` elements are cut into `parts` (first length %
    parts get one more), written out here from the rule, not taken from the oracle."""
    q, r = divmod(length, parts)
    start = i * q + min(i, r)
    return start, start + q + (1 if i < r else 0)


def _multiring_expected(xs, K, count, reverse_odd=True):
    n = len(xs)
    out = np.empty(count, np.float32)
    for k in range(K):
        a, b = _split(count, K, k)
        d = -1 if (reverse_odd and k % 2 == 1) else 1
        for c in range(n):
            ca, cb = _split(b - a, n, c)
            for e in range(a + ca, a + cb):
                acc = np.float32(xs[c][e])
                for j in range(1, n):
                    acc = np.float32(acc + xs[(c + d * j) % n][e])
                out[e] = acc
    return out


CASES = [(3, 2, 31), (4, 2, 64), (5, 3, 47), (8, 2, 96), (8, 4, 1001), (7, 5, 200), (16, 3, 160), (4, 8, 37)]


@pytest.mark.parametrize("n,K,count", CASES)
def test_multiring_fold_is_the_closed_form(n, K, count):
    xs = _spread_f32(51, n, count)
    out, _ = C.multiring_allreduce(xs, K)
    want = _multiring_expected(xs, K, count)
    for o in out:
        assert np.array_equal(_bits(o), _bits(want))


@pytest.mark.parametrize("n,K,count", [(4, 2, 64), (8, 3, 96)])
def test_probe_tells_the_ring_directions_apart(n, K, count):
    xs = _spread_f32(52, n, count)
    assert not np.array_equal(_bits(_multiring_expected(xs, K, count)),
                              _bits(_multiring_expected(xs, K, count, reverse_odd=False)))


@pytest.mark.parametrize("n,count", [(2, 17), (5, 33), (8, 100)])
def test_one_ring_is_the_plain_ring_and_two_ranks_ignore_direction(n, count):
    xs = _spread_f32(53, n, count)
    a, ma = C.multiring_allreduce(xs, 1, scale=0.25)
    b, mb = C.ring_allreduce(xs, scale=0.25)
    assert all(np.array_equal(_bits(u), _bits(v)) for u, v in zip(a, b)) and ma.sent == mb.sent
    two = _spread_f32(54, 2, count)
    ring, _ = C.ring_allreduce(two)
    for K in (2, 3, 4):
        mr, _ = C.multiring_allreduce(two, K)
        assert all(np.array_equal(_bits(u), _bits(v)) for u, v in zip(mr, ring))


def test_n1_identity():
    x = _spread_f32(55, 1, 23)[0]
    out, mesh = C.multiring_allreduce([x], 3, scale=0.5)
    assert np.array_equal(_bits(out[0]), _bits(x * np.float32(0.5))) and mesh.sent == [0]


@pytest.mark.parametrize("n,K,count", [(3, 2, 101), (8, 4, 999), (17, 3, 33), (64, 2, 130)])
def test_int32_sums_equal_brute_force(n, K, count):
    xs = [synth.int32_uniform(56, r, count, -2**31, 2**31 - 1) for r in range(n)]
    want = (np.sum(np.stack(xs).astype(np.int64), axis=0) & 0xFFFFFFFF).astype(np.uint32).view(np.int32)
    out, _ = C.multiring_allreduce(xs, K, in_dtype="i32")
    assert all(np.array_equal(o, want) for o in out)


@pytest.mark.parametrize("n,K", [(4, 2), (8, 2), (8, 4), (5, 3)])
def test_bytes_per_rank_and_per_direction(n, K):
    """Divisible sizes: every rank sends 2T(N-1)/N in all (lecture 09 §4.4), split between
    its two neighbours in proportion to the even and odd rings' parts."""
    count = n * K * 8
    T = 4 * count
    xs = [np.ones(count, np.float32) for _ in range(n)]
    _, mesh = C.multiring_allreduce(xs, K)
    Tk = T // K
    even, odd = (K + 1) // 2, K // 2
    for r in range(n):
        assert mesh.sent[r] == 2 * T * (n - 1) // n
        right, left = mesh.link_bytes[(r, (r + 1) % n)], mesh.link_bytes[(r, (r - 1) % n)]
        if n > 2:
            assert right == 2 * (n - 1) * even * Tk // n and left == 2 * (n - 1) * odd * Tk // n


@pytest.mark.parametrize("n,K,count", [(5, 2, 101), (8, 3, 999)])
def test_bytes_ragged_closed_form(n, K, count):
    """Rank r sends every chunk of a part but one in each phase: in an even ring it skips
    chunks r+1 and r+2, in an odd ring chunks r-1 and r-2."""
    xs = [np.ones(count, np.float32) for _ in range(n)]
    _, mesh = C.multiring_allreduce(xs, K)
    for r in range(n):
        want = 0
        for k in range(K):
            a, b = _split(count, K, k)
            size = [4 * (hi - lo) for lo, hi in (_split(b - a, n, c) for c in range(n))]
            d = 1 if k % 2 == 0 else -1
            want += 2 * 4 * (b - a) - size[(r + d) % n] - size[(r + 2 * d) % n]
        assert mesh.sent[r] == want


def test_fp32_within_fp64_bound_and_sampling():
    n, K, count = 8, 3, 4099
    xs = [synth.uniform_f32(57, r, count) for r in range(n)]
    out, _ = C.multiring_allreduce(xs, K)
    x64 = np.stack(xs).astype(np.float64)
    assert np.all(np.abs(out[0].astype(np.float64) - x64.sum(0)) <= (n - 1) * 2.0 ** -24 * np.abs(x64).sum(0))
    pos = np.unique(np.concatenate([[0, count - 1], np.arange(5, count, 61)]))
    part, _ = C.multiring_allreduce([x[pos] for x in xs], K, count=count, positions=pos)
    assert np.array_equal(_bits(out[3][pos]), _bits(part[3]))


def test_planted_mistakes_are_caught(monkeypatch):
    n, K, count = 6, 2, 90
    xs = _spread_f32(58, n, count)
    want = _multiring_expected(xs, K, count)
    # odd rings run forward like the even ones: the closed form must fail
    real_rs, real_ag = C._ring_rs_dir, C._ring_ag_dir
    monkeypatch.setattr(C, "_ring_rs_dir", lambda ctx, buf, sl, op, d, tag: real_rs(ctx, buf, sl, op, 1, tag))
    monkeypatch.setattr(C, "_ring_ag_dir", lambda ctx, buf, sl, d, tag: real_ag(ctx, buf, sl, 1, tag))
    out, _ = C.multiring_allreduce(xs, K)
    monkeypatch.undo()
    assert not np.array_equal(_bits(out[0]), _bits(want))
    # the parts cut by N instead of K
    real_cb = C.chunk_bounds
    monkeypatch.setattr(C, "chunk_bounds", lambda c, parts: real_cb(c, n if parts == K else parts))
    out, _ = C.multiring_allreduce(xs, K)
    monkeypatch.undo()
    assert not np.array_equal(_bits(out[0]), _bits(want))


def test_threaded_mesh_gives_the_lockstep_result():
    """One thread per rank with receive timeouts (the from-scratch page's queue mesh) runs the
    same multi-ring schedule to the same bits and byte counts."""
    from oracle.mesh import LockstepMesh, ThreadedMesh
    xs = _spread_f32(59, 6, 301)
    a, ma = C.multiring_allreduce(xs, 3, mesh=LockstepMesh(6))
    b, mb = C.multiring_allreduce(xs, 3, mesh=ThreadedMesh(6, recv_timeout_s=5.0))
    assert all(np.array_equal(_bits(u), _bits(v)) for u, v in zip(a, b))
    assert ma.sent == mb.sent and dict(ma.link_bytes) == dict(mb.link_bytes)
