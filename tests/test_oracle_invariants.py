"""Oracle pins that do not come from the oracle itself: the pages' byte counts, the
AllReduce = ReduceScatter + AllGather identity, the N = 1 identity, brute-force int32
sums, an independent left-fold evaluator for the ring order, an fp64 error bound,
tree-shape invariants, sampling consistency, the threaded mesh with injected faults,
and planted mistakes that the pins must catch."""
import math

import numpy as np
import pytest

import synth
from oracle import collectives as C
from oracle import layout as L
from oracle.mesh import LockstepMesh, MeshTimeout, ProtocolError, ThreadedMesh


def _bits(a):
    return np.ascontiguousarray(a).view(np.uint32 if a.dtype == np.float32 else a.dtype)


def _spread_f32(seed, n, count):
    """fp32 values whose magnitudes span 2^-20..2^20, so that the bracketing of a sum
    shows in its rounding."""
    out = []
    for r in range(n):
        u = synth.uniform_f32(seed, r, count)
        e = synth.int32_uniform(seed, r, count, -20, 20, stream=1)
        out.append((u * np.exp2(e).astype(np.float32)).astype(np.float32))
    return out


# ---- byte counters (lecture 09 §4.4; from-scratch page table "每 rank 字节") --------------------

@pytest.mark.parametrize("n,count", [(2, 8), (4, 4096), (8, 800), (5, 35), (16, 64)])
def test_ring_allreduce_bytes_per_rank_is_2T_times_N_minus_1_over_N(n, count):
    xs = [np.ones(count, np.float32) for _ in range(n)]
    _, mesh = C.ring_allreduce(xs)
    T = count * 4
    assert all(s == 2 * T * (n - 1) // n for s in mesh.sent)
    assert all(r == 2 * T * (n - 1) // n for r in mesh.recvd)


@pytest.mark.parametrize("n,count", [(3, 10), (7, 100), (8, 1001), (64, 70)])
def test_ring_allreduce_bytes_ragged(n, count):
    """Ragged chunks: rank r sends every chunk but r+1 in reduce-scatter and every chunk
    but r+2 in allgather, so it sends 2T - |chunk r+1| - |chunk r+2| bytes."""
    xs = [np.ones(count, np.float32) for _ in range(n)]
    _, mesh = C.ring_allreduce(xs)
    b = L.chunk_bounds(count, n)
    size = [4 * (hi - lo) for lo, hi in b]
    for r in range(n):
        assert mesh.sent[r] == 2 * 4 * count - size[(r + 1) % n] - size[(r + 2) % n]


@pytest.mark.parametrize("n,count", [(4, 4096), (8, 800), (2, 2)])
def test_rs_and_ag_bytes_are_T_times_N_minus_1_over_N(n, count):
    T = 4 * count
    _, m1 = C.ring_reduce_scatter([np.ones(count, np.float32) for _ in range(n)])
    assert m1.sent == [T * (n - 1) // n] * n
    shards = [np.ones(count // n, np.float32) for _ in range(n)]
    _, m2 = C.ring_allgather(shards)
    assert m2.sent == [T * (n - 1) // n] * n


@pytest.mark.parametrize("n,root", [(1, 0), (2, 1), (4, 0), (7, 3), (16, 5), (17, 16)])
def test_broadcast_each_non_root_receives_T_once(n, root):
    x = np.arange(10, dtype=np.float32)
    out, mesh = C.broadcast(x, n, root)
    for r in range(n):
        assert np.array_equal(out[r], x)
        assert mesh.recvd[r] == (0 if r == root else x.nbytes)
    assert sum(mesh.sent) == (n - 1) * x.nbytes


@pytest.mark.parametrize("n", [2, 3, 4, 5, 8, 13, 16, 64])
def test_tree_bytes_match_own_schedule_and_stay_under_2T(n):
    count = 2 * n + 1
    xs = [np.ones(count, np.float32) for _ in range(n)]
    _, mesh = C.tree_allreduce(xs)
    mid = L.tree_half_split(count)
    halves = [4 * mid, 4 * (count - mid)]
    trees = [L.BinaryTree(n, False), L.BinaryTree(n, True)]
    for r in range(n):
        want = 0
        for t, h in zip(trees, halves):
            want += (h if t.parent[r] is not None else 0) + h * len(t.children(r))
        assert mesh.sent[r] == want
        # even N: every rank is a leaf in one tree, so it sends at most 2T (the 2M figure of
        # lecture 09 appendix A Q3); odd N: a rank can be interior in both trees (<= 3T)
        assert mesh.sent[r] <= (2 if n % 2 == 0 else 3) * 4 * count + 8


# ---- identities -----------------------------------------------------------------------------------

@pytest.mark.parametrize("n,count", [(2, 9), (3, 30), (4, 4096), (5, 17), (8, 1000), (13, 200), (4, 3)])
@pytest.mark.parametrize("scale", [1.0, 0.125, 1.0 / 3.0])
def test_allreduce_equals_allgather_of_reduce_scatter_bitwise(n, count, scale):
    """Lecture 09 §3.9: AllReduce = ReduceScatter + AllGather."""
    xs = _spread_f32(11, n, count)
    ar, _ = C.ring_allreduce(xs, scale=scale)
    rs, _ = C.ring_reduce_scatter(xs, scale=scale)
    ag, _ = C.ring_allgather(rs, count=count)
    for r in range(n):
        assert np.array_equal(_bits(ar[r]), _bits(ag[r]))


def test_n1_identity():
    x = _spread_f32(3, 1, 37)[0]
    for fn in (C.ring_allreduce, C.tree_allreduce):
        out, mesh = fn([x], scale=0.5)
        assert np.array_equal(_bits(out[0]), _bits(x * np.float32(0.5)))
        assert mesh.sent == [0] and mesh.messages == 0
    rs, _ = C.ring_reduce_scatter([x])
    assert np.array_equal(_bits(rs[0]), _bits(x))
    ag, _ = C.ring_allgather([x])
    assert np.array_equal(_bits(ag[0]), _bits(x))


# ---- int32 against brute force (any order gives the same wrapped sum) ----------------------------

@pytest.mark.parametrize("n,count", [(1, 5), (2, 7), (3, 101), (8, 999), (17, 33), (64, 130)])
def test_int32_sums_equal_brute_force(n, count):
    xs = [synth.int32_uniform(5, r, count, -2**31, 2**31 - 1) for r in range(n)]
    want = (np.sum(np.stack(xs).astype(np.int64), axis=0) & 0xFFFFFFFF).astype(np.uint32).view(np.int32)
    for fn in (C.ring_allreduce, C.tree_allreduce):
        out, _ = fn(xs, in_dtype="i32")
        for o in out:
            assert np.array_equal(o, want)
    rs, _ = C.ring_reduce_scatter(xs, in_dtype="i32")
    assert np.array_equal(np.concatenate(rs), want)
    red, _ = C.reduce(xs, root=n - 1, in_dtype="i32")
    assert np.array_equal(red, want)


# ---- ring fold order against an independent left-fold evaluator ---------------------------------

def _left_fold_expected(xs, count, origin_shift=0):
    """Element e of chunk c: ((x_c + x_{c+1}) + ...) + x_{c-1}, one fp32 add at a time,
    written from the closed form (not from the oracle's code)."""
    n = len(xs)
    q, r = divmod(count, n)
    out = np.empty(count, np.float32)
    for e in range(count):
        c = e // (q + 1) if e < r * (q + 1) else r + (e - r * (q + 1)) // q
        c = (c + origin_shift) % n
        acc = np.float32(xs[c][e])
        for j in range(1, n):
            acc = np.float32(acc + xs[(c + j) % n][e])
        out[e] = acc
    return out


def _ring_matches_left_fold(n, count, seed=7):
    xs = _spread_f32(seed, n, count)
    want = _left_fold_expected(xs, count)
    out, _ = C.ring_allreduce(xs)
    return all(np.array_equal(_bits(o), _bits(want)) for o in out)


@pytest.mark.parametrize("n,count", [(2, 10), (3, 31), (4, 64), (5, 23), (8, 96), (11, 50)])
def test_ring_fold_order_is_left_fold_from_origin_rank(n, count):
    assert _ring_matches_left_fold(n, count)


@pytest.mark.parametrize("n,count", [(4, 64), (8, 96)])
def test_left_fold_inputs_distinguish_origins(n, count):
    """The probe values are sensitive to the bracketing: another origin gives other bits."""
    xs = _spread_f32(7, n, count)
    a, b = _left_fold_expected(xs, count), _left_fold_expected(xs, count, origin_shift=1)
    assert not np.array_equal(_bits(a), _bits(b))


def test_planted_origin_mistake_is_caught(monkeypatch):
    """Plant an off-by-one in the oracle's send index (chunk r - s + 1 instead of r - s):
    the left-fold pin must fail."""
    def wrong_rs(ctx, buf, sl, op):
        r, n = ctx.rank, ctx.n
        for s in range(n - 1):
            ctx.send((r + 1) % n, buf[sl[(r - s + 1) % n]], tag=("rs", s))
            c_in = (r - s) % n
            incoming = yield from ctx.recv((r - 1) % n, tag=("rs", s))
            buf[sl[c_in]] = C.combine(buf[sl[c_in]], incoming, C.SUM)

    monkeypatch.setattr(C, "_ring_rs_phase", wrong_rs)
    assert not _ring_matches_left_fold(4, 64)


def test_planted_dropped_term_is_caught(monkeypatch):
    """Plant a dropped term (the receiver keeps its own value): brute force must fail."""
    real = C.combine

    def drop_first(local, incoming, op):
        return local.copy()

    monkeypatch.setattr(C, "combine", drop_first)
    xs = [synth.int32_uniform(1, r, 40, -100, 100) for r in range(4)]
    out, _ = C.ring_allreduce(xs, in_dtype="i32")
    monkeypatch.setattr(C, "combine", real)
    want = np.sum(np.stack(xs), axis=0, dtype=np.int32)
    assert not np.array_equal(out[0], want)


# ---- fp32 error bound against fp64 ---------------------------------------------------------------

@pytest.mark.parametrize("n,count", [(2, 1000), (8, 4096), (64, 640)])
def test_fp32_result_within_fp64_bound(n, count):
    xs = [synth.uniform_f32(9, r, count) for r in range(n)]
    x64 = np.stack(xs).astype(np.float64)
    exact, mag = x64.sum(0), np.abs(x64).sum(0)
    bound = (n - 1) * 2.0 ** -24 * mag
    for fn in (C.ring_allreduce, C.tree_allreduce):
        out, _ = fn(xs)
        assert np.all(np.abs(out[0].astype(np.float64) - exact) <= bound)


# ---- double binary tree ----------------------------------------------------------------------------

@pytest.mark.parametrize("n", list(range(1, 65)))
def test_tree_shape_invariants(n):
    for mirrored in (False, True):
        t = L.BinaryTree(n, mirrored)
        assert t.parent[t.root] is None
        assert sum(p is None for p in t.parent) == 1
        seen, stack = set(), [t.root]
        while stack:
            v = stack.pop()
            assert v not in seen
            seen.add(v)
            stack += t.children(v)
        assert seen == set(range(n))
        assert max(t.depth(r) for r in range(n)) <= math.ceil(math.log2(n)) + 1 if n > 1 else True
    if n % 2 == 0:
        a, b = L.BinaryTree(n, False), L.BinaryTree(n, True)
        for r in range(n):
            assert (not a.children(r)) + (not b.children(r)) == 1


def test_tree_shape_n8_example():
    """N = 8, tree A: root rank 7 <- 3 <- {1 <- {0, 2}, 5 <- {4, 6}}."""
    t = L.BinaryTree(8, False)
    assert t.root == 7 and t.children(7) == [3] and t.children(3) == [1, 5]
    assert t.children(1) == [0, 2] and t.children(5) == [4, 6]
    b = L.BinaryTree(8, True)
    assert b.root == 0 and b.children(0) == [4] and b.children(4) == [6, 2]


def _tree_recursive(xs, e, tree):
    def val(v):
        acc = np.float32(xs[v][e])
        if tree.left[v] is not None:
            acc = np.float32(val(tree.left[v]) + acc)
        if tree.right[v] is not None:
            acc = np.float32(acc + val(tree.right[v]))
        return acc
    return val(tree.root)


@pytest.mark.parametrize("n,count", [(2, 9), (3, 12), (6, 25), (8, 40), (13, 27)])
def test_tree_message_passing_equals_recursive_evaluation(n, count):
    xs = _spread_f32(21, n, count)
    out, _ = C.tree_allreduce(xs)
    mid = L.tree_half_split(count)
    ta, tb = L.BinaryTree(n, False), L.BinaryTree(n, True)
    for e in range(count):
        want = _tree_recursive(xs, e, ta if e < mid else tb)
        for o in out:
            assert _bits(o[e:e + 1])[0] == np.float32(want).view(np.uint32)


# ---- sampling: a subset of positions sees exactly the full run's operations -----------------------

@pytest.mark.parametrize("n,count", [(4, 1001), (8, 999), (5, 64)])
def test_positions_subset_matches_full_run(n, count):
    xs = _spread_f32(4, n, count)
    pos = np.unique(np.concatenate([[0, count - 1], np.arange(3, count, 37)]))
    for fn in (C.ring_allreduce, C.tree_allreduce):
        full, _ = fn(xs, scale=0.25)
        part, _ = fn([x[pos] for x in xs], scale=0.25, count=count, positions=pos)
        for r in range(n):
            assert np.array_equal(_bits(full[r][pos]), _bits(part[r]))
    ag_full, _ = C.ring_allgather([x[a:b] for x, (a, b) in zip(xs, L.chunk_bounds(count, n))], count=count)
    ag_part, _ = C.ring_allgather(
        [x[pos[(pos >= a) & (pos < b)]] for x, (a, b) in zip(xs, L.chunk_bounds(count, n))],
        count=count, positions=pos)
    assert np.array_equal(ag_full[0][pos], ag_part[0])


# ---- other primitives -------------------------------------------------------------------------------

@pytest.mark.parametrize("n,count", [(4, 16), (5, 23), (1, 3)])
def test_scatter_then_gather_round_trip(n, count):
    x = np.arange(count, dtype=np.float32) * 3
    parts, _ = C.scatter(x, n, root=n - 1)
    back, _ = C.gather(parts, root=n - 1)
    assert np.array_equal(back, x)


def test_bf16_input_widens_exactly():
    xs = [synth.to_bf16_bits(synth.normal_f32(2, r, 257)) for r in range(8)]
    wide = [synth.bf16_bits_to_f32(x) for x in xs]
    a, _ = C.ring_reduce_scatter(xs, in_dtype="bf16")
    b, _ = C.ring_reduce_scatter(wide, in_dtype="f32")
    for u, v in zip(a, b):
        assert np.array_equal(_bits(u), _bits(v))


@pytest.mark.parametrize("op", [C.MAX, C.MIN, C.PROD])
def test_other_ops_match_brute_force(op):
    n, count = 6, 50
    xs = [synth.int32_uniform(8, r, count, -9, 9) for r in range(n)]
    st = np.stack(xs).astype(np.int64)
    want = {C.MAX: st.max(0), C.MIN: st.min(0), C.PROD: np.prod(st, 0)}[op].astype(np.int32)
    out, _ = C.ring_allreduce(xs, op=op, in_dtype="i32")
    assert np.array_equal(out[0], want)
    f = [x.astype(np.float32) for x in xs]
    fo, _ = C.ring_allreduce(f, op=op)
    wf = {C.MAX: st.max(0), C.MIN: st.min(0), C.PROD: np.prod(st, 0)}[op].astype(np.float32)
    assert np.array_equal(fo[0], wf)


def test_max_orders_signed_zero_below_positive_zero():
    xs = [np.array([-0.0, 0.0, -0.0], np.float32), np.array([0.0, -0.0, -0.0], np.float32)]
    mx, _ = C.ring_allreduce(xs, op=C.MAX, count=3)
    mn, _ = C.ring_allreduce(xs, op=C.MIN, count=3)
    assert list(np.signbit(mx[0])) == [False, False, True]
    assert list(np.signbit(mn[0])) == [True, True, True]


# ---- threaded mesh: same results, timeouts and protocol errors instead of hangs --------------------

def test_threaded_mesh_matches_lockstep():
    xs = _spread_f32(6, 6, 301)
    for fn in (C.ring_allreduce, C.tree_allreduce):
        a, ma = fn(xs, mesh=LockstepMesh(6))
        b, mb = fn(xs, mesh=ThreadedMesh(6, recv_timeout_s=5.0))
        for u, v in zip(a, b):
            assert np.array_equal(_bits(u), _bits(v))
        assert ma.sent == mb.sent


def test_dropped_message_times_out():
    xs = [np.ones(40, np.float32) for _ in range(4)]
    drop = lambda src, dst, tag, seq: "drop" if (src, dst, tag) == (2, 3, ("rs", 1)) else None
    with pytest.raises(MeshTimeout):
        C.ring_allreduce(xs, mesh=ThreadedMesh(4, recv_timeout_s=0.3, fault=drop))


def test_duplicated_message_is_a_protocol_error():
    xs = [np.ones(40, np.float32) for _ in range(4)]
    dup = lambda src, dst, tag, seq: "dup" if (src, dst, tag) == (0, 1, ("ag", 0)) else None
    with pytest.raises(ProtocolError):
        C.ring_allreduce(xs, mesh=ThreadedMesh(4, recv_timeout_s=0.5, fault=dup))


def test_delayed_message_still_correct():
    xs = _spread_f32(2, 4, 64)
    delay = lambda src, dst, tag, seq: ("delay", 0.05) if src == 1 else None
    a, _ = C.ring_allreduce(xs)
    b, _ = C.ring_allreduce(xs, mesh=ThreadedMesh(4, recv_timeout_s=5.0, fault=delay))
    assert all(np.array_equal(_bits(u), _bits(v)) for u, v in zip(a, b))


def test_lockstep_deadlock_is_reported():
    mesh = LockstepMesh(2)

    def program(ctx):
        yield from ctx.recv(1 - ctx.rank)

    with pytest.raises(ProtocolError):
        mesh.run(program)


# ---- hierarchical allreduce (lecture 09 §9.3 Q1, appendix A Q4) ------------------------------------

HIER = [(8, 4), (16, 8), (6, 2), (9, 3), (4, 1), (4, 4), (64, 8), (12, 4)]


def _hier_expected(xs, G, count):
    """Written from the two-level closed form: within each node a left fold over local ranks
    starting at local chunk c; across nodes a left fold starting at sub-chunk j."""
    n = len(xs)
    M = n // G
    out = np.empty(count, np.float32)
    for e in range(count):
        a_c = b_c = c = 0
        for cc, (a, b) in enumerate(L.chunk_bounds(count, G)):
            if a <= e < b:
                c, a_c, b_c = cc, a, b
        j = next(jj for jj, (p, q) in enumerate(L.chunk_bounds(b_c - a_c, M)) if p <= e - a_c < q)
        outer = None
        for dm in range(M):
            m = (j + dm) % M
            inner = np.float32(xs[m * G + c][e])
            for dl in range(1, G):
                inner = np.float32(inner + xs[m * G + (c + dl) % G][e])
            outer = inner if outer is None else np.float32(outer + inner)
        out[e] = outer
    return out


@pytest.mark.parametrize("n,G", HIER)
def test_hierarchical_int32_equals_brute_force(n, G):
    count = 3 * n + 5
    xs = [synth.int32_uniform(31, r, count, -2**31, 2**31 - 1) for r in range(n)]
    want = (np.sum(np.stack(xs).astype(np.int64), axis=0) & 0xFFFFFFFF).astype(np.uint32).view(np.int32)
    out, _ = C.hierarchical_allreduce(xs, G, in_dtype="i32")
    assert all(np.array_equal(o, want) for o in out)


@pytest.mark.parametrize("n,G", [(8, 4), (6, 2), (9, 3), (12, 4)])
def test_hierarchical_fold_is_the_two_level_closed_form(n, G):
    count = 2 * n + 7
    xs = _spread_f32(33, n, count)
    out, _ = C.hierarchical_allreduce(xs, G)
    want = _hier_expected(xs, G, count)
    assert all(np.array_equal(_bits(o), _bits(want)) for o in out)
    flat, _ = C.ring_allreduce(xs)
    assert not np.array_equal(_bits(flat[0]), _bits(want))  # the probe tells the orders apart


@pytest.mark.parametrize("n", [4, 8])
def test_hierarchical_degenerates_to_the_flat_ring(n):
    xs = _spread_f32(35, n, 5 * n + 3)
    flat, _ = C.ring_allreduce(xs, scale=0.5)
    for G in (1, n):  # one rank per node, or a single node
        h, _ = C.hierarchical_allreduce(xs, G, scale=0.5)
        assert all(np.array_equal(_bits(a), _bits(b)) for a, b in zip(h, flat))


@pytest.mark.parametrize("n,G", [(16, 8), (64, 8), (8, 2)])
def test_hierarchical_cuts_cross_node_bytes_per_nic(n, G):
    """Appendix A Q4: per NIC, cross-node traffic falls by the node size: each rank sends
    2(M-1)/M * T/G across nodes instead of the flat ring's 2(N-1)/N * T on the node-boundary
    ranks."""
    M = n // G
    count = n * M * 4
    T = 4 * count
    xs = [np.ones(count, np.float32) for _ in range(n)]
    _, mh = C.hierarchical_allreduce(xs, G)
    assert mh.sent_off_node == [2 * (M - 1) * T // (M * G)] * n
    _, mf = C.ring_allreduce(xs, mesh=LockstepMesh(n, ranks_per_node=G))
    assert max(mf.sent_off_node) == 2 * (n - 1) * T // n
    assert max(mf.sent_off_node) / max(mh.sent_off_node) == pytest.approx(G * (n - 1) * M / (n * (M - 1)))


def test_hierarchical_within_fp64_bound_and_sampling():
    n, G, count = 16, 4, 5003
    xs = [synth.uniform_f32(36, r, count) for r in range(n)]
    out, _ = C.hierarchical_allreduce(xs, G, scale=1.0 / n)
    x64 = np.stack(xs).astype(np.float64)
    bound = ((n - 1) * 2.0 ** -24 * np.abs(x64).sum(0) + 2.0 ** -24 * np.abs(x64.sum(0))) / n
    assert np.all(np.abs(out[0].astype(np.float64) - x64.sum(0) / n) <= bound + 1e-30)
    pos = np.unique(np.concatenate([[0, count - 1], np.arange(1, count, 97)]))
    part, _ = C.hierarchical_allreduce([x[pos] for x in xs], G, scale=1.0 / n, count=count, positions=pos)
    assert np.array_equal(_bits(out[5][pos]), _bits(part[5]))
