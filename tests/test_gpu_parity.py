"""GPU parity: libcc (through the C ABI, via the binding) against the oracle, element by
element, on seeded inputs. Bit-exact throughout: integer sums, every data movement, and
floating-point folds in the schedule's prescribed order."""
import numpy as np
import pytest

import synth
from oracle import collectives as C
from oracle import layout as L

from .helpers import Guarded, bits, misaligned, to_dev, to_host, torch_dtype

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)
import collective_communication_primitives_rank_b200 as cc  # noqa: E402


def _inputs(kind, n, count, seed=3):
    if kind == "f32":
        return [synth.uniform_f32(seed, r, count) for r in range(n)]
    if kind == "spread":  # magnitudes 2^-20..2^20: the bracketing shows in the rounding
        return [(synth.uniform_f32(seed, r, count) *
                 np.exp2(synth.int32_uniform(seed, r, count, -20, 20, stream=1)).astype(np.float32)).astype(np.float32)
                for r in range(n)]
    if kind == "i32":
        return [synth.int32_uniform(seed, r, count, -2**31, 2**31 - 1) for r in range(n)]
    if kind == "bf16":
        return [synth.to_bf16_bits(synth.normal_f32(seed, r, count, 1e-2)) for r in range(n)]
    raise ValueError(kind)


_IN = {"f32": "f32", "spread": "f32", "i32": "i32", "bf16": "bf16"}


def _out_dtype(kind):
    return torch.int32 if kind == "i32" else torch.float32


def _assert_same(got: np.ndarray, want: np.ndarray, what=""):
    g, w = bits(got), bits(want)
    if not np.array_equal(g, w):
        bad = np.flatnonzero(g != w)
        raise AssertionError(f"{what}: {bad.size} of {w.size} elements differ, first at {bad[:5]}: "
                             f"got {got[bad[:5]]} want {want[bad[:5]]}")


# ---- config 1: N = 4, 4096 elements, fp32 uniform[-1, 1] and int32 uniform[-1000, 1000] ------------------

@pytest.mark.parametrize("kind", ["f32", "i32"])
def test_config1_allreduce_reduce_scatter_allgather(kind):
    n, count = 4, 4096
    xs = [synth.uniform_f32(1, r, count) for r in range(n)] if kind == "f32" else \
        [synth.int32_uniform(1, r, count, -1000, 1000) for r in range(n)]
    send = [to_dev(x) for x in xs]
    want_ar, _ = C.ring_allreduce(xs, in_dtype=_IN[kind])
    out = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    cc.cc_allreduce(send, [o.t for o in out])
    want_rs, _ = C.ring_reduce_scatter(xs, in_dtype=_IN[kind])
    rs = [Guarded(count // n, _out_dtype(kind)) for _ in range(n)]
    cc.cc_reduce_scatter(send, [o.t for o in rs])
    ag = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    cc.cc_allgather([o.t for o in rs], [o.t for o in ag])
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r].t), want_ar[r], f"allreduce rank {r}")
        _assert_same(to_host(rs[r].t), want_rs[r], f"reduce_scatter rank {r}")
        _assert_same(to_host(ag[r].t), want_ar[r], f"allgather(reduce_scatter) rank {r}")
        for g in (out[r], rs[r], ag[r]):
            g.check()


# ---- allreduce across shapes, dtypes, ops and both algorithms -------------------------------------------

AR_CASES = [(1, 37), (2, 4096), (3, 1001), (4, 5), (5, 12345), (8, 8 * 1024 * 4 + 13), (13, 777),
            (16, 65536), (33, 2000), (64, 64 * 100 + 63), (64, 40), (7, 3)]


@pytest.mark.parametrize("n,count", AR_CASES)
@pytest.mark.parametrize("algo", ["ring", "tree"])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_allreduce_matches_oracle(n, count, algo, kind):
    xs = _inputs(kind, n, count)
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    scale = 1.0 if kind == "i32" else 1.0 / n
    want, _ = fn(xs, in_dtype=_IN[kind], scale=scale)
    out = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    cc.cc_allreduce([to_dev(x) for x in xs], [o.t for o in out], algo=algo, scale=scale)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r].t), want[r], f"{algo} {kind} N={n} rank {r}")
        out[r].check()


@pytest.mark.parametrize("op", ["max", "min", "prod"])
@pytest.mark.parametrize("algo", ["ring", "tree"])
@pytest.mark.parametrize("kind", ["spread", "i32"])
def test_other_ops_match_oracle(op, algo, kind):
    n, count = 6, 999
    xs = _inputs(kind, n, count, seed=8)
    if op == "prod" and kind == "spread":
        xs = [(1.0 + 0.01 * x).astype(np.float32) for x in _inputs("f32", n, count, seed=8)]
    xs[0][:7] = np.array([0.0, -0.0, 0.0, -0.0, 0, 0, 0], dtype=xs[0].dtype)
    xs[1][:7] = np.array([-0.0, 0.0, -0.0, -0.0, 0, 0, 0], dtype=xs[0].dtype)
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn(xs, op=op, in_dtype=_IN[kind])
    out = [torch.empty(count, dtype=_out_dtype(kind), device="cuda") for _ in range(n)]
    cc.cc_allreduce([to_dev(x) for x in xs], out, op=op, algo=algo)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r]), want[r], f"{op} {algo} rank {r}")


def test_allreduce_in_place_and_misaligned():
    n, count = 8, 10_003
    xs = _inputs("spread", n, count)
    want, _ = C.ring_allreduce(xs, scale=0.125)
    buf = [to_dev(x) for x in xs]
    cc.cc_allreduce(buf, buf, scale=0.125)
    mis = [misaligned(x) for x in xs]
    mout = [misaligned(np.zeros(count, np.float32)) for _ in range(n)]
    cc.cc_allreduce(mis, mout, scale=0.125)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(buf[r]), want[r], "in place")
        _assert_same(to_host(mout[r]), want[r], "misaligned")


def _shifted(a: np.ndarray, elems: int):
    """A CUDA tensor holding `a`, `elems` elements past a 16-byte boundary."""
    return to_dev(np.concatenate([np.zeros(elems, a.dtype), a]))[elems:]


@pytest.mark.parametrize("algo", ["ring", "tree"])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
@pytest.mark.parametrize("ss,sd", [(1, 1), (3, 3), (2, 2), (1, 0), (0, 3), (2, 1)])
def test_allreduce_reduce_scatter_and_reduce_with_shifted_buffers(algo, kind, ss, sd):
    """Sources `ss` and outputs `sd` elements past a 16-byte boundary: equal shifts take the
    16-byte units after an element-wise head (fp32 and int32; bf16 inputs with fp32 outputs
    keep the element path), unequal shifts the sources' units with element stores (sums), or
    the element path; every result bit for bit against the oracle, over several tiles and a
    ragged tail."""
    n, count = 8, 8 * 12_289 + 5
    xs = _inputs(kind, n, count, seed=31)
    scale = 1.0 if kind == "i32" else 0.125
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn(xs, in_dtype=_IN[kind], scale=scale)
    od = np.int32 if kind == "i32" else np.float32
    srcs = [_shifted(x, ss) for x in xs]
    outs = [_shifted(np.zeros(count, od), sd) for _ in range(n)]
    cc.cc_allreduce(srcs, outs, algo=algo, scale=scale)
    rs_want, _ = C.ring_reduce_scatter(xs, in_dtype=_IN[kind], scale=scale)
    shards = [_shifted(np.zeros(cc.cc_chunk(count, n, c)[1], od), sd) for c in range(n)]
    cc.cc_reduce_scatter(srcs, shards, scale=scale)
    red_want, _ = C.reduce(xs, 5, in_dtype=_IN[kind])
    root = _shifted(np.zeros(count, od), sd)
    cc.cc_reduce(srcs, root, 5)
    torch.cuda.synchronize()
    for r in (0, 3, n - 1):
        _assert_same(to_host(outs[r]), want[r], f"allreduce {algo} {kind} ({ss},{sd}) rank {r}")
    for c in range(n):
        _assert_same(to_host(shards[c]), rs_want[c], f"reduce-scatter {kind} ({ss},{sd}) shard {c}")
    _assert_same(to_host(root), red_want, f"reduce {kind} ({ss},{sd})")


@pytest.mark.parametrize("n", [2, 5, 8, 16])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
@pytest.mark.parametrize("offs,sd", [("mixed", 0), ("mixed", 2), ("one", 0), ("zero", 3), ("one", 2)])
def test_sums_with_sources_and_outputs_at_different_offsets(n, kind, offs, sd):
    """Sources at one offset from a 16-byte boundary and outputs at another take the sources'
    16-byte units with element stores (sums); sources at different offsets ("mixed": rank r
    r mod 4 elements past a boundary) take the element path. Ring, double binary tree,
    multi-ring and hierarchical allreduce, reduce-scatter (each shard at its own offset) and
    reduce to a root, bit for bit against the oracle over several tiles and a ragged tail, no
    write outside an output; a MAX over the same buffers (element path) as well."""
    count = n * 6_007 + 3
    xs = _inputs(kind, n, count, seed=33)
    scale = 1.0 if kind == "i32" else 0.125
    ss = [r % 4 if offs == "mixed" else 1 if offs == "one" else 0 for r in range(n)]
    srcs = [_shifted(x, s) for x, s in zip(xs, ss)]
    od = _out_dtype(kind)

    def outs():
        return [Guarded(count, od, misalign=sd) for _ in range(n)]

    cases = [("ring", lambda o: cc.cc_allreduce(srcs, o, algo="ring", scale=scale),
              C.ring_allreduce(xs, in_dtype=_IN[kind], scale=scale)[0]),
             ("tree", lambda o: cc.cc_allreduce(srcs, o, algo="tree", scale=scale),
              C.tree_allreduce(xs, in_dtype=_IN[kind], scale=scale)[0]),
             ("multiring", lambda o: cc.cc_allreduce_multiring(srcs, o, 2, scale=scale),
              C.multiring_allreduce(xs, 2, in_dtype=_IN[kind], scale=scale)[0])]
    if n % 4 == 0:
        cases.append(("hierarchical", lambda o: cc.cc_allreduce_hierarchical(srcs, o, 4, scale=scale),
                      C.hierarchical_allreduce(xs, 4, in_dtype=_IN[kind], scale=scale)[0]))
    for name, call, want in cases:
        out = outs()
        call([g.t for g in out])
        torch.cuda.synchronize()
        for r in range(n):
            _assert_same(to_host(out[r].t), want[r], f"{name} {kind} {offs}/{sd} N={n} rank {r}")
            out[r].check()
    rs_want, _ = C.ring_reduce_scatter(xs, in_dtype=_IN[kind], scale=scale)
    shards = [Guarded(cc.cc_chunk(count, n, c)[1], od, misalign=(sd + c) % 4) for c in range(n)]
    cc.cc_reduce_scatter(srcs, [g.t for g in shards], scale=scale)
    root = n // 2
    red_want, _ = C.reduce(xs, root, in_dtype=_IN[kind])
    red = Guarded(count, od, misalign=sd)
    cc.cc_reduce(srcs, red.t, root)
    mx_want, _ = C.ring_allreduce(xs, op="max", in_dtype=_IN[kind])
    mx = outs()
    cc.cc_allreduce(srcs, [g.t for g in mx], op="max")
    torch.cuda.synchronize()
    for c in range(n):
        _assert_same(to_host(shards[c].t), rs_want[c], f"reduce-scatter {kind} {offs}/{sd} N={n} shard {c}")
        shards[c].check()
    _assert_same(to_host(red.t), red_want, f"reduce {kind} {offs}/{sd} N={n}")
    red.check()
    for r in range(n):
        _assert_same(to_host(mx[r].t), mx_want[r], f"max {kind} {offs}/{sd} N={n} rank {r}")
        mx[r].check()


@pytest.mark.parametrize("n", [2, 5, 8])
@pytest.mark.parametrize("op", ["sum", "max"])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_in_place_with_per_rank_offsets(n, op, kind):
    """In-place allreduce (ring, tree, multi-ring) over buffers that sit at different offsets per
    rank (rank r: r mod 4 elements past a 16-byte boundary): the element paths, each element's
    column read and written by one thread. bf16 inputs are not in place (fp32 outputs)."""
    count = n * 5_003 + 1
    xs = _inputs(kind, n, count, seed=34)
    scale = 1.0 if kind == "i32" or op != "sum" else 0.25
    for algo, fn in (("ring", C.ring_allreduce), ("tree", C.tree_allreduce),
                     ("multiring", lambda v, **kw: C.multiring_allreduce(v, 3, **kw))):
        want, _ = fn(xs, op=op, in_dtype=_IN[kind], scale=scale)
        if kind == "bf16":
            bufs = [_shifted(x, r % 4) for r, x in enumerate(xs)]
            outs = [_shifted(np.zeros(count, np.float32), (r + 1) % 4) for r in range(n)]
        else:
            bufs = outs = [_shifted(x, r % 4) for r, x in enumerate(xs)]
        if algo == "multiring":
            cc.cc_allreduce_multiring(bufs, outs, 3, op=op, scale=scale)
        else:
            cc.cc_allreduce(bufs, outs, op=op, algo=algo, scale=scale)
        torch.cuda.synchronize()
        for r in range(n):
            _assert_same(to_host(outs[r]), want[r], f"in place {algo} {kind} {op} N={n} rank {r}")


def test_allreduce_empty_is_a_no_op():
    t = [torch.empty(0, device="cuda") for _ in range(4)]
    cc.cc_allreduce(t, t)
    torch.cuda.synchronize()


# ---- reduce-scatter / allgather ------------------------------------------------------------------------

@pytest.mark.parametrize("n,count", [(2, 9), (4, 4096), (5, 1003), (8, 8 * 4096), (8, 8 * 4096 + 5), (3, 2),
                                     (16, 160), (64, 64 * 33 + 17)])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_reduce_scatter_and_allgather_match_oracle(n, count, kind):
    xs = _inputs(kind, n, count)
    scale = 1.0 if kind == "i32" else 0.25
    want, _ = C.ring_reduce_scatter(xs, in_dtype=_IN[kind], scale=scale)
    lens = [b - a for a, b in L.chunk_bounds(count, n)]
    rs = [Guarded(ln, _out_dtype(kind)) for ln in lens]
    cc.cc_reduce_scatter([to_dev(x) for x in xs], [g.t for g in rs], scale=scale)
    ag = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    cc.cc_allgather([g.t for g in rs], [g.t for g in ag])
    want_ag, _ = C.ring_allgather(want, count=count)
    want_ar, _ = C.ring_allreduce(xs, in_dtype=_IN[kind], scale=scale)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(rs[r].t), want[r], f"RS shard {r}")
        _assert_same(to_host(ag[r].t), want_ag[r], f"AG rank {r}")
        _assert_same(to_host(ag[r].t), want_ar[r], f"AG(RS) == AR rank {r}")
        rs[r].check()
        ag[r].check()


def test_allgather_misaligned_shards_and_bf16_width():
    n, count = 4, 4 * 1000 + 3
    shards = [synth.to_bf16_bits(synth.normal_f32(2, r, b - a)) for r, (a, b) in enumerate(L.chunk_bounds(count, n))]
    want, _ = C.ring_allgather(shards, count=count)
    out = [Guarded(count, torch.bfloat16, misalign=1) for _ in range(n)]
    cc.cc_allgather([misaligned(s) for s in shards], [g.t for g in out])
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r].t), want[r])
        out[r].check()


# ---- broadcast, reduce, scatter, gather ------------------------------------------------------------------

@pytest.mark.parametrize("n,root,count", [(1, 0, 10), (4, 0, 4099), (7, 3, 100_000), (64, 63, 333),
                                          (64, 5, 64 * 1024 + 3), (16, 0, 3 * 512 + 1)])
def test_broadcast(n, root, count):
    x = synth.uniform_f32(5, 0, count)
    want, _ = C.broadcast(x, n, root)
    src = to_dev(x)
    out = [Guarded(count, torch.float32) for _ in range(n)]
    cc.cc_broadcast(src, [g.t for g in out], root)
    inplace = [src if r == root else torch.empty(count, device="cuda") for r in range(n)]
    cc.cc_broadcast(src, inplace, root)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r].t), want[r])
        _assert_same(to_host(inplace[r]), want[r])
        out[r].check()


# N = 2, 3: the binomial program is a left fold from the root (linear kernel); SUM at N = 4,
# 8, 16, 32, 64: the program compiled to straight-line code; other N and ops: the fold machines
@pytest.mark.parametrize("n,root", [(1, 0), (2, 1), (3, 2), (4, 0), (4, 3), (5, 3), (6, 0), (7, 6), (8, 5), (9, 4),
                                    (10, 9), (11, 1), (12, 7), (13, 12), (14, 2), (15, 8), (16, 9), (17, 3), (32, 31),
                                    (64, 17), (64, 0)])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
@pytest.mark.parametrize("count", [2049, 4 * 8192 + 7])
def test_reduce_to_root(n, root, kind, count):
    xs = _inputs(kind, n, count, seed=12)
    want, _ = C.reduce(xs, root, in_dtype=_IN[kind])
    out = Guarded(count, _out_dtype(kind))
    cc.cc_reduce([to_dev(x) for x in xs], out.t, root)
    torch.cuda.synchronize()
    _assert_same(to_host(out.t), want)
    out.check()


@pytest.mark.parametrize("n,count", [(4, 4), (4, 4099), (9, 100_001), (64, 70), (16, 16 * 2048 + 15),
                                     (3, 3 * 4096 * 7)])
def test_scatter_and_gather(n, count):
    x = synth.int32_uniform(6, 0, count, -5, 5)
    parts, _ = C.scatter(x, n, root=n - 1)
    out = [Guarded(p.size, torch.int32) for p in parts]
    cc.cc_scatter(to_dev(x), [g.t for g in out], n - 1)
    back = Guarded(count, torch.int32)
    cc.cc_gather([g.t for g in out], back.t, n - 1)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r].t), parts[r])
        out[r].check()
    _assert_same(to_host(back.t), x)
    back.check()


@pytest.mark.parametrize("n,shard", [(64, 4096), (64, 4096 + 13), (16, 512 * 7 + 1), (32, 511)])
@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_wide_allgather_spans_many_bulk_tiles(n, shard, kind):
    """Fan-out to many ranks with shards of several 2 KiB bulk tiles and a ragged last tile
    (every tile stored to all N outputs), bit for bit against the oracle's ring allgather."""
    count = n * shard
    shards = []
    for c in range(n):
        _, ln = cc.cc_chunk(count, n, c)
        x = synth.uniform_f32(8, c, ln)
        shards.append(synth.to_bf16_bits(x) if kind == "bf16" else x)
    want, _ = C.ring_allgather(shards)
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    out = [Guarded(count, dt) for _ in range(n)]
    cc.cc_allgather([to_dev(x) for x in shards], [g.t for g in out])
    torch.cuda.synchronize()
    for r in (0, n // 2, n - 1):
        _assert_same(to_host(out[r].t), want[r], f"allgather N={n} rank {r}")
        out[r].check()


def _off(a: np.ndarray, elems: int):
    """A CUDA tensor holding `a`, `elems` elements past a 16-byte boundary."""
    full = to_dev(np.concatenate([np.zeros(elems, a.dtype), a]))
    return full[elems:]


@pytest.mark.parametrize("kind", ["f32", "bf16"])
@pytest.mark.parametrize("shift_src,shift_dst", [(1, 1), (3, 3), (1, 2), (2, 0), (0, 1), (0, 3), (3, 1)])
def test_misaligned_copies_equal_or_unequal_offsets(kind, shift_src, shift_dst):
    """Allgather, scatter and gather with sources and destinations off 16-byte boundaries:
    equally misaligned (128-bit copies after a short head) or not (128-bit stores on the
    destinations' boundaries, each 16 bytes loaded element by element), large enough for several
    64 KiB tiles, bit for bit against the oracle."""
    n, count = 4, 4 * 70_001
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    def data(seed, r, ln):
        x = synth.uniform_f32(seed, r, ln)
        return synth.to_bf16_bits(x) if kind == "bf16" else x
    shards = [data(21, c, cc.cc_chunk(count, n, c)[1]) for c in range(n)]
    want, _ = C.ring_allgather(shards)
    zeros = np.zeros(count, np.uint16 if kind == "bf16" else np.float32)
    outs = [_off(zeros, shift_dst) for _ in range(n)]
    cc.cc_allgather([_off(x, shift_src) for x in shards], outs)
    x = data(22, 0, count)
    parts, _ = C.scatter(x, n, root=1)
    sc = [_off(np.zeros(p.size, zeros.dtype), shift_dst) for p in parts]
    cc.cc_scatter(_off(x, shift_src), sc, 1)
    back = _off(np.zeros(count, zeros.dtype), shift_src)
    cc.cc_gather(sc, back, 1)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(outs[r]), want[r], f"allgather rank {r}")
        _assert_same(to_host(sc[r]), parts[r], f"scatter rank {r}")
    _assert_same(to_host(back), x, "gather")


@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_copies_with_destinations_at_different_offsets(kind):
    """Allgather into outputs at different offsets from each other (rank r: r mod 4 elements
    past a 16-byte boundary: element copies) and from the shards, and broadcast / flatten /
    unflatten of odd-sized tensors whose places in the flat buffer fall at every offset
    (destination-aligned 128-bit stores per entry); guard bands around every output."""
    n, count = 5, 5 * 40_003 + 2
    dt = torch.bfloat16 if kind == "bf16" else torch.float32

    def data(seed, r, ln):
        x = synth.uniform_f32(seed, r, ln)
        return synth.to_bf16_bits(x) if kind == "bf16" else x
    shards = [data(23, c, cc.cc_chunk(count, n, c)[1]) for c in range(n)]
    want, _ = C.ring_allgather(shards)
    outs = [Guarded(count, dt, misalign=r % 4) for r in range(n)]
    cc.cc_allgather([_off(x, 1) for x in shards], [g.t for g in outs])
    x = data(24, 0, count)
    bwant, _ = C.broadcast(x, n, 2)
    bout = [Guarded(count, dt, misalign=3) for _ in range(n)]
    cc.cc_broadcast(_off(x, 2), [g.t for g in bout], 2)
    sizes = [70_001 + 13 * i for i in range(9)]
    ts = [data(25, i, m) for i, m in enumerate(sizes)]
    flat = Guarded(sum(sizes), dt, misalign=1)
    cc.cc_bucket_flatten([_off(t, i % 4) for i, t in enumerate(ts)], flat.t)
    back = [Guarded(m, dt, misalign=(i + 2) % 4) for i, m in enumerate(sizes)]
    cc.cc_bucket_unflatten(flat.t, [g.t for g in back])
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(outs[r].t), want[r], f"allgather rank {r}")
        outs[r].check()
        _assert_same(to_host(bout[r].t), bwant[r], f"broadcast rank {r}")
        bout[r].check()
    _assert_same(to_host(flat.t), np.concatenate(ts), "flatten")
    flat.check()
    for i in range(len(sizes)):
        _assert_same(to_host(back[i].t), ts[i], f"unflatten {i}")
        back[i].check()


# ---- failure detection on the device: a bounded wait that runs out reports, never hangs ----------

def test_bounded_wait_timeout_is_reported_and_the_context_survives():
    assert cc.cc_async_status(reset=True) in (cc.CC_OK, cc.CC_ERR_TIMEOUT)
    assert cc.cc_async_status() == cc.CC_OK
    st = cc.lib.cc_selftest_bounded_wait(20000, torch.cuda.current_stream().cuda_stream)  # 20 ms
    assert st == cc.CC_OK
    assert cc.cc_async_status() == cc.CC_ERR_TIMEOUT
    assert cc.cc_async_status(reset=True) == cc.CC_ERR_TIMEOUT
    assert cc.cc_async_status() == cc.CC_OK
    # the context still runs collectives correctly
    shards = [synth.uniform_f32(4, r, 1000) for r in range(4)]
    out = [torch.empty(4000, device="cuda") for _ in range(4)]
    cc.cc_allgather([to_dev(x) for x in shards], out)
    want, _ = C.ring_allgather(shards)
    torch.cuda.synchronize()
    for r in range(4):
        _assert_same(to_host(out[r]), want[r])
    assert cc.cc_async_status() == cc.CC_OK


# ---- stepped (schedule-faithful) allreduce: the same bits as the fused kernels -------------------------

@pytest.mark.parametrize("n,count", [(1, 37), (2, 4096), (3, 1001), (4, 4096), (5, 777), (8, 8 * 4096), (8, 999),
                                     (13, 2000), (16, 65536), (64, 64 * 40), (64, 70)])
@pytest.mark.parametrize("algo", ["ring", "tree"])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_stepped_allreduce_matches_oracle(n, count, algo, kind):
    xs = _inputs(kind, n, count, seed=15)
    scale = 1.0 if kind == "i32" else 1.0 / n
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn(xs, in_dtype=_IN[kind], scale=scale)
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    cc.cc_allreduce_stepped([to_dev(x) for x in xs], [o.t for o in out], ws, algo=algo, scale=scale)
    torch.cuda.synchronize()
    assert cc.cc_async_status() == cc.CC_OK
    for r in range(n):
        _assert_same(to_host(out[r].t), want[r], f"stepped {algo} {kind} N={n} rank {r}")
        out[r].check()


@pytest.mark.parametrize("op", ["max", "prod"])
def test_stepped_in_place_other_ops(op):
    n, count = 6, 4096
    xs = [(1.0 + 0.01 * x).astype(np.float32) for x in _inputs("f32", n, count, seed=16)]
    for algo in ("ring", "tree"):
        fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
        want, _ = fn(xs, op=op)
        buf = [to_dev(x) for x in xs]
        ws = torch.zeros(64, dtype=torch.int32, device="cuda")
        cc.cc_allreduce_stepped(buf, buf, ws, op=op, algo=algo)
        torch.cuda.synchronize()
        for r in range(n):
            _assert_same(to_host(buf[r]), want[r], f"stepped in place {op} {algo} rank {r}")


# ---- hierarchical allreduce: the two-level fold, fused ----------------------------------------------------

@pytest.mark.parametrize("n,G,count", [(8, 4, 4096), (16, 8, 16 * 1000 + 7), (6, 2, 999), (9, 3, 3001), (4, 1, 77),
                                       (4, 4, 4096), (64, 8, 64 * 50 + 13), (2, 1, 10), (12, 4, 12 * 4096)])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_hierarchical_allreduce_matches_oracle(n, G, count, kind):
    xs = _inputs(kind, n, count, seed=40)
    scale = 1.0 if kind == "i32" else 1.0 / n
    want, _ = C.hierarchical_allreduce(xs, G, in_dtype=_IN[kind], scale=scale)
    out = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    cc.cc_allreduce_hierarchical([to_dev(x) for x in xs], [o.t for o in out], G, scale=scale)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r].t), want[r], f"hierarchical {kind} N={n} G={G} rank {r}")
        out[r].check()


def test_hierarchical_in_place_and_large_sampled():
    n, G, count = 64, 8, 4 * 1024 * 1024 + 5
    xs = [synth.uniform_f32(41, r, count) for r in range(n)]
    buf = [to_dev(x) for x in xs]
    cc.cc_allreduce_hierarchical(buf, buf, G, scale=1.0 / n)
    torch.cuda.synchronize()
    pos = np.unique(np.concatenate([[0, count - 1], np.arange(3, count, 4099)]))
    want, _ = C.hierarchical_allreduce([x[pos] for x in xs], G, scale=1.0 / n, count=count, positions=pos)
    idx = torch.from_numpy(pos).cuda()
    for r in (0, 37, n - 1):
        _assert_same(buf[r][idx].cpu().numpy(), want[r], f"rank {r}")


# ---- CC_SCALE_MEAN: the library takes the average itself (fl(1/N) in binary32) -------------------------

@pytest.mark.parametrize("n", [3, 5, 6, 7, 8])
def test_scale_mean_sentinel_equals_explicit_reciprocal(n):
    count = 3 * 1024 + 5
    xs = _inputs("spread", n, count, seed=50)
    inv = float(np.float32(1) / np.float32(n))  # fl(1/N), one correctly rounded binary32 division
    send = [to_dev(x) for x in xs]
    for algo, fn in (("ring", C.ring_allreduce), ("tree", C.tree_allreduce)):
        want, _ = fn(xs, scale=inv)
        out = [torch.empty(count, device="cuda") for _ in range(n)]
        cc.cc_allreduce(send, out, algo=algo, scale=None)
        torch.cuda.synchronize()
        for r in range(n):
            _assert_same(to_host(out[r]), want[r], f"mean {algo} N={n} rank {r}")
    want_rs, _ = C.ring_reduce_scatter(xs, scale=inv)
    shards = [torch.empty(cc.cc_chunk(count, n, c)[1], device="cuda") for c in range(n)]
    cc.cc_reduce_scatter(send, shards, scale=None)
    want_red, _ = C.reduce(xs, n - 1)
    red = torch.empty(count, device="cuda")
    cc.cc_reduce(send, red, n - 1, scale=None)
    torch.cuda.synchronize()
    for c in range(n):
        _assert_same(to_host(shards[c]), want_rs[c], f"mean reduce-scatter N={n} shard {c}")
    _assert_same(to_host(red), (want_red * np.float32(inv)).astype(np.float32), f"mean reduce N={n}")


# ---- multi-ring allreduce: K rings side by side, odd rings reversed ---------------------------------------

@pytest.mark.parametrize("n,K,count", [(2, 2, 4096 + 3), (3, 2, 1001), (4, 3, 4096), (8, 2, 8 * 4096), (8, 4, 999),
                                       (13, 3, 2000), (16, 5, 65536 + 17), (64, 2, 64 * 40), (64, 4, 70), (8, 64, 1000),
                                       (5, 1, 777)])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_multiring_allreduce_matches_oracle(n, K, count, kind):
    xs = _inputs(kind, n, count, seed=60)
    scale = 1.0 if kind == "i32" else 1.0 / n
    want, _ = C.multiring_allreduce(xs, K, in_dtype=_IN[kind], scale=scale)
    out = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    cc.cc_allreduce_multiring([to_dev(x) for x in xs], [o.t for o in out], K, scale=scale)
    torch.cuda.synchronize()
    for r in range(n):
        _assert_same(to_host(out[r].t), want[r], f"multi-ring {kind} N={n} K={K} rank {r}")
        out[r].check()


def test_multiring_in_place_misaligned_and_large_sampled():
    n, K, count = 8, 4, 16 * 1024 * 1024 + 5
    xs = [synth.uniform_f32(61, r, count) for r in range(n)]
    buf = [to_dev(x) for x in xs]
    cc.cc_allreduce_multiring(buf, buf, K, scale=0.125)
    torch.cuda.synchronize()
    pos = np.unique(np.concatenate([[0, count - 1], np.arange(7, count, 4093)]))
    want, _ = C.multiring_allreduce([x[pos] for x in xs], K, scale=0.125, count=count, positions=pos)
    idx = torch.from_numpy(pos).cuda()
    for r in (0, 5, n - 1):
        _assert_same(buf[r][idx].cpu().numpy(), want[r], f"multi-ring in place rank {r}")
    small = _inputs("spread", 6, 3001, seed=62)
    want_s, _ = C.multiring_allreduce(small, 3)
    mis = [misaligned(x) for x in small]
    mout = [misaligned(np.zeros_like(x)) for x in small]
    cc.cc_allreduce_multiring(mis, mout, 3)
    torch.cuda.synchronize()
    for r in range(6):
        _assert_same(to_host(mout[r]), want_s[r], f"multi-ring misaligned rank {r}")


@pytest.mark.parametrize("n,count,kind", [(8, 8 * 1024 * 1024 + 5, "f32"), (3, 4 * 1024 * 1024 + 1, "bf16"),
                                          (64, 64 * 65536 + 63, "i32"), (2, 6 * 1024 * 1024, "f32")])
@pytest.mark.parametrize("algo", ["ring", "tree"])
def test_stepped_large_messages_sampled(n, count, kind, algo):
    """Messages whose phases run on the tile path (more units than the resident grid has
    threads), checked on sampled positions against the oracle's full-size chunk map."""
    xs = _inputs(kind, n, count, seed=17)
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = [torch.empty(count, dtype=_out_dtype(kind), device="cuda") for _ in range(n)]
    scale = 1.0 if kind == "i32" else 0.5
    cc.cc_allreduce_stepped([to_dev(x) for x in xs], out, ws, algo=algo, scale=scale)
    torch.cuda.synchronize()
    assert cc.cc_async_status() == cc.CC_OK
    pos = np.unique(np.concatenate([[0, 1, 2, 3, count - 1], np.arange(5, count, 2039)]))
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn([x[pos] for x in xs], in_dtype=_IN[kind], scale=scale, count=count, positions=pos)
    idx = torch.from_numpy(pos).cuda()
    for r in sorted({0, n // 2, n - 1}):
        _assert_same(out[r][idx].cpu().numpy(), want[r], f"stepped {algo} {kind} N={n} rank {r}")


@pytest.mark.parametrize("n,root", [(4, 1), (8, 7), (64, 33)])
@pytest.mark.parametrize("op", ["max", "prod"])
def test_reduce_other_ops_take_the_fold_machine(n, root, op):
    xs = [(1.0 + 0.01 * x).astype(np.float32) for x in _inputs("f32", n, 3001, seed=13)]
    want, _ = C.reduce(xs, root, op=op)
    out = torch.empty(3001, device="cuda")
    cc.cc_reduce([to_dev(x) for x in xs], out, root, op=op)
    torch.cuda.synchronize()
    _assert_same(to_host(out), want, f"reduce {op} N={n} root {root}")


def test_reduce_large_sampled():
    n, count = 64, 4 * 1024 * 1024 + 3
    xs = _inputs("spread", n, count, seed=14)
    out = torch.empty(count, device="cuda")
    cc.cc_reduce([to_dev(x) for x in xs], out, 5)
    torch.cuda.synchronize()
    pos = np.unique(np.concatenate([[0, 1, count - 1], np.arange(2, count, 4091)]))
    want, _ = C.reduce([x[pos] for x in xs], 5)
    _assert_same(out[torch.from_numpy(pos).cuda()].cpu().numpy(), want, "reduce N=64 sampled")


@pytest.mark.parametrize("algo", ["ring", "tree"])
def test_stepped_misaligned_large_takes_the_element_tiles(algo):
    """Outputs one element off a 16-byte boundary and large enough for the large-phase kernel:
    its element-wise tiles, compared with the oracle on sampled positions."""
    n, count = 3, 1024 * 1024 + 7
    xs = _inputs("spread", n, count, seed=18)
    out = [misaligned(np.zeros(count, np.float32)) for _ in range(n)]
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    cc.cc_allreduce_stepped([to_dev(x) for x in xs], out, ws, algo=algo, scale=0.25)
    torch.cuda.synchronize()
    assert cc.cc_async_status() == cc.CC_OK
    pos = np.unique(np.concatenate([[0, 1, 2, count - 1], np.arange(3, count, 997)]))
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn([x[pos] for x in xs], scale=0.25, count=count, positions=pos)
    idx = torch.from_numpy(pos).cuda()
    for r in range(n):
        _assert_same(out[r][idx].cpu().numpy(), want[r], f"stepped misaligned {algo} rank {r}")


def test_calls_replay_from_a_cuda_graph():
    """The calls are stream-ordered and do no host synchronisation, so they can be captured in a
    CUDA graph and replayed: a captured allreduce, reduce-scatter + allgather, stepped allreduce
    and fused bucket allreduce give the oracle's bits on every replay, with new inputs copied in
    between replays."""
    n, count = 8, 3 * 4096 + 5
    s = torch.cuda.Stream()
    send = [torch.empty(count, device="cuda") for _ in range(n)]
    ar = [torch.empty(count, device="cuda") for _ in range(n)]
    st = [torch.empty(count, device="cuda") for _ in range(n)]
    shards = [torch.empty(cc.cc_chunk(count, n, c)[1], device="cuda") for c in range(n)]
    ag = [torch.empty(count, device="cuda") for _ in range(n)]
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    with torch.cuda.stream(s):  # warm up (lazy set-up) outside the capture
        cc.cc_allreduce(send, ar, scale=None, stream=s)
        cc.cc_reduce_scatter(send, shards, stream=s)
        cc.cc_allgather(shards, ag, stream=s)
        cc.cc_allreduce_stepped(send, st, ws, algo="tree", stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cc.cc_allreduce(send, ar, scale=None, stream=s)
        cc.cc_reduce_scatter(send, shards, stream=s)
        cc.cc_allgather(shards, ag, stream=s)
        cc.cc_allreduce_stepped(send, st, ws, algo="tree", stream=s)
    for rep in range(2):
        xs = _inputs("spread", n, count, seed=70 + rep)
        for r in range(n):
            send[r].copy_(to_dev(xs[r]))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        want_ar, _ = C.ring_allreduce(xs, scale=float(np.float32(1) / np.float32(n)))
        want_rs, _ = C.ring_allreduce(xs)
        want_st, _ = C.tree_allreduce(xs)
        for r in range(n):
            _assert_same(to_host(ar[r]), want_ar[r], f"graph allreduce replay {rep} rank {r}")
            _assert_same(to_host(ag[r]), want_rs[r], f"graph RS+AG replay {rep} rank {r}")
            _assert_same(to_host(st[r]), want_st[r], f"graph stepped replay {rep} rank {r}")
