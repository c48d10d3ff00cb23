"""Seeded random shapes for every reduction entry point against the oracle, bit for bit: rank
counts 1..64, ragged counts including counts below the rank count, every op, every dtype pair,
aligned and misaligned buffers, in place and out of place."""
import numpy as np
import pytest

import synth
from oracle import collectives as C

from .helpers import Guarded, bits, misaligned, to_dev, to_host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)
import collective_communication_primitives_rank_b200 as cc  # noqa: E402

OPS = ["sum", "max", "min", "prod"]
KINDS = ["f32", "i32", "bf16"]


def _case(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.choice([1, 2, 3, 4, 5, 7, 8, 9, 13, 16, 31, 32, 64]))
    count = int(rng.choice([1, 2, 3, n - 1 if n > 1 else 1, n, n + 1, 17, 1000, 4099, 65536 + 3, 250_007]))
    kind = KINDS[int(rng.integers(0, 3))]
    op = OPS[int(rng.integers(0, 4))] if kind != "bf16" else ["sum", "max"][int(rng.integers(0, 2))]
    return n, max(count, 1), kind, op, bool(rng.integers(0, 2)), int(rng.integers(0, 1 << 30))


def _inputs(kind, n, count, seed, op):
    if kind == "i32":
        lo, hi = (-3, 3) if op == "prod" else (-2**31, 2**31 - 1)
        return [synth.int32_uniform(seed, r, count, lo, hi) for r in range(n)]
    if kind == "bf16":
        return [synth.to_bf16_bits(synth.normal_f32(seed, r, count)) for r in range(n)]
    x = [synth.uniform_f32(seed, r, count) for r in range(n)]
    if op == "prod":
        x = [(1.0 + 0.05 * v).astype(np.float32) for v in x]
    return x


def _dev(x, mis):
    return misaligned(x) if mis else to_dev(x)


def _out(count, kind, mis):
    z = np.zeros(count, np.int32 if kind == "i32" else np.float32)
    return misaligned(z) if mis else to_dev(z)


@pytest.mark.parametrize("seed", range(24))
def test_allreduce_family_random_shapes(seed):
    n, count, kind, op, mis, s = _case(seed)
    xs = _inputs(kind, n, count, s, op)
    ind = {"f32": "f32", "i32": "i32", "bf16": "bf16"}[kind]
    scale = 1.0 if kind == "i32" else 0.5
    send = [_dev(x, mis) for x in xs]
    for algo, fn in (("ring", C.ring_allreduce), ("tree", C.tree_allreduce)):
        want, _ = fn(xs, op=op, in_dtype=ind, scale=scale)
        out = [_out(count, kind, mis) for _ in range(n)]
        cc.cc_allreduce(send, out, op=op, algo=algo, scale=scale)
        torch.cuda.synchronize()
        for r in range(n):
            assert np.array_equal(bits(to_host(out[r])), bits(want[r])), f"{algo} {kind} {op} N={n} count={count}"
    K = 1 + seed % 5
    want, _ = C.multiring_allreduce(xs, K, op=op, in_dtype=ind, scale=scale)
    out = [_out(count, kind, mis) for _ in range(n)]
    cc.cc_allreduce_multiring(send, out, K, op=op, scale=scale)
    torch.cuda.synchronize()
    for r in range(n):
        assert np.array_equal(bits(to_host(out[r])), bits(want[r])), f"multiring K={K} {kind} {op} N={n}"
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    algo = "ring" if seed % 2 else "tree"
    want, _ = (C.ring_allreduce if algo == "ring" else C.tree_allreduce)(xs, op=op, in_dtype=ind, scale=scale)
    out = [_out(count, kind, mis) for _ in range(n)]
    cc.cc_allreduce_stepped(send, out, ws, op=op, algo=algo, scale=scale)
    torch.cuda.synchronize()
    assert cc.cc_async_status() == cc.CC_OK
    for r in range(n):
        assert np.array_equal(bits(to_host(out[r])), bits(want[r])), f"stepped {algo} {kind} {op} N={n}"


@pytest.mark.parametrize("seed", range(24, 40))
def test_reduce_scatter_reduce_allgather_random_shapes(seed):
    n, count, kind, op, mis, s = _case(seed)
    xs = _inputs(kind, n, count, s, op)
    ind = {"f32": "f32", "i32": "i32", "bf16": "bf16"}[kind]
    send = [_dev(x, mis) for x in xs]
    want, _ = C.ring_reduce_scatter(xs, op=op, in_dtype=ind)
    shards = [_out(cc.cc_chunk(count, n, c)[1], kind, mis) if cc.cc_chunk(count, n, c)[1] else
              torch.empty(0, dtype=torch.int32 if kind == "i32" else torch.float32, device="cuda") for c in range(n)]
    cc.cc_reduce_scatter(send, shards, op=op)
    root = s % n
    want_red, _ = C.reduce(xs, root, op=op, in_dtype=ind)
    red = _out(count, kind, mis)
    cc.cc_reduce(send, red, root, op=op)
    torch.cuda.synchronize()
    for c in range(n):
        assert np.array_equal(bits(to_host(shards[c])), bits(want[c])), f"RS {kind} {op} N={n} count={count} c={c}"
    assert np.array_equal(bits(to_host(red)), bits(want_red)), f"reduce {kind} {op} N={n} root={root}"
    if kind != "bf16":  # allgather of the reduce-scatter shards gives the allreduce
        full = [_out(count, kind, mis) for _ in range(n)]
        cc.cc_allgather(shards, full)
        want_ar, _ = C.ring_allreduce(xs, op=op, in_dtype=ind)
        torch.cuda.synchronize()
        for r in range(n):
            assert np.array_equal(bits(to_host(full[r])), bits(want_ar[r])), f"AG(RS) {kind} {op} N={n}"


def _at(x: np.ndarray, elems: int):
    """A CUDA tensor holding `x`, `elems` elements past a 16-byte boundary."""
    return to_dev(np.concatenate([np.zeros(elems, x.dtype), x]))[elems:]


@pytest.mark.parametrize("seed", range(40, 64))
def test_random_offsets_for_sources_and_outputs(seed):
    """Sources at one common or at per-rank random offsets from a 16-byte boundary, outputs at
    another (the element-store, realigned-copy and element paths, and line-skewed tiles over
    several hundred tiles), guard bands around every output: allreduce (ring, tree), reduce-
    scatter, reduce and allgather, bit for bit against the oracle."""
    n, count, kind, op, _, s = _case(seed)
    rng = np.random.default_rng(seed + 1000)
    if seed % 3 == 0:  # hundreds of tiles
        count = int(rng.integers(1 << 20, 3 << 20)) if n <= 16 else int(rng.integers(1 << 16, 1 << 18))
    xs = _inputs(kind, n, count, s, op)
    ind = {"f32": "f32", "i32": "i32", "bf16": "bf16"}[kind]
    common = bool(rng.integers(0, 2))
    so = [int(rng.integers(0, 4))] * n if common else [int(x) for x in rng.integers(0, 4, n)]
    do = int(rng.integers(0, 4))
    send = [_at(x, o) for x, o in zip(xs, so)]
    od = torch.int32 if kind == "i32" else torch.float32
    scale = 1.0 if kind == "i32" or op != "sum" else 0.5
    for algo, fn in (("ring", C.ring_allreduce), ("tree", C.tree_allreduce)):
        want, _ = fn(xs, op=op, in_dtype=ind, scale=scale)
        out = [Guarded(count, od, misalign=do) for _ in range(n)]
        cc.cc_allreduce(send, [g.t for g in out], op=op, algo=algo, scale=scale)
        torch.cuda.synchronize()
        for r in range(n):
            assert np.array_equal(bits(to_host(out[r].t)), bits(want[r])), f"{algo} {kind} {op} N={n} {so}/{do}"
            out[r].check()
    want, _ = C.ring_reduce_scatter(xs, op=op, in_dtype=ind)
    shards = [Guarded(cc.cc_chunk(count, n, c)[1], od, misalign=(do + c) % 4) for c in range(n)]
    cc.cc_reduce_scatter(send, [g.t for g in shards], op=op)
    root = s % n
    want_red, _ = C.reduce(xs, root, op=op, in_dtype=ind)
    red = Guarded(count, od, misalign=do)
    cc.cc_reduce(send, red.t, root, op=op)
    torch.cuda.synchronize()
    for c in range(n):
        assert np.array_equal(bits(to_host(shards[c].t)), bits(want[c])), f"RS {kind} {op} N={n} {so}/{do} c={c}"
        shards[c].check()
    assert np.array_equal(bits(to_host(red.t)), bits(want_red)), f"reduce {kind} {op} N={n} {so}/{do}"
    red.check()
    if kind != "bf16":  # allgather of the shards (each at its own offset) into outputs at `do`
        full = [Guarded(count, od, misalign=do) for _ in range(n)]
        cc.cc_allgather([g.t for g in shards], [g.t for g in full])
        want_ar, _ = C.ring_allreduce(xs, op=op, in_dtype=ind)
        torch.cuda.synchronize()
        for r in range(n):
            assert np.array_equal(bits(to_host(full[r].t)), bits(want_ar[r])), f"AG {kind} {op} N={n} {so}/{do}"
            full[r].check()
