"""Full-size parity: the workloads at their real sizes, launched as bench.py launches them.

The oracle cannot run 8 x 1.2 GB, so it runs each schedule on sampled element positions
(chunk boundaries, bucket edges, tails and a random spread) with the full-size chunk map:
every sampled element sees exactly the operations it sees in the full run. Properties that
hold at any size (identical replicas, allgather of the shards = the shards) are checked on
the whole buffers on the device."""
import numpy as np
import pytest

import synth
from oracle import collectives as C
from oracle import ddp, moe
from oracle import layout as L

from .helpers import bits, to_host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)
import collective_communication_primitives_rank_b200 as cc  # noqa: E402

SEED = 0x5EED  # the bench's seed


def _positions(count, bounds, rng, extra=2000):
    pts = {0, count - 1}
    for a, b in bounds:
        for d in (-3, -2, -1, 0, 1, 2, 3):
            for p in (a + d, b + d):
                if 0 <= p < count:
                    pts.add(p)
    pts.update(rng.integers(0, count, extra).tolist())
    return np.array(sorted(pts), dtype=np.int64)


def _gather(dev, pos):
    return dev[torch.from_numpy(pos).cuda()].cpu().numpy()


@pytest.mark.parametrize("algo", ["ring", "tree"])
def test_config2_ddp_full_size_sampled(algo):
    n, cap = 8, 25 * 1024 * 1024
    shapes = synth.transformer_grad_shapes()
    numels = [synth.numel(s) for _, s in shapes]
    total = sum(numels)
    offs = np.cumsum([0] + numels)
    host = [synth.normal_f32(SEED, r, total, 1e-3) for r in range(n)]  # as bench.py builds them
    dev_in = [torch.from_numpy(h).cuda() for h in host]
    dev_out = [torch.empty_like(d) for d in dev_in]
    views = lambda flat: [flat[offs[i]:offs[i + 1]].view(shapes[i][1]) for i in range(len(numels))]
    plan = cc.BucketAllreducePlan([views(d) for d in dev_in], [views(d) for d in dev_out], cap_bytes=cap,
                                  scale=1.0 / n, algo=algo)
    plan.run()
    torch.cuda.synchronize()
    for r in range(1, n):
        assert torch.equal(dev_out[r], dev_out[0]), f"replica {r} differs"
    rng = np.random.default_rng(1)
    buckets = ddp.assign_buckets(numels)
    assert len(buckets) == 17
    for members in buckets:
        bcount = sum(numels[i] for i in members)
        bounds = L.chunk_bounds(bcount, n) if algo == "ring" else [(0, (bcount + 1) // 2), ((bcount + 1) // 2, bcount)]
        bpos = _positions(bcount, bounds, rng, extra=300)
        # bucket position -> flat offset of the per-rank buffer
        starts = np.cumsum([0] + [numels[i] for i in members])
        k = np.searchsorted(starts, bpos, side="right") - 1
        flat = offs[np.array(members)[k]] + (bpos - starts[k])
        fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
        want, _ = fn([h[flat] for h in host], scale=1.0 / n, count=bcount, positions=bpos)
        got = _gather(dev_out[3], flat)
        assert np.array_equal(bits(got), bits(want[3])), f"bucket {members[:3]}..."


def test_config3_zero_full_size_sampled():
    n, count = 8, 300_000_000
    bounds = L.chunk_bounds(count, n)
    rng = np.random.default_rng(2)
    pos = _positions(count, bounds, rng)
    dev, dev_b, samp, samp_b = [], [], [], []
    for r in range(n):
        h = synth.normal_f32(SEED + 3, r, count, 1e-2)
        hb = synth.to_bf16_bits(h)
        samp.append(h[pos].copy())
        samp_b.append(hb[pos].copy())
        dev.append(torch.from_numpy(h).cuda())
        dev_b.append(torch.from_numpy(hb.view(np.int16)).cuda().view(torch.bfloat16))
        del h, hb
    shard = count // n
    rs = [torch.empty(shard, device="cuda") for _ in range(n)]
    cc.cc_reduce_scatter(dev, rs)
    ag = [torch.empty(count, device="cuda") for _ in range(n)]
    cc.cc_allgather(rs, ag)
    torch.cuda.synchronize()
    want_rs, _ = C.ring_reduce_scatter(samp, count=count, positions=pos)
    for c, (a, b) in enumerate(bounds):
        sel = (pos >= a) & (pos < b)
        got = _gather(rs[c], pos[sel] - a)
        assert np.array_equal(bits(got), bits(want_rs[c])), f"shard {c}"
    for r in range(n):
        assert torch.equal(ag[r], ag[0])
    for c, (a, b) in enumerate(bounds):
        assert torch.equal(ag[5][a:b], rs[c])
    del ag
    cc.cc_reduce_scatter(dev_b, rs)
    torch.cuda.synchronize()
    want_b, _ = C.ring_reduce_scatter(samp_b, in_dtype="bf16", count=count, positions=pos)
    for c, (a, b) in enumerate(bounds):
        sel = (pos >= a) & (pos < b)
        assert np.array_equal(bits(_gather(rs[c], pos[sel] - a)), bits(want_b[c])), f"bf16 shard {c}"


def test_config4_moe_full_size():
    n, tokens, hidden, epr = 8, 8192, 4096, 8
    E = n * epr
    lg = [synth.normal_f32(SEED + 4, r, tokens * E, stream=3).reshape(tokens, E) for r in range(n)]
    toks = [synth.to_bf16_bits(synth.normal_f32(SEED + 4, r, tokens * hidden, stream=4)).reshape(tokens, hidden)
            for r in range(n)]
    ids = [torch.empty(tokens, 2, dtype=torch.int32, device="cuda") for _ in range(n)]
    cc.cc_route_topk([torch.from_numpy(x).cuda() for x in lg], ids)
    torch.cuda.synchronize()
    ids_h = [to_host(i) for i in ids]
    for r in range(n):
        assert np.array_equal(ids_h[r], moe.route_topk(lg[r], 2))
    want, _ = moe.dispatch(toks, ids_h, epr)
    cap = tokens * 2 * 2
    d_tok = [torch.from_numpy(t.view(np.int16)).cuda().view(torch.bfloat16) for t in toks]
    recv = [torch.empty(cap, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    back = [torch.empty(tokens, 2, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, 2, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv(d_tok, recv, ids, epr, ws, direction=0)
    cc.cc_alltoallv(recv, back, ids, epr, ws, direction=1)
    torch.cuda.synchronize()
    for d in range(n):
        got = to_host(recv[d])[:want[d].shape[0]]
        assert np.array_equal(got, want[d]), f"dispatch rank {d}"
    for s in range(n):
        for k in range(2):
            assert torch.equal(back[s][:, k].view(torch.int16), d_tok[s].view(torch.int16))


@pytest.mark.parametrize("n,mib", [(8, 256), (64, 64), (2, 256)])
@pytest.mark.parametrize("algo", ["ring", "tree"])
def test_config5_sweep_large_points_sampled(n, mib, algo):
    count = mib * 1024 * 1024 // 4
    bounds = L.chunk_bounds(count, n) if algo == "ring" else [(0, (count + 1) // 2), ((count + 1) // 2, count)]
    pos = _positions(count, bounds, np.random.default_rng(n))
    dev, samp = [], []
    for r in range(n):
        h = synth.uniform_f32(SEED + 5, r, count)
        samp.append(h[pos].copy())
        dev.append(torch.from_numpy(h).cuda())
        del h
    out = [torch.empty(count, device="cuda") for _ in range(n)]
    cc.cc_allreduce(dev, out, algo=algo)
    torch.cuda.synchronize()
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn(samp, count=count, positions=pos)
    for r in (0, n - 1):
        assert np.array_equal(bits(_gather(out[r], pos)), bits(want[r]))
    for r in range(1, n):
        assert torch.equal(out[r], out[0])


@pytest.mark.parametrize("so,do", [(1, 1), (1, 0), (0, 3)])
@pytest.mark.parametrize("algo", ["ring", "tree"])
def test_large_allreduce_and_reduce_scatter_off_a_boundary_sampled(so, do, algo):
    """N = 8 x 128 MiB with every source `so` and every output `do` elements past a 16-byte
    boundary (tens of thousands of line-skewed tiles; element stores where the offsets differ),
    sampled at every chunk edge and at random positions against the oracle."""
    n, count = 8, 32 * 1024 * 1024
    bounds = L.chunk_bounds(count, n) if algo == "ring" else [(0, (count + 1) // 2), ((count + 1) // 2, count)]
    pos = _positions(count, bounds, np.random.default_rng(so * 4 + do))
    # every element within 40 of a tile edge (tiles of 1024 elements, skewed onto lines) at
    # a few hundred places
    near = (np.arange(1024, count, 1024 * 97)[:, None] + np.arange(-40, 41)[None, :]).ravel()
    pos = np.unique(np.concatenate([pos, near[(near >= 0) & (near < count)]]))
    dev, samp = [], []
    for r in range(n):
        h = synth.uniform_f32(SEED + 9, r, count)
        samp.append(h[pos].copy())
        full = torch.empty(count + 4, device="cuda")
        full[so:so + count].copy_(torch.from_numpy(h))
        dev.append(full[so:so + count])
        del h
    out = [torch.empty(count + 4, device="cuda")[do:do + count] for _ in range(n)]
    cc.cc_allreduce(dev, out, algo=algo, scale=0.125)
    torch.cuda.synchronize()
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn(samp, count=count, positions=pos, scale=0.125)
    for r in (0, n - 1):
        assert np.array_equal(bits(_gather(out[r], pos)), bits(want[r])), f"{algo} {so}/{do} rank {r}"
    if algo == "ring":
        shards = [torch.empty(b - a + 4, device="cuda")[do:do + b - a] for a, b in L.chunk_bounds(count, n)]
        cc.cc_reduce_scatter(dev, shards, scale=0.125)
        torch.cuda.synchronize()
        want_rs, _ = C.ring_reduce_scatter(samp, count=count, positions=pos, scale=0.125)
        for c, (a, b) in enumerate(L.chunk_bounds(count, n)):
            inside = (pos >= a) & (pos < b)
            assert np.array_equal(bits(_gather(shards[c], pos[inside] - a)), bits(want_rs[c])), \
                f"reduce-scatter {so}/{do} shard {c}"
