"""GPU parity of the one-rank-per-process slice calls against the oracle.

Every rank's slice, run one after another in one process on local buffers, must leave
exactly the single-call result (each slice folds and writes only its own chunk, so the
order of the ranks does not matter). Then two processes on the same GPU exchange CUDA IPC
handles over a gloo group and each runs its own slice on the other's mapped buffers, the
ranks ordered by host barriers only (no kernel waits on another)."""
import datetime
import os
import socket

import numpy as np
import pytest

import synth
from oracle import collectives as C
from oracle import layout as L

from .helpers import Guarded, to_dev, to_host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)
import collective_communication_primitives_rank_b200 as cc  # noqa: E402

_IN = {"spread": "f32", "i32": "i32", "bf16": "bf16"}


def _inputs(kind, n, count, seed=21):
    if kind == "spread":  # magnitudes 2^-20..2^20: the bracketing shows in the rounding
        return [(synth.uniform_f32(seed, r, count) *
                 np.exp2(synth.int32_uniform(seed, r, count, -20, 20, stream=1)).astype(np.float32)).astype(np.float32)
                for r in range(n)]
    if kind == "i32":
        return [synth.int32_uniform(seed, r, count, -2**31, 2**31 - 1) for r in range(n)]
    return [synth.to_bf16_bits(synth.normal_f32(seed, r, count, 1e-2)) for r in range(n)]


def _out_dtype(kind):
    return torch.int32 if kind == "i32" else torch.float32


def _same(got, want, what):
    g = np.ascontiguousarray(got).view(np.uint32)
    w = np.ascontiguousarray(want).view(np.uint32)
    bad = np.flatnonzero(g != w)
    assert bad.size == 0, f"{what}: {bad.size} elements differ, first at {bad[0]}"


@pytest.mark.parametrize("n,count", [(1, 1000), (3, 4099), (8, 10007), (13, 2049), (8, 5)])
@pytest.mark.parametrize("algo", ["ring", "tree"])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_allreduce_slices_equal_allreduce(n, count, algo, kind):
    xs = _inputs(kind, n, count)
    scale = 1.0 if kind == "i32" else 1.0 / n
    fn = C.ring_allreduce if algo == "ring" else C.tree_allreduce
    want, _ = fn(xs, in_dtype=_IN[kind], scale=scale)
    send = [to_dev(x) for x in xs]
    out = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    for r in reversed(range(n)):
        cc.cc_allreduce_slice(send, [o.t for o in out], r, algo=algo, scale=scale)
    torch.cuda.synchronize()
    for r in range(n):
        _same(to_host(out[r].t), want[r], f"{algo} {kind} N={n} rank {r}")
        out[r].check()


def test_allreduce_slices_in_place():
    n, count = 5, 30001
    xs = _inputs("spread", n, count, seed=22)
    want, _ = C.ring_allreduce(xs, in_dtype="f32", scale=0.5)
    buf = [to_dev(x) for x in xs]
    for r in range(n):
        cc.cc_allreduce_slice(buf, buf, r, scale=0.5)
    torch.cuda.synchronize()
    for r in range(n):
        _same(to_host(buf[r]), want[r], f"in place rank {r}")


@pytest.mark.parametrize("n,count", [(2, 1 << 16), (7, 12345), (8, 3)])
@pytest.mark.parametrize("kind", ["spread", "i32", "bf16"])
def test_reduce_scatter_and_allgather_slices(n, count, kind):
    xs = _inputs(kind, n, count, seed=23)
    scale = 1.0 if kind == "i32" else 0.25
    want_rs, _ = C.ring_reduce_scatter(xs, in_dtype=_IN[kind], scale=scale)
    want_ag, _ = C.ring_allgather(want_rs, count=count)
    send = [to_dev(x) for x in xs]
    lens = [b - a for a, b in L.chunk_bounds(count, n)]
    shards = [Guarded(ln, _out_dtype(kind)) for ln in lens]
    for r in range(n):
        cc.cc_reduce_scatter_slice(send, shards[r].t, r, scale=scale)
    out = [Guarded(count, _out_dtype(kind)) for _ in range(n)]
    for r in reversed(range(n)):
        cc.cc_allgather_slice(shards[r].t, [o.t for o in out], r)
    torch.cuda.synchronize()
    for r in range(n):
        _same(to_host(shards[r].t), want_rs[r], f"RS shard {r}")
        _same(to_host(out[r].t), want_ag[r], f"AG rank {r}")
        shards[r].check()
        out[r].check()


# ---- two processes on one GPU, buffers mapped over CUDA IPC --------------------------------

WORLD = 2
COUNT = 100_003


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _ipc_worker(rank, port, q):
    import torch as t
    import torch.distributed as dist
    import collective_communication_primitives_rank_b200 as lib
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        t.cuda.set_device(0)
        dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
        xs = _inputs("spread", WORLD, COUNT, seed=24)
        send = t.from_numpy(xs[rank]).cuda()
        # an offset inside a larger allocation: the handle must carry the offset
        block = t.zeros(COUNT + 64, device="cuda")
        recv = block[16:16 + COUNT]
        ar = lib.PeerAllreduce(send, recv, scale=1.0 / WORLD)
        ar.run()
        want, _ = C.ring_allreduce(xs, in_dtype="f32", scale=1.0 / WORLD)
        got = recv.cpu().numpy()
        ok_ar = bool(np.array_equal(got.view(np.uint32), want[rank].view(np.uint32)))
        ok_guard = bool((block[:16] == 0).all().item() and (block[16 + COUNT:] == 0).all().item())
        # reduce-scatter into a local shard, then allgather the shards over the mapped outputs
        a, ln = lib.cc_chunk(COUNT, WORLD, rank)
        shard = t.empty(ln, device="cuda")
        out = t.zeros(COUNT, device="cuda")
        peers = lib.PeerGroup([send, out])
        t.cuda.synchronize()
        dist.barrier()
        lib.cc_reduce_scatter_slice(peers.buffers(0), shard, rank)
        t.cuda.synchronize()
        dist.barrier()
        lib.cc_allgather_slice(shard, peers.buffers(1), rank)
        t.cuda.synchronize()
        dist.barrier()
        want_rs, _ = C.ring_reduce_scatter(xs, in_dtype="f32")
        want_ag, _ = C.ring_allgather(want_rs, count=COUNT)
        ok_rs = bool(np.array_equal(shard.cpu().numpy().view(np.uint32), want_rs[rank].view(np.uint32)))
        ok_ag = bool(np.array_equal(out.cpu().numpy().view(np.uint32), want_ag[rank].view(np.uint32)))
        dist.barrier()  # nobody unmaps before both ranks are done reading
        peers.close()
        ar.close()
        dist.barrier()
        q.put((rank, ok_ar, ok_guard, ok_rs, ok_ag, ""))
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, False, False, False, False, repr(e)))


@pytest.mark.timeout(300)
def test_slices_over_ipc_in_two_processes():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        item = q.get(timeout=240)
        res[item[0]] = item[1:]
    for p in procs:
        p.join(timeout=60)
    for r in range(WORLD):
        ok_ar, ok_guard, ok_rs, ok_ag, err = res[r]
        assert err == "", f"rank {r}: {err}"
        assert ok_ar and ok_guard and ok_rs and ok_ag, f"rank {r}: {res[r]}"
    for p in procs:
        assert p.exitcode == 0
