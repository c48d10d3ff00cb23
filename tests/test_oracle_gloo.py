"""Third-party cross-check of the oracle: gloo collectives on 4 CPU processes (lecture 09
§7.2 experiment 2 runs the same calls). int32 only: gloo's fp32 summation order is its
own, so only order-free arithmetic can be compared bit for bit."""
import os
import socket

import numpy as np
import pytest

import synth
from oracle import collectives as C

WORLD = 4
COUNT = 1003


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x = torch.from_numpy(synth.int32_uniform(77, rank, COUNT, -2**31, 2**31 - 1))
    ar = x.clone()
    dist.all_reduce(ar)
    gl = [torch.zeros(COUNT // world + 1, dtype=torch.int32) for _ in range(world)]
    shard = torch.from_numpy(synth.int32_uniform(78, rank, COUNT // world + 1, -5, 5))
    dist.all_gather(gl, shard)
    q.put((rank, ar.numpy(), torch.cat(gl).numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_oracle_matches_gloo_int32():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, WORLD, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        r, ar, ag = q.get(timeout=150)
        res[r] = (ar, ag)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    xs = [synth.int32_uniform(77, r, COUNT, -2**31, 2**31 - 1) for r in range(WORLD)]
    ours, _ = C.ring_allreduce(xs, in_dtype="i32")
    shards = [synth.int32_uniform(78, r, COUNT // WORLD + 1, -5, 5) for r in range(WORLD)]
    ag, _ = C.ring_allgather(shards)
    for r in range(WORLD):
        assert np.array_equal(res[r][0], ours[r])
        assert np.array_equal(res[r][1], ag[r])
