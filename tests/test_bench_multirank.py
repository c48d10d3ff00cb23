"""The multi-GPU plumbing of bench.py on CPU: gloo, world size 2. Each rank holds its own
replica (its own seed), the step time is the max over ranks, and the job value aggregates
all ranks. The reference arm under torchrun prints one line from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = 10.0 + 5.0 * rank
    worst = bench.max_over_ranks(dist, torch, local_ms, "cpu")
    q.put((rank, bench.replica_seed(rank), worst, bench.aggregate_gbps(world, 7_016_448_000, worst)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_aggregate_with_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict((r, (seed, worst, agg)) for r, seed, worst, agg in (q.get(timeout=90) for _ in range(2)))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert got[0][0] != got[1][0]                     # independent replicas
    assert got[0][1] == got[1][1] == 15.0             # the slowest rank's time
    assert abs(got[0][2] - 2 * 7.016448 / 0.015) < 1e-6  # both ranks' bytes over that time


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--layers", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=280, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_profile_traffic_goes_null_when_the_kernel_source_changes(tmp_path):
    # a committed ncu summary carries the SHA-256 of the kernel source it measured; bench.py
    # reports its DRAM traffic only while that source is unchanged
    import hashlib
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()
    (tmp_path / "profiles" / "p.txt").write_text(
        f"kernel_source: k.cu\nkernel_source_sha256: {sha}\ndram_bytes_per_launch_full_workload: 1234\n"
        "  launch  0  1.0 us\n")
    b.ROOT = str(tmp_path)
    assert b.profile_traffic("p.txt") == 1234
    src.write_text("kernel v2\n")
    assert b.profile_traffic("p.txt") is None
    assert b.profile_traffic("missing.txt") is None
    # a kernel spread over two files: both must be unchanged
    hdr = tmp_path / "k.cuh"
    hdr.write_text("folds v1\n")
    sha1 = hashlib.sha256(b"kernel v2\n").hexdigest()
    sha2 = hashlib.sha256(b"folds v1\n").hexdigest()
    (tmp_path / "profiles" / "q.txt").write_text(
        f"kernel_source: k.cu, k.cuh\nkernel_source_sha256: {sha1}, {sha2}\n"
        "dram_bytes_per_launch_full_workload: 99\n")
    assert b.profile_traffic("q.txt") == 99
    hdr.write_text("folds v2\n")
    assert b.profile_traffic("q.txt") is None


def _layout_worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    numels = [synth.numel(s) for _, s in synth.transformer_grad_shapes(layers=2)]
    offs, ranges = bench.bucket_order_layout(numels, cap=4 * 1024 * 1024)
    every = [None] * world
    dist.all_gather_object(every, (offs, ranges))
    # fake peer base addresses: every rank's flat buffer at its own address
    bases = [0x7000_0000_0000 + r * 0x1_0000_0000 for r in range(world)]
    ptrs = [bench.offset_ptrs(bases, start) for start, _ in ranges]
    q.put((rank, every, offs, ranges, numels, ptrs, bases))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_multi_gpu_bucket_layout_agrees_across_ranks_and_tiles_the_buffer():
    """The one-rank-per-GPU path: every rank derives the same flat bucket-order layout, each
    bucket is one contiguous range holding exactly its tensors, the ranges tile the buffer,
    and a bucket's pointers are every rank's base advanced by the bucket's start."""
    import torch.multiprocessing as mp
    sys.path.insert(0, ROOT)
    import collective_communication_primitives_rank_b200 as cc
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_layout_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=90) for _ in range(2)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, every, offs, ranges, numels, ptrs, bases in got:
        assert every[0] == every[1]
        assert ranges[0][0] == 0 and sum(c for _, c in ranges) == sum(numels)
        for (s0, c0), (s1, _) in zip(ranges, ranges[1:]):
            assert s0 + c0 == s1
        buckets = cc.cc_bucket_assign(numels, 4, 4 * 1024 * 1024)
        assert len(buckets) == len(ranges)
        for members, (start, count) in zip(buckets, ranges):
            assert sorted(offs[i] for i in members) == [offs[i] for i in members]  # in the order taken
            assert offs[members[0]] == start and sum(numels[i] for i in members) == count
        for (start, _), p in zip(ranges, ptrs):
            assert p == [b + 4 * start for b in bases]


def test_alpha_beta_model_against_closed_forms():
    """The lecture's alpha-beta model (lecture 09 §7.3: ring 2(N-1) alpha + 2(N-1)/N M / B, tree
    2 log2(N) alpha + 2 M / B): with one alpha and one B the ring's extra latency
    2(N-1-log2 N) alpha is paid back by its smaller per-byte term at
    M* = 2(N-1-log2 N) alpha / (2/B - 2(N-1)/(N B)) = (N-1-log2 N) N alpha B."""
    sys.path.insert(0, ROOT)
    import bench
    a, B = 2e-6, 100e9
    for n in (4, 8, 16, 64):
        import math
        want = (n - 1 - math.log2(n)) * n * a * B
        got = bench.alpha_beta_crossover(n, a, a, B, B)
        assert abs(got - want) <= 1e-9 * want, (n, got, want)
        assert bench.crossover_reading(n, a, a, B, B).startswith("ring faster above")
    # the fitted stepped numbers of one GPU: the tree wins both terms, so no crossover
    assert bench.alpha_beta_crossover(8, 1.78e-6, 2.71e-6, 200e9, 254e9) is None
    assert "tree is faster at every size" in bench.crossover_reading(8, 1.78e-6, 2.71e-6, 200e9, 254e9)
    # N = 2: the same steps, so the ring's smaller per-byte term never loses
    assert bench.alpha_beta_crossover(2, a, a, B, B) is None
    assert "ring is at least as fast" in bench.crossover_reading(2, a, a, B, B)
