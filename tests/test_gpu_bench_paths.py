"""The one-rank-per-GPU bench path (what `bench.py --gpus N` runs under torchrun) on one GPU: the
slice calls over the IPC plumbing with a single rank, NCCL beside them, and rank 0's bit-exact
check against the single-GPU fused call. Runs bench.py as a child process."""
import json
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.timeout(600)
def test_one_rank_per_gpu_path_runs_and_matches_the_single_gpu_call():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_port()), RANK="0", WORLD_SIZE="1",
               LOCAL_RANK="0")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "peer", "--layers", "1", "--steps", "2",
           "--warmup", "1", "--e2e-steps", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=540, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["parity_rank0_vs_single_gpu"] == "bit-exact"
    assert line["comm_nranks"] == 1 and line["value"] > 0 and line["config"]["buckets"] >= 1


@pytest.mark.timeout(900)
def test_two_ranks_on_one_gpu_over_gloo_match_the_single_gpu_call():
    """Two processes (torchrun), both on this GPU, host barriers over gloo: the bucket layout,
    the IPC mappings of the other rank's buffers, the 17-bucket step of slice calls and rank 0's
    bit-exact comparison with the single-GPU fused call over both ranks' gradients. No kernel
    waits on the other rank; the barriers order them."""
    env = dict(os.environ, CC_BENCH_BACKEND="gloo", CC_BENCH_DEVICE="0")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_port()), os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--workload", "peer", "--layers", "1", "--steps", "2", "--warmup", "1", "--e2e-steps", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=840, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["parity_rank0_vs_single_gpu"] == "bit-exact"
    assert line["comm_nranks"] == 2 and line["n_gpus"] == 2 and line["backend"] == "gloo"


@pytest.mark.timeout(600)
@pytest.mark.parametrize("algo", ["ring", "tree"])
def test_default_line_carries_every_contract_key(algo):
    """The one-GPU headline line (1-layer model, no rows): the keys the bench contract names,
    with a roofline against the copy rate, the end-to-end number through host buffers, the
    clock record and the count of the library's launches."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--layers", "1", "--steps", "3", "--warmup", "3",
           "--e2e-steps", "1", "--no-rows", "--no-cpu-baseline", "--algo", algo]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=540, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == 3 and line["value"] > 0 and line["higher_is_better"] is True
    assert line["gpu_launches"] == 3 and line["config"]["workload"]
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9 and algo in roof["kernel"]
    e2e = line["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] == e2e["d2h_bytes_per_step"] > 0
    assert line["clocks"]["samples"] >= 1 and "reasons" in line["clocks"]
