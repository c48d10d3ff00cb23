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
