"""Benchmark of libcc, the collective-primitives library, on B200.

Default (one GPU): the headline is config 2, the fused DDP gradient-bucket allreduce. N = 8
simulated ranks each hold the fp32 gradients of a 12-layer d = 768 transformer (147 tensors,
109,632,000 elements = 438.5 MB per rank, normal(0, 1e-3)), packed into 25 MiB buckets (17)
in reverse registration order; one step is a ring allreduce of every bucket with the 1/N
mean, unflattened, in one fused kernel launch (cc_bucket_allreduce), inputs and outputs
resident in HBM. Metric: allreduce effective HBM GB/s = (N·T in + N·T out) / step time, plus
its share of ~8 TB/s and elements/s. The same line carries `e2e` (the step from pinned host
memory through cc_bucket_allreduce_host), `cpu_baseline` (the oracle on a sample), and
`rows` with configs 1, 3, 4 and 5 (latency-bound config 1; ZeRO reduce-scatter / allgather;
MoE routing, dispatch, combine; the large ring / tree points and the stepped schedules with
the alpha-beta model's crossover), each timed with CUDA events and with its own clock record.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ddp|zero|moe|sweep|peer]

--gpus N > 1 runs under torchrun, one process per GPU: each rank holds its own gradients of
the same model and the ranks allreduce them for real, through libcc's slice calls over CUDA
IPC (plain NVLink loads and stores), with NCCL's all_reduce timed beside it (weak scaling:
T per GPU is fixed); the step time is the max over ranks.
--workload zero / moe / sweep prints one config alone in detail (the sweep covers N in
{2..64} x 1 KiB..256 MiB with the measured and modelled ring / tree crossovers).
--impl reference times the oracle (the plain CPU message-passing simulator) on a bounded
sample of the headline workload.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "allreduce effective HBM GB/s (N·T in + N·T out) and % of ~8 TB/s; elems/s"
NOMINAL_HBM_GBS = 8000.0
N_SIM = 8
CAP = 25 * 1024 * 1024
SEED = 0x5EED
KERNEL_SRC = os.path.join(ROOT, "collective_communication_primitives_rank_b200", "csrc", "k_reduce.cu")


def replica_seed(rank):
    """Each GPU of a multi-GPU run holds its own replica of the workload (independent problem)."""
    return SEED + 1000 * rank


def max_over_ranks(dist, torch, value, device):
    """The slowest rank's time (one float through the process group; not on the data path)."""
    t = torch.tensor([float(value)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbps(world, bytes_per_step, ms_per_step):
    """Whole-job throughput: every rank moves bytes_per_step in the (max-over-ranks) step time."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


def workload_desc(layers, algo="ring"):
    fold = "ring" if algo == "ring" else "double-binary-tree"
    return (f"ddp_bucket_allreduce: N={N_SIM} simulated ranks on one GPU, fp32 gradients of a "
            f"{layers}-layer d=768 ffn=3072 vocab=32000 transformer, 25 MiB buckets in reverse "
            f"registration order, {fold} allreduce with scale 1/{N_SIM}, fused flatten/unflatten")


def measured_peak():
    """HBM roofline denominator: the measured copy rate (a copy kernel's read + write bytes per
    second, not a hard ceiling: a read-heavy kernel can pass it), else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured copy rate (MEASURED_PEAKS.json hbm_gbs; not a ceiling)"
    except Exception:
        return 6650.0, "fallback copy rate (6650 GB/s, earlier measurement; not a ceiling)"


DDP_PROFILES = {"ring": "bucket_allreduce_ddp.txt", "tree": "bucket_allreduce_ddp_tree.txt"}


def profile_traffic(name="bucket_allreduce_ddp.txt"):
    """DRAM bytes per launch of a line's dominant kernel from a committed ncu summary in
    profiles/, or None when a source file of the kernel changed since the counters were taken
    (the summary records the files, comma-separated, and their SHA-256s in the same order)."""
    try:
        text = open(os.path.join(ROOT, "profiles", name)).read()
        lines = dict(l.split(":", 1) for l in text.splitlines() if ":" in l and not l.startswith(" "))
        srcs = [x.strip() for x in lines.get("kernel_source", os.path.relpath(KERNEL_SRC, ROOT)).split(",")]
        shas = [x.strip() for x in lines.get("kernel_source_sha256", "").split(",")]
        if len(srcs) != len(shas):
            return None
        for src, sha in zip(srcs, shas):
            if sha != hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest():
                return None
        return int(float(lines["dram_bytes_per_launch_full_workload"].strip()))
    except Exception:
        return None


class Clocks:
    """SM clock and clock-event reasons sampled while the timed region runs: NVML polled
    every ~2 ms from a thread (the timed region can be a few tens of ms), nvidia-smi at
    200 ms as the fallback."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.samples, self.max_mhz, self.source = [], None, None
        self._stop = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.cuda_index)
        try:
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.source = "nvml"

            def poll():
                while not self._stop.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        pass
                    time.sleep(0.002)
            self._thread = threading.Thread(target=poll, daemon=True)
            self._thread.start()
        except Exception:
            self.source = "nvidia-smi"
            self._proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        time.sleep(0.01)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.source == "nvml":
            self._thread.join(timeout=2)
        elif self.source == "nvidia-smi":
            time.sleep(0.25)
            self._proc.terminate()
            try:
                out, _ = self._proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
                out = ""
            for line in (out or "").splitlines():
                f = [x.strip() for x in line.split(",")]
                try:
                    self.max_mhz = float(f[1])
                    self.samples.append((float(f[0]), int(f[2], 16)))
                except (ValueError, IndexError):
                    pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "samples": 0, "reasons": ["unsampled"]}
        mask = 0
        for _, r in self.samples:
            mask |= r
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "source": self.source,
                "reasons": sorted(name for bit, name in self.REASONS.items() if mask & bit)}


def build_workload(torch, layers, seed, pinned_inputs):
    import synth
    shapes = synth.transformer_grad_shapes(layers=layers)
    numels = [synth.numel(s) for _, s in shapes]
    total = sum(numels)
    offs = [0]
    for n in numels:
        offs.append(offs[-1] + n)

    def views(flat):
        return [flat[offs[i]:offs[i + 1]].view(shapes[i][1]) for i in range(len(numels))]

    host = []
    for r in range(N_SIM):
        h = torch.empty(total, dtype=torch.float32, pin_memory=pinned_inputs)
        h.numpy()[:] = synth.normal_f32(seed, r, total, 1e-3)
        host.append(h)
    dev_in = [h.to("cuda", non_blocking=False) for h in host]
    dev_out = [torch.empty_like(d) for d in dev_in]
    return dict(shapes=shapes, numels=numels, total=total, host=host, views=views,
                dev_in=[views(d) for d in dev_in], dev_out=[views(d) for d in dev_out],
                dev_in_flat=dev_in, dev_out_flat=dev_out)


def oracle_sample_seconds(numels, rank_arrays, base, nbuckets):
    """The oracle (message-passing simulator) on the first `nbuckets` buckets of the same
    host data; rank_arrays[r] holds rank r's flat gradients from element `base` on.
    Returns (seconds, bytes of N·T in + N·T out covered, elements per rank covered)."""
    import numpy as np
    from oracle import ddp
    from oracle.collectives import ring_allreduce
    buckets = ddp.assign_buckets(numels)[:nbuckets]
    offs = np.cumsum([0] + list(numels)) - base
    t0 = time.perf_counter()
    moved = 0
    for members in buckets:
        flats = [np.concatenate([a[offs[i]:offs[i + 1]] for i in members]) for a in rank_arrays]
        ring_allreduce(flats, scale=1.0 / N_SIM)
        moved += 2 * N_SIM * flats[0].nbytes
    return time.perf_counter() - t0, moved, sum(sum(numels[i] for i in m) for m in buckets)


def sample_range(numels, nbuckets):
    """[lo, hi) of the flat per-rank buffer that the first nbuckets buckets cover."""
    import numpy as np
    from oracle import ddp
    offs = np.cumsum([0] + list(numels))
    members = [i for m in ddp.assign_buckets(numels)[:nbuckets] for i in m]
    return int(min(offs[i] for i in members)), int(max(offs[i + 1] for i in members))


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    shapes = synth.transformer_grad_shapes(layers=args.layers)
    numels = [synth.numel(s) for _, s in shapes]
    lo, hi = sample_range(numels, 1)
    arrays = [synth.normal_f32(SEED, r, hi - lo, 1e-3, start=lo) for r in range(N_SIM)]
    times = []
    moved = elems = 0
    for step in range(args.warmup + args.steps):
        dt, moved, elems = oracle_sample_seconds(numels, arrays, lo, 1)
        if step >= args.warmup:
            times.append(dt)
    t = sum(times) / len(times)
    v = moved / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": workload_desc(args.layers), "sample": "bucket 0 of 17 per step"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"bucket 0 ({elems} fp32 per rank, {N_SIM} ranks) per step"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ---- the other hot-path rows: configs 1, 3, 4 and 5 ---------------------------------------------------

SPIN_CYCLES = 200_000  # about 0.1 ms of spinning at the B200's 1.97 GHz SM clock


def _event_time_ms(torch, fn, iters, flush=None, host_launch=False):
    """Sum of per-iteration CUDA-event times of fn() on the current stream; `flush` (outside
    the timed spans) evicts L2 between iterations when the working set would fit in it.
    Each span opens on a busy GPU (behind the flush, else behind a ~0.1 ms spin kernel), so it
    holds the device time of fn and not the host's cost of launching it; host_launch=True
    leaves the GPU idle before each span, which counts that cost too."""
    total = 0.0
    stream = torch.cuda.current_stream()
    for _ in range(iters):
        if flush is not None:
            flush()
        elif not host_launch:
            torch.cuda._sleep(SPIN_CYCLES)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    return total


def _prepared(cc, name, *args):
    """A C entry point with its arguments marshalled once (timed spans hold only the call)."""
    fn = getattr(cc.get_lib(), name)

    def call():
        st = fn(*args)
        if st != cc.CC_OK:
            raise RuntimeError(f"{name}: status {st}")
    return call


def roofline_fields(achieved, peak, peak_kind):
    """The fraction against the measured copy rate (a torch copy_, not a hard ceiling: a
    read-heavy kernel can pass it) and against the nominal 8 TB/s, side by side."""
    return {"achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_kind": peak_kind, "frac_of_nominal_8TBps": achieved / NOMINAL_HBM_GBS, "bound": "hbm"}


def timed_row(torch, call, iters, nbytes, launches_per_call, *, flush=None, warmup=3, local=0, **extra):
    """One measured row: device time per call from CUDA events (after `warmup` untimed calls;
    spans opened on a busy GPU, see _event_time_ms), the algorithmic bytes, GB/s against the
    measured copy rate, and the clocks sampled while the timed calls ran."""
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        ms = _event_time_ms(torch, call, iters, flush) / iters
    peak, kind = measured_peak()
    gbps = nbytes / (ms * 1e-3) / 1e9
    row = {"ms": ms, "bytes": nbytes, "GBps": gbps, "roofline": roofline_fields(gbps, peak, kind),
           "gpu_launches": launches_per_call * iters, "clocks": clk.summary()}
    row.update(extra)
    return row


def _us(ms):
    return None if ms is None else ms * 1e3


def _flusher(torch):
    buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")  # 256 MiB write, twice the L2
    return lambda: buf.fill_(1.0)


def rows_config1(torch, cc, local, with_cpu=True):
    """Config 1: N = 4 simulated ranks, 4096 elements per rank, fp32 U[-1,1] and int32
    U[-1000,1000]: ring allreduce, reduce-scatter, allgather (latency-bound: 16 KiB per rank;
    L2 flushed before every timed call)."""
    import synth
    n, count = 4, 4096
    st = torch.cuda.current_stream().cuda_stream
    flush = _flusher(torch)
    rows = {}
    host = {}
    for kind in ("f32", "i32"):
        if kind == "f32":
            xs = [synth.uniform_f32(1, r, count) for r in range(n)]
            dt, tdt = cc.CC_F32, torch.float32
        else:
            xs = [synth.int32_uniform(1, r, count, -1000, 1000) for r in range(n)]
            dt, tdt = cc.CC_I32, torch.int32
        host[kind] = xs
        send = [torch.from_numpy(x).cuda() for x in xs]
        y = [torch.empty(count, dtype=tdt, device="cuda") for _ in range(n)]
        shards = [torch.empty(count // n, dtype=tdt, device="cuda") for _ in range(n)]
        ag = [torch.empty(count, dtype=tdt, device="cuda") for _ in range(n)]
        T = count * 4
        calls = {}
        for algo in ("ring", "tree"):
            calls[f"allreduce_{algo}_{kind}"] = (2 * n * T, lambda h, a=algo: _prepared(
                cc, "cc_allreduce", cc._ptrs(send), cc._ptrs(y), n, count, dt, dt, cc.CC_SUM,
                cc.CC_ALGO_RING if a == "ring" else cc.CC_ALGO_TREE, 1.0, h))
        calls[f"reduce_scatter_{kind}"] = ((n + 1) * T, lambda h: _prepared(
            cc, "cc_reduce_scatter", cc._ptrs(send), cc._ptrs(shards), n, count, dt, dt, cc.CC_SUM, cc.CC_ALGO_RING,
            1.0, h))
        calls[f"allgather_{kind}"] = ((n + 1) * T, lambda h: _prepared(
            cc, "cc_allgather", cc._ptrs(shards), cc._ptrs(ag), n, count, dt, h))
        for name, (nbytes, make) in calls.items():
            rows[name] = timed_row(torch, make(st), 200, nbytes, 1, flush=flush, local=local)
            rows[name]["device_us"] = _us(graph_time_ms(torch, make))
            rows[name]["roofline"]["bound"] = "latency"  # a few microseconds per call, not bytes
    for r in rows.values():
        r["us"] = r["ms"] * 1e3
    out = {"workload": "config 1: N=4 simulated ranks x 4096 elements, fp32 U[-1,1] and int32 U[-1000,1000] "
                       "(host-seeded), ring allreduce / reduce-scatter / allgather and tree allreduce; latency-bound",
           "l2": "256 MiB flush before every timed call",
           "timing": "us: CUDA events around each call, opened behind the L2 flush; device_us: the same calls "
                     "replayed from a CUDA graph, flush graph subtracted",
           "rows": rows}
    if with_cpu:
        from oracle import collectives as C
        dt, reps, tot = _timed_cpu(lambda: C.ring_allreduce(host["f32"]))
        out["cpu_baseline"] = {"value": 2 * n * count * 4 / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": f"the whole config (fp32 ring allreduce), {reps} runs in {tot:.1f} s"}
    return out


def rows_config3(torch, cc, gen, local, iters, with_cpu=True):
    """Config 3 (ZeRO): N = 8, 300M fp32 per rank normal(0, 1e-2): ring reduce-scatter to
    37.5M-element shards, allgather of the shards, and the bf16-input reduce-scatter with fp32
    accumulation (device-seeded inputs; all far larger than L2)."""
    n, count = N_SIM, 300_000_000
    x = [torch.randn(count, device="cuda", generator=gen) * 1e-2 for _ in range(n)]
    shard = count // n
    rs = [torch.empty(shard, device="cuda") for _ in range(n)]
    ag = [torch.empty(count, device="cuda") for _ in range(n)]
    st = torch.cuda.current_stream().cuda_stream
    T = count * 4
    rs_call = _prepared(cc, "cc_reduce_scatter", cc._ptrs(x), cc._ptrs(rs), n, count, cc.CC_F32, cc.CC_F32,
                        cc.CC_SUM, cc.CC_ALGO_RING, 1.0, st)
    ag_call = _prepared(cc, "cc_allgather", cc._ptrs(rs), cc._ptrs(ag), n, count, cc.CC_F32, st)
    rows = {"reduce_scatter_f32": timed_row(torch, rs_call, iters, (n + 1) * T, 1, local=local,
                                            kernel="reduce_kernel<f32,sum,ring> (reduce-scatter)"),
            "allgather_f32": timed_row(torch, ag_call, iters, (n + 1) * T, 1, local=local,
                                       kernel="copy_bulk_tile_kernel (TMA fan-out)")}
    del ag, ag_call
    xb = [t.to(torch.bfloat16) for t in x]
    del x, rs_call
    bf_call = _prepared(cc, "cc_reduce_scatter", cc._ptrs(xb), cc._ptrs(rs), n, count, cc.CC_BF16, cc.CC_F32,
                        cc.CC_SUM, cc.CC_ALGO_RING, 1.0, st)
    rows["reduce_scatter_bf16_in_f32_out"] = timed_row(torch, bf_call, iters, n * T // 2 + T, 1, local=local,
                                                       kernel="reduce_kernel<bf16,sum,ring> (reduce-scatter)")
    del xb, bf_call, rs
    torch.cuda.empty_cache()
    ms = rows["reduce_scatter_f32"]["ms"] + rows["allgather_f32"]["ms"]
    out = {"workload": "config 3 (ZeRO): N=8 simulated ranks, 300M fp32 per rank normal(0,1e-2), ring reduce-scatter "
                       "to 37.5M-element shards, allgather of the shards; bf16-input reduce-scatter with fp32 "
                       "accumulation (device-seeded inputs)",
           "l2": "inputs larger than L2; no flush", "rows": rows,
           "rs_plus_ag": {"ms": ms, "metric_GBps": 2 * n * T / (ms * 1e-3) / 1e9},
           "traffic_profile": profile_traffic("reduce_scatter_allgather_zero.txt")}
    if with_cpu:
        import numpy as np
        import synth
        from oracle import collectives as C
        k = 1 << 20  # sampled positions per rank, spread over every chunk of the full count
        pos = np.unique(np.linspace(0, count - 1, k).astype(np.int64))
        xs = [synth.normal_f32(SEED, r, len(pos), 1e-2, stream=3) for r in range(n)]
        def rs_ag():
            sh, _ = C.ring_reduce_scatter(xs, count=count, positions=pos)
            C.ring_allgather(sh, count=count, positions=pos)
        dt, reps, tot = _timed_cpu(rs_ag)
        out["cpu_baseline"] = {"value": 2 * n * len(pos) * 4 / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": f"reduce-scatter + allgather on {len(pos)} sampled positions per rank "
                                         f"(full-size chunk map), {reps} runs in {tot:.1f} s"}
    return out


def rows_config4(torch, cc, gen, local, iters, with_cpu=True):
    """Config 4 (MoE): N = 8, 8192 tokens x 4096 bf16 per rank, 64 experts (8 per rank), top-2
    routing from normal router logits; dispatch, then the inverse combine."""
    n, tokens, hidden, epr, topk = N_SIM, 8192, 4096, 8, 2
    E = n * epr
    logits = [torch.randn(tokens, E, device="cuda", generator=gen) for _ in range(n)]
    toks = [torch.randn(tokens, hidden, device="cuda", generator=gen).to(torch.bfloat16) for _ in range(n)]
    ids = [torch.empty(tokens, topk, dtype=torch.int32, device="cuda") for _ in range(n)]
    cc.cc_route_topk(logits, ids)
    ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, topk, epr) // 4 + 64, dtype=torch.int32, device="cuda")
    cap = tokens * topk * 2
    recv = [torch.empty(cap, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    back = [torch.empty(tokens, topk, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    counts = torch.zeros(n, dtype=torch.int32, device="cuda")
    cc.cc_alltoallv(toks, recv, ids, epr, ws, direction=0)
    cc.cc_alltoallv_recv_counts(ws, n, counts)
    torch.cuda.synchronize()
    rows_recv = int(counts.sum().item())
    row = hidden * 2
    st = torch.cuda.current_stream().cuda_stream
    wsb = ws.numel() * 4
    route = _prepared(cc, "cc_route_topk", cc._ptrs(logits), cc._ptrs(ids), n, tokens, E, topk, st)
    disp = _prepared(cc, "cc_alltoallv", cc._ptrs(toks), cc._ptrs(recv), n, row, cc._ptrs(ids), tokens, topk, epr,
                     cap, 0, ws.data_ptr(), wsb, st)
    comb = _prepared(cc, "cc_alltoallv", cc._ptrs(recv), cc._ptrs(back), n, row, cc._ptrs(ids), tokens, topk, epr,
                     cap, 1, ws.data_ptr(), wsb, st)
    plan = _prepared(cc, "cc_alltoallv_plan", cc._ptrs(ids), n, tokens, topk, epr, ws.data_ptr(), wsb, st)
    disp_run = _prepared(cc, "cc_alltoallv_run", cc._ptrs(toks), cc._ptrs(recv), n, row, cc._ptrs(ids), tokens,
                         topk, epr, cap, 0, ws.data_ptr(), wsb, st)
    comb_run = _prepared(cc, "cc_alltoallv_run", cc._ptrs(recv), cc._ptrs(back), n, row, cc._ptrs(ids), tokens,
                         topk, epr, cap, 1, ws.data_ptr(), wsb, st)
    b_d = n * tokens * row + rows_recv * row
    b_c = 2 * rows_recv * row
    b_ids = n * tokens * topk * 4
    rows = {"route_topk": timed_row(torch, route, iters, n * tokens * E * 4 + b_ids, 1, local=local),
            "dispatch": timed_row(torch, disp, iters, b_d, A2A_LAUNCHES, local=local,
                                  kernel="alltoallv dispatch (routing tables + row copy)"),
            "combine": timed_row(torch, comb, iters, b_c, A2A_LAUNCHES, local=local,
                                 kernel="alltoallv combine (routing tables + row copy)"),
            # one routing plan, then the copies alone: the combine reuses the dispatch's routes
            "plan": timed_row(torch, plan, iters, b_ids, 1, local=local,
                              kernel="alltoallv routing tables alone (latency-bound: bytes are the ids)"),
            "dispatch_run": timed_row(torch, disp_run, iters, b_d, 1, local=local,
                                      kernel="alltoallv dispatch row copy over a plan"),
            "combine_run": timed_row(torch, comb_run, iters, b_c, 1, local=local,
                                     kernel="alltoallv combine row copy over a plan")}
    for k in ("route_topk", "plan"):  # microseconds of dependent steps, not bytes
        rows[k]["roofline"]["bound"] = "latency"
    ms = sum(rows[k]["ms"] for k in ("route_topk", "dispatch", "combine"))
    ms_plan = sum(rows[k]["ms"] for k in ("route_topk", "plan", "dispatch_run", "combine_run"))
    out = {"workload": "config 4 (MoE): N=8 simulated ranks, 8192 tokens x 4096 bf16 per rank, 64 experts (8 per "
                       "rank), top-2 routing from normal logits, dispatch then combine (device-seeded inputs)",
           "l2": "inputs larger than L2; no flush", "rows": rows, "rows_routed_total": rows_recv,
           "route_dispatch_combine": {"ms": ms, "GBps": (b_d + b_c) / (ms * 1e-3) / 1e9},
           "route_plan_dispatch_combine": {"ms": ms_plan, "GBps": (b_d + b_c) / (ms_plan * 1e-3) / 1e9},
           "traffic_profile": profile_traffic("alltoallv_dispatch_moe.txt")}
    del logits, toks, ids, ws, recv, back
    torch.cuda.empty_cache()
    if with_cpu:
        import numpy as np
        import synth
        from oracle import moe
        t_s = 1024  # sampled tokens per rank
        lg = [synth.normal_f32(SEED, r, t_s * E, stream=5).reshape(t_s, E) for r in range(n)]
        tk = [synth.to_bf16_bits(synth.normal_f32(SEED, r, t_s * hidden, stream=6)).reshape(t_s, hidden)
              for r in range(n)]
        def rdc():
            eid = [moe.route_topk(l, topk) for l in lg]
            d, _ = moe.dispatch(tk, eid, epr)
            moe.combine(d, eid, epr)
        dt, reps, tot = _timed_cpu(rdc)
        nb = n * t_s * row + 3 * n * t_s * topk * row
        out["cpu_baseline"] = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": f"route + dispatch + combine of {t_s} tokens per rank, {reps} runs in "
                                         f"{tot:.1f} s"}
    return out


def graph_time_ms(torch, make_call, iters=20, reps=5, flush_bytes=256 * 1024 * 1024):
    """Device time per call, without the host's per-call launch cost: `iters` calls captured in
    one CUDA graph on a side stream, each preceded by an L2 flush (a write of flush_bytes),
    replayed `reps` times (median); a graph of the flushes alone is timed the same way and
    subtracted. make_call(stream_handle) returns the call. None if the capture fails."""
    s = torch.cuda.Stream()
    call = make_call(s.cuda_stream)
    buf = torch.empty(flush_bytes // 4, device="cuda") if flush_bytes else None
    with torch.cuda.stream(s):
        for _ in range(3):
            call()
    torch.cuda.synchronize()

    def capture(with_call):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(iters):
                if buf is not None:
                    buf.fill_(1.0)
                if with_call:
                    call()
        return g

    def replay_ms(g):
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(s):  # the graph runs on s, between the two events
                a.record(s)
                g.replay()
                b.record(s)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    try:
        g1 = capture(True)
        g0 = capture(False) if buf is not None else None
    except Exception:
        torch.cuda.synchronize()
        return None
    t = (replay_ms(g1) - (replay_ms(g0) if g0 is not None else 0.0)) / iters
    del g1, g0
    return max(t, 0.0)


def launch_latency_s(torch, cc, st):
    """Median CUDA-event time of a minimal cc_allreduce (N = 8 ranks x 4 elements), the
    per-call startup cost that the alpha of the alpha-beta model stands for."""
    x = [torch.zeros(4, device="cuda") for _ in range(8)]
    call = _prepared(cc, "cc_allreduce", cc._ptrs(x), cc._ptrs(x), 8, 4, cc.CC_F32, cc.CC_F32, cc.CC_SUM,
                     cc.CC_ALGO_RING, 1.0, st)
    for _ in range(10):
        call()
    times = [_event_time_ms(torch, call, 1, host_launch=True) for _ in range(200)]
    return statistics.median(times) * 1e-3


def _timed_cpu(fn, min_s=2.0):
    """Seconds per run of fn(), repeated until min_s have passed (at least once)."""
    t0 = time.perf_counter()
    reps = 0
    while True:
        fn()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            return dt / reps, reps, dt


def alpha_beta_crossover(n, alpha_ring, alpha_tree, bw_ring, bw_tree):
    """Message size per rank (bytes) above which the ring's time drops below the tree's in
    the alpha-beta model of lecture 09 §7.3 / appendix A Q3:
        T_ring = 2(N-1)·alpha + 2(N-1)/N · M / B_ring,   T_tree = 2·ceil(log2 N)·alpha + 2·M / B_tree.
    None when one of them is faster at every size."""
    import math
    steps_tree = 2 * math.ceil(math.log2(n)) if n > 1 else 0
    lat = 2 * (n - 1) * alpha_ring - steps_tree * alpha_tree   # the ring's extra latency
    per_byte = 2.0 / bw_tree - 2.0 * (n - 1) / n / bw_ring     # the tree's extra time per byte
    if lat <= 0 or per_byte <= 0:
        return None
    return lat / per_byte


def crossover_reading(n, alpha_ring, alpha_tree, bw_ring, bw_tree):
    """The model's answer in words: the crossover size, or which schedule is faster at every
    size (and why) when there is none."""
    import math
    m = alpha_beta_crossover(n, alpha_ring, alpha_tree, bw_ring, bw_tree)
    if m is not None:
        return f"ring faster above {m / 1e6:.3g} MB per rank, tree below"
    steps_tree = 2 * math.ceil(math.log2(n)) if n > 1 else 0
    ring_lat = 2 * (n - 1) * alpha_ring > steps_tree * alpha_tree
    ring_byte = 2.0 * (n - 1) / n / bw_ring > 2.0 / bw_tree
    if ring_lat and ring_byte:
        return "no crossover: the tree is faster at every size (smaller latency and per-byte terms)"
    if not ring_lat and not ring_byte:
        return "no crossover: the ring is at least as fast at every size (latency and per-byte terms no larger)"
    return "no crossover"


def fit_alpha_beta(n, small_bytes, t_small, large_bytes, t_large, algo):
    """alpha from the smallest message (its time over the schedule's step count) and the
    bandwidth B from the largest (M over the model's bandwidth term), per algorithm."""
    import math
    steps = 2 * (n - 1) if algo == "ring" else 2 * math.ceil(math.log2(n))
    alpha = t_small / max(1, steps)
    bw = (2.0 * (n - 1) / n if algo == "ring" else 2.0) * large_bytes / t_large
    return alpha, bw


def rows_config5(torch, cc, gen, local, with_cpu=True):
    """Config 5, its large points and the ring-vs-tree crossover at N = 8: the fused ring and
    tree allreduce at N = 8 x 256 MiB and N = 64 x 64 MiB, the stepped (schedule-faithful)
    ring and tree at N = 8 x 1 KiB and x 256 MiB, the alpha-beta model crossover from those,
    and the measured launch latency of a minimal call."""
    st = torch.cuda.current_stream().cuda_stream
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    flush = _flusher(torch)
    rows = {}
    stepped = {}
    for n, size in ((8, 256 * 1024 * 1024), (64, 64 * 1024 * 1024), (8, 1024)):
        count = size // 4
        x = [torch.rand(count, device="cuda", generator=gen) * 2 - 1 for _ in range(n)]
        y = [torch.empty_like(t) for t in x]
        small = 2 * n * size < 126 * 1024 * 1024
        for algo in ("ring", "tree"):
            a = cc.CC_ALGO_RING if algo == "ring" else cc.CC_ALGO_TREE
            key = f"n{n}_{_size_name(size)}_{algo}"
            if size >= 1024 * 1024:
                call = _prepared(cc, "cc_allreduce", cc._ptrs(x), cc._ptrs(y), n, count, cc.CC_F32, cc.CC_F32,
                                 cc.CC_SUM, a, 1.0, st)
                rows[key] = timed_row(torch, call, 10, 2 * n * size, 1, local=local, flush=flush if small else None,
                                      kernel=f"reduce_kernel<f32,sum,{algo}>")
            if n == 8:
                make = (lambda h, a=a: _prepared(cc, "cc_allreduce_stepped", cc._ptrs(x), cc._ptrs(y), n, count,
                                                 cc.CC_F32, cc.CC_F32, cc.CC_SUM, a, 1.0, ws.data_ptr(),
                                                 ws.numel() * 4, h))
                r = timed_row(torch, make(st), 10 if size > 1024 * 1024 else 50, 2 * n * size, 1, local=local,
                              flush=flush if small else None, kernel=f"stepped_kernel ({algo}, one launch)",
                              own_traffic_bytes=stepped_traffic(n, count, 4, algo))
                r["own_traffic_GBps"] = r["own_traffic_bytes"] / (r["ms"] * 1e-3) / 1e9
                r["own_traffic_frac"] = r["own_traffic_GBps"] / measured_peak()[0]
                if small:  # 2(N-1) or 2 depth dependent steps of a few KiB each
                    r["roofline"]["bound"] = "latency"
                t = r["ms"] * 1e-3
                if small:
                    r["device_us"] = _us(graph_time_ms(torch, make))
                    if r["device_us"] is not None:
                        t = r["device_us"] * 1e-6
                rows["stepped_" + key] = r
                stepped[(size, algo)] = t
        if n == 8 and size >= 1024 * 1024:
            for K in (2, 4):
                call = _prepared(cc, "cc_allreduce_multiring", cc._ptrs(x), cc._ptrs(y), n, K, count, cc.CC_F32,
                                 cc.CC_F32, cc.CC_SUM, 1.0, st)
                rows[f"n{n}_{_size_name(size)}_multiring{K}"] = timed_row(
                    torch, call, 10, 2 * n * size, 1, local=local,
                    kernel=f"reduce_kernel<f32,sum,multi-ring K={K}>")
        del x, y
    lat = launch_latency_s(torch, cc, st)
    x = [torch.zeros(4, device="cuda") for _ in range(8)]
    lat_dev = graph_time_ms(torch, lambda h: _prepared(cc, "cc_allreduce", cc._ptrs(x), cc._ptrs(x), 8, 4, cc.CC_F32,
                                                       cc.CC_F32, cc.CC_SUM, cc.CC_ALGO_RING, 1.0, h))
    n, small, large = 8, 1024, 256 * 1024 * 1024
    ar, br = fit_alpha_beta(n, small, stepped[(small, "ring")], large, stepped[(large, "ring")], "ring")
    at, bt = fit_alpha_beta(n, small, stepped[(small, "tree")], large, stepped[(large, "tree")], "tree")
    model = {"n": n, "alpha_ring_us": ar * 1e6, "alpha_tree_us": at * 1e6, "B_ring_GBps": br / 1e9,
             "B_tree_GBps": bt / 1e9, "launch_latency_us": lat * 1e6, "minimal_call_device_us": _us(lat_dev),
             "alpha_from": "the stepped schedules' 1 KiB time (CUDA-graph device time) over their step counts; "
                           "B from their 256 MiB time",
             "crossover_fitted_alpha_bytes": alpha_beta_crossover(n, ar, at, br, bt),
             "crossover_fitted_alpha": crossover_reading(n, ar, at, br, bt),
             "crossover_launch_alpha_bytes": alpha_beta_crossover(n, lat, lat, br, bt),
             "crossover_launch_alpha": crossover_reading(n, lat, lat, br, bt)}
    out = {"workload": "config 5 large points: fused ring / tree allreduce, N=8 x 256 MiB and N=64 x 64 MiB fp32 "
                       "U[-1,1] (device-seeded); stepped ring / tree at N=8 x 1 KiB and 256 MiB",
           "l2": "256 MiB flush before each timed call whose working set fits in L2; the large points exceed it",
           "rows": rows, "alpha_beta_model_n8": model}
    if with_cpu:
        import numpy as np
        import synth
        from oracle import collectives as C
        count = 256 * 1024 * 1024 // 4
        pos = np.unique(np.linspace(0, count - 1, 1 << 19).astype(np.int64))
        xs = [synth.uniform_f32(SEED, r, len(pos), stream=7) for r in range(8)]
        dt, reps, tot = _timed_cpu(lambda: C.ring_allreduce(xs, count=count, positions=pos))
        out["cpu_baseline"] = {"value": 2 * 8 * len(pos) * 4 / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": f"N=8 ring allreduce on {len(pos)} sampled positions per rank of the "
                                         f"256 MiB buffer, {reps} runs in {tot:.1f} s"}
    return out


def _size_name(b):
    return f"{b >> 20}MiB" if b >= 1 << 20 else f"{b >> 10}KiB"


def stepped_traffic(n, count, elem, algo):
    """Bytes the stepped schedule itself moves when not in place: the copy-in (N·T read, N·T
    written), then ring reduce-scatter steps that read the own and the left neighbour's chunk
    and write the own (3 accesses per chunk and rank), allgather steps that read the left
    neighbour's chunk and write the own (2); tree up steps read a node and its children and
    write the node, down steps read the parent and write the node. Each tree has N // 2
    interior nodes (the even labels) and N - 1 child links, so over both halves the tree
    moves (2·(N // 2) + 3(N - 1))·T."""
    T = count * elem
    if n == 1:
        return 2 * T
    if algo == "ring":
        return 2 * n * T + 5 * (n - 1) * T
    return 2 * n * T + (2 * (n // 2) + 3 * (n - 1)) * T


A2A_LAUNCHES = 2  # routing tables (one launch) + row copy per alltoallv call


# ---- one rank per GPU: the DDP step as a real collective over NVLink ---------------------------------

def bucket_order_layout(numels, cap=CAP):
    """Flat per-rank layout of the gradients in bucket order (cc_bucket_assign's order: reverse
    registration order, 25 MiB buckets), so that every bucket is one contiguous range.
    Returns (offset of each tensor in the flat buffer, [(bucket start, bucket count)])."""
    import collective_communication_primitives_rank_b200 as cc
    offs = [0] * len(numels)
    ranges = []
    pos = 0
    for members in cc.cc_bucket_assign(list(numels), 4, cap):
        start = pos
        for i in members:
            offs[i] = pos
            pos += numels[i]
        ranges.append((start, pos - start))
    return offs, ranges


def offset_ptrs(ptrs, elems, elem_bytes=4):
    """The same N device pointers advanced by `elems` elements (a bucket inside every rank's
    flat buffer)."""
    return [int(p) + elems * elem_bytes for p in ptrs]


def run_multi_gpu(args):
    """One rank per GPU (torchrun): each rank holds its own fp32 gradients of the config-2
    model (rank r's values are simulated rank r's of the single-GPU workload), laid out flat in
    bucket order. One step = every bucket allreduced (ring order, mean) by libcc's slice
    calls over CUDA IPC peer mappings: rank c folds chunk c of the bucket from every GPU and
    writes it into every GPU (plain loads and stores over NVLink), the ranks ordered by a
    stream synchronisation and a group barrier before and after the step. NCCL's all_reduce
    of the same buckets is timed beside it, and NCCL's all_gather bus bandwidth serves as the
    measured NVLink rate. Rank 0 then checks its output bit for bit against the single-GPU
    fused call (cc_bucket_allreduce) over all ranks' gradients regenerated on its own GPU."""
    import ctypes
    import datetime
    import torch
    import torch.distributed as dist
    import collective_communication_primitives_rank_b200 as cc
    import synth
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    # CC_BENCH_BACKEND=gloo with CC_BENCH_DEVICE=0 runs every rank's process on one GPU with host
    # barriers over gloo and without the NCCL comparator: the slice path's plumbing (layout, IPC
    # mappings, the step, the parity check) on a machine with fewer GPUs than ranks. The ranks'
    # kernels never wait on one another; the host barriers order them.
    backend = os.environ.get("CC_BENCH_BACKEND", "nccl")
    device = int(os.environ.get("CC_BENCH_DEVICE", local))
    torch.cuda.set_device(device)
    for k, v in (("MASTER_ADDR", "127.0.0.1"), ("MASTER_PORT", "29531"), ("RANK", str(rank)),
                 ("WORLD_SIZE", str(world))):
        os.environ.setdefault(k, v)
    if not dist.is_initialized():
        if backend == "nccl":
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", device))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    nccl = backend == "nccl"
    mdev = "cuda" if nccl else "cpu"  # where the max over ranks is reduced
    shapes = synth.transformer_grad_shapes(layers=args.layers)
    numels = [synth.numel(s) for _, s in shapes]
    total = sum(numels)
    offs, ranges = bucket_order_layout(numels)
    host = torch.empty(total, dtype=torch.float32, pin_memory=True)
    reg = synth.normal_f32(SEED, rank, total, 1e-3)  # registration order, as the single-GPU workload
    for i, n_i in enumerate(numels):
        a = sum(numels[:i])
        host.numpy()[offs[i]:offs[i] + n_i] = reg[a:a + n_i]
    del reg
    send = host.to("cuda")
    recv = torch.empty_like(send)
    stream = torch.cuda.current_stream()
    peers = cc.PeerGroup([send, recv])
    lib = cc.get_lib()
    sp, rp = peers.buffers(0), peers.buffers(1)
    sp = [t.data_ptr() if isinstance(t, torch.Tensor) else t for t in sp]
    rp = [t.data_ptr() if isinstance(t, torch.Tensor) else t for t in rp]
    calls = []
    for start, count in ranges:
        s_arr = (ctypes.c_void_p * world)(*offset_ptrs(sp, start))
        r_arr = (ctypes.c_void_p * world)(*offset_ptrs(rp, start))
        calls.append((s_arr, r_arr, count))

    def launch_slices():
        for s_arr, r_arr, count in calls:
            stt = lib.cc_allreduce_slice(s_arr, r_arr, world, rank, count, cc.CC_F32, cc.CC_F32, cc.CC_SUM,
                                         cc.CC_ALGO_RING, cc.CC_SCALE_MEAN, stream.cuda_stream)
            if stt != cc.CC_OK:
                raise RuntimeError(f"cc_allreduce_slice: status {stt}")

    def step(before=False):
        # every rank's slices of a step are done on every GPU once the barrier after it has
        # passed, so back-to-back steps need no barrier before (the inputs did not change);
        # a step whose inputs were just rewritten (the end-to-end copy in) takes one
        if before:
            stream.synchronize()
            dist.barrier()
        launch_slices()
        stream.synchronize()
        dist.barrier()

    def timed(fn, steps):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        return max_over_ranks(dist, torch, a.elapsed_time(b) / steps, mdev)

    with Clocks(device) as clk:
        ms = timed(step, args.steps)
    T = total * 4
    value = aggregate_gbps(world, 2 * T, ms)
    bus = 2.0 * (world - 1) / world * T / (ms * 1e-3) / 1e9

    # NCCL: all_reduce of the same buckets (sum), and all_gather of 256 MiB shards as the
    # measured NVLink rate
    ms_nccl, ag_busbw = None, 0.0
    if nccl:
        x = send.clone()

        def nccl_step():
            for start, count in ranges:
                dist.all_reduce(x[start:start + count])

        ms_nccl = timed(nccl_step, args.steps)
        shard = torch.empty(64 * 1024 * 1024, device="cuda")
        gathered = torch.empty(world * shard.numel(), device="cuda")
        ms_ag = timed(lambda: dist.all_gather_into_tensor(gathered, shard), max(3, args.steps // 2))
        ag_busbw = (world - 1) * shard.numel() * 4 / (ms_ag * 1e-3) / 1e9
        del x, gathered, shard

    # end to end: pinned host gradients -> device, the step, device -> pinned host
    host_out = torch.empty_like(host, pin_memory=True)

    def e2e_step():
        send.copy_(host, non_blocking=True)
        step(before=True)
        host_out.copy_(recv, non_blocking=True)

    ems = timed(e2e_step, args.e2e_steps)

    # parity: rank 0's output against the single-GPU fused call over every rank's gradients
    parity = None
    if rank == 0:
        flat_in = [torch.empty(total, device="cuda") for _ in range(world)]
        flat_out = [torch.empty(total, device="cuda") for _ in range(world)]
        for r in range(world):
            reg = torch.from_numpy(synth.normal_f32(SEED, r, total, 1e-3))
            for i, n_i in enumerate(numels):
                a = sum(numels[:i])
                flat_in[r][offs[i]:offs[i] + n_i].copy_(reg[a:a + n_i])
        views = lambda f: [f[offs[i]:offs[i] + n_i] for i, n_i in enumerate(numels)]
        cc.cc_bucket_allreduce([views(f) for f in flat_in], [views(f) for f in flat_out], cap_bytes=CAP)
        step()
        torch.cuda.synchronize()
        parity = "bit-exact" if torch.equal(recv.view(torch.int32), flat_out[0].view(torch.int32)) else "MISMATCH"
        del flat_in, flat_out
    else:
        step()
    dist.barrier()
    peers.close()
    dist.barrier()
    if rank == 0:
        peak = ag_busbw
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"ddp_bucket_allreduce across GPUs: {world} ranks, one per GPU, each with its own "
                                   f"fp32 gradients of the {args.layers}-layer d=768 transformer (flat, bucket order, "
                                   "25 MiB buckets), ring-order allreduce with the 1/N mean by cc_allreduce_slice "
                                   "over CUDA IPC, host barriers included",
                       "ranks": world, "bytes_per_rank": T, "buckets": len(ranges),
                       "l2": "inputs larger than L2; no flush", "parallelism": f"ranks x{world}"},
            "comm_nranks": world, "busbw": bus, "parity_rank0_vs_single_gpu": parity,
            "nccl": ({"ms_per_step": ms_nccl, "busbw": 2.0 * (world - 1) / world * T / (ms_nccl * 1e-3) / 1e9,
                      "all_gather_busbw": ag_busbw} if nccl else None),
            "backend": backend,
            "roofline": {"bound": "nvlink", "achieved": bus, "peak": peak, "unit": "GB/s",
                         "frac": bus / peak if peak > 0 else None,
                         "peak_kind": "NCCL all_gather bus bandwidth measured in this run", "traffic": None},
            "e2e": {"value": aggregate_gbps(world, 2 * T, ems), "unit": "GB/s", "h2d_bytes_per_step": world * T,
                    "d2h_bytes_per_step": world * T},
            "gpu_launches": len(ranges) * args.steps, "clocks": clk.summary()}))
    dist.destroy_process_group()
    return 0


def run_rows(args):
    """--workload zero / moe / sweep: one detailed line for that config alone."""
    import torch
    import collective_communication_primitives_rank_b200 as cc
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(SEED)
    iters = max(1, args.steps)
    cpu = not args.no_cpu_baseline
    if args.workload == "zero":
        d = rows_config3(torch, cc, gen, local, iters, cpu)
        print(json.dumps(_detail_line(args, METRIC, d["rs_plus_ag"]["metric_GBps"], d["rs_plus_ag"]["ms"], d,
                                      "reduce_scatter_f32", d["traffic_profile"])))
        return 0
    if args.workload == "moe":
        d = rows_config4(torch, cc, gen, local, iters, cpu)
        print(json.dumps(_detail_line(args, "alltoallv effective HBM GB/s (dispatch: tokens read once + routed rows "
                                            "written; combine: routed rows read + written)",
                                      d["route_dispatch_combine"]["GBps"], d["route_dispatch_combine"]["ms"], d,
                                      "dispatch", d["traffic_profile"], dtype="bf16 (bit copy)")))
        return 0
    return run_sweep(args, torch, cc, gen, local)


def _detail_line(args, metric, value, ms, d, top, traffic, dtype="f32"):
    row = d["rows"][top]
    line = {"metric": metric, "value": value, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dtype, "data": "synthetic",
            "config": {"workload": d["workload"], "l2": d["l2"]},
            "roofline": dict(row["roofline"], bound="hbm", traffic=traffic, kernel=row.get("kernel", top)),
            "gpu_launches": sum(r["gpu_launches"] for r in d["rows"].values()),
            "clocks": row["clocks"], "rows": d["rows"]}
    for k in ("cpu_baseline", "alpha_beta_model_n8"):
        if k in d:
            line[k] = d[k]
    return line


def run_sweep(args, torch, cc, gen, local):
    """Config 5: ring vs double-binary-tree allreduce, N in {2..64}, 1 KiB .. 256 MiB per rank,
    fused and stepped, with the measured crossovers and the alpha-beta model's crossover per N
    (alpha and B fitted per algorithm from the stepped schedule's smallest and largest points,
    and with the launch latency of a minimal call as alpha)."""
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    table = []
    best = None
    with Clocks(local) as clk:
        for n in (2, 4, 8, 16, 32, 64):
            for i in range(10):
                size = 1024 * 4 ** i
                count = size // 4
                if n * size > 16 * 1024 ** 3:
                    continue
                x = [torch.rand(count, device="cuda", generator=gen) * 2 - 1 for _ in range(n)]
                y = [torch.empty_like(t) for t in x]
                small = 2 * n * size < 2 * 126 * 1024 * 1024
                flush = (lambda: flush_buf.fill_(1.0)) if small else None
                reps = max(3, min(50, int(2e9 // (2 * n * size + 1))))
                row = {"n": n, "bytes_per_rank": size}
                for algo in ("ring", "tree"):
                    a = cc.CC_ALGO_RING if algo == "ring" else cc.CC_ALGO_TREE
                    call = _prepared(cc, "cc_allreduce", cc._ptrs(x), cc._ptrs(y), n, count, cc.CC_F32, cc.CC_F32,
                                     cc.CC_SUM, a, 1.0, st)
                    for _ in range(3):
                        call()
                    ms = _event_time_ms(torch, call, reps, flush) / reps
                    row[algo + "_us"] = ms * 1e3
                    row[algo + "_GBps"] = 2 * n * size / (ms * 1e-3) / 1e9
                    make = (lambda h, a=a: _prepared(cc, "cc_allreduce_stepped", cc._ptrs(x), cc._ptrs(y), n, count,
                                                     cc.CC_F32, cc.CC_F32, cc.CC_SUM, a, 1.0, ws.data_ptr(),
                                                     ws.numel() * 4, h))
                    stepped = make(st)
                    for _ in range(2):
                        stepped()
                    sreps = max(2, reps // 4)
                    ms = _event_time_ms(torch, stepped, sreps, flush) / sreps
                    if size <= 1024 * 1024:  # latency-bound: the device time, without the host's launch cost
                        dev = graph_time_ms(torch, make, iters=10, reps=3)
                        row[algo + "_stepped_event_us"] = ms * 1e3
                        if dev is not None:
                            ms = dev
                    row[algo + "_stepped_us"] = ms * 1e3
                    row[algo + "_stepped_GBps"] = 2 * n * size / (ms * 1e-3) / 1e9
                    row[algo + "_stepped_own_GBps"] = stepped_traffic(n, count, 4, algo) / (ms * 1e-3) / 1e9
                for K in (2, 4):
                    mr = _prepared(cc, "cc_allreduce_multiring", cc._ptrs(x), cc._ptrs(y), n, K, count, cc.CC_F32,
                                   cc.CC_F32, cc.CC_SUM, 1.0, st)
                    for _ in range(2):
                        mr()
                    ms = _event_time_ms(torch, mr, reps, flush) / reps
                    row[f"multiring{K}_GBps"] = 2 * n * size / (ms * 1e-3) / 1e9
                if n == 8:
                    bc = _prepared(cc, "cc_broadcast", x[0].data_ptr(), cc._ptrs(y), n, 0, count, cc.CC_F32, st)
                    ms = _event_time_ms(torch, bc, reps, flush) / reps
                    row["broadcast_GBps"] = (n + 1) * size / (ms * 1e-3) / 1e9
                table.append(row)
                if n == 8 and size == 256 * 1024 * 1024:
                    best = row
                del x, y
        hier = []
        for n, mib in ((16, 256), (64, 64)):
            count = mib * 1024 * 1024 // 4
            x = [torch.rand(count, device="cuda", generator=gen) * 2 - 1 for _ in range(n)]
            y = [torch.empty_like(t) for t in x]
            call = _prepared(cc, "cc_allreduce_hierarchical", cc._ptrs(x), cc._ptrs(y), n, 8, count, cc.CC_F32,
                             cc.CC_F32, cc.CC_SUM, 1.0, st)
            for _ in range(3):
                call()
            ms = _event_time_ms(torch, call, 5) / 5
            hier.append({"n": n, "ranks_per_node": 8, "bytes_per_rank": count * 4, "us": ms * 1e3,
                         "GBps": 2 * n * count * 4 / (ms * 1e-3) / 1e9})
            del x, y
        lat = launch_latency_s(torch, cc, st)
    cross, cross_stepped, model = {}, {}, {}
    for n in (2, 4, 8, 16, 32, 64):
        pts = [r for r in table if r["n"] == n]
        for key, dst in (("", cross), ("_stepped", cross_stepped)):
            over = [r["bytes_per_rank"] for r in pts if r["ring" + key + "_GBps"] > 1.03 * r["tree" + key + "_GBps"]]
            under = [r["bytes_per_rank"] for r in pts if r["tree" + key + "_GBps"] > 1.03 * r["ring" + key + "_GBps"]]
            dst[str(n)] = {"ring_faster_by_3pct_at": over, "tree_faster_by_3pct_at": under}
        lo, hi = pts[0], pts[-1]
        fits = {algo: fit_alpha_beta(n, lo["bytes_per_rank"], lo[algo + "_stepped_us"] * 1e-6, hi["bytes_per_rank"],
                                     hi[algo + "_stepped_us"] * 1e-6, algo) for algo in ("ring", "tree")}
        (ar, br), (at, bt) = fits["ring"], fits["tree"]
        model[str(n)] = {"alpha_ring_us": ar * 1e6, "alpha_tree_us": at * 1e6, "B_ring_GBps": br / 1e9,
                         "B_tree_GBps": bt / 1e9,
                         "crossover_fitted_alpha_bytes": alpha_beta_crossover(n, ar, at, br, bt),
                         "crossover_launch_alpha_bytes": alpha_beta_crossover(n, lat, lat, br, bt)}
    peak, kind = measured_peak()
    line = {"metric": METRIC, "value": best["ring_GBps"], "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": best["ring_us"] / 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "sweep: ring vs double-binary-tree allreduce, N in {2,4,8,16,32,64}, fp32 U[-1,1] "
                                   "1 KiB..256 MiB per rank (powers of 4), fused and stepped, and the multi-ring "
                                   "(K = 2, 4); headline value = N=8, 256 MiB, fused ring",
                       "l2": "L2 flushed (256 MiB write) before every timed call whose working set fits in L2"},
            "roofline": dict(roofline_fields(best["ring_GBps"], peak, kind), bound="hbm", traffic=None,
                             kernel="reduce_kernel<f32,sum,ring>"),
            "gpu_launches": None, "clocks": clk.summary(),
            "sweep": table, "crossover": cross, "crossover_stepped": cross_stepped, "alpha_beta_model": model,
            "launch_latency_us": lat * 1e6, "hierarchical": hier}
    print(json.dumps(line))
    return 0


def run_kernel(args):
    """--workload kernel: one collective call, repeated (warm-up, then --steps timed calls), on
    device-seeded fp32 inputs of --n ranks x --mib MiB: a small, fixed case for profilers.
    Prints the mean CUDA-event time per call (not a bench line)."""
    import torch
    import collective_communication_primitives_rank_b200 as cc
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(SEED)
    n, count = args.n, args.mib * 1024 * 1024 // 4
    x = [torch.rand(count, device="cuda", generator=gen) * 2 - 1 for _ in range(n)]
    y = [torch.empty_like(t) for t in x]
    st = torch.cuda.current_stream().cuda_stream
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    k = args.kernel
    if k.startswith("stepped_"):
        call = _prepared(cc, "cc_allreduce_stepped", cc._ptrs(x), cc._ptrs(y), n, count, cc.CC_F32, cc.CC_F32,
                         cc.CC_SUM, cc.CC_ALGO_RING if k.endswith("ring") else cc.CC_ALGO_TREE, 1.0,
                         ws.data_ptr(), ws.numel() * 4, st)
    elif k.startswith("multiring"):
        call = _prepared(cc, "cc_allreduce_multiring", cc._ptrs(x), cc._ptrs(y), n, int(k[len("multiring"):] or 2),
                         count, cc.CC_F32, cc.CC_F32, cc.CC_SUM, 1.0, st)
    elif k == "reduce":
        call = _prepared(cc, "cc_reduce", cc._ptrs(x), y[0].data_ptr(), n, 0, count, cc.CC_F32, cc.CC_F32, cc.CC_SUM,
                         1.0, st)
    elif k == "rs":
        shards = [torch.empty(cc.cc_chunk(count, n, c)[1], device="cuda") for c in range(n)]
        call = _prepared(cc, "cc_reduce_scatter", cc._ptrs(x), cc._ptrs(shards), n, count, cc.CC_F32, cc.CC_F32,
                         cc.CC_SUM, cc.CC_ALGO_RING, 1.0, st)
    elif k == "ag":
        shards = [x[c][:cc.cc_chunk(count, n, c)[1]] for c in range(n)]
        call = _prepared(cc, "cc_allgather", cc._ptrs(shards), cc._ptrs(y), n, count, cc.CC_F32, st)
    elif k in ("ring", "tree"):
        call = _prepared(cc, "cc_allreduce", cc._ptrs(x), cc._ptrs(y), n, count, cc.CC_F32, cc.CC_F32, cc.CC_SUM,
                         cc.CC_ALGO_RING if k == "ring" else cc.CC_ALGO_TREE, 1.0, st)
    else:
        raise SystemExit(f"unknown --kernel {k}")
    for _ in range(args.warmup):
        call()
    ms = _event_time_ms(torch, call, max(1, args.steps)) / max(1, args.steps)
    print(json.dumps({"kernel": k, "n": n, "mib_per_rank": args.mib, "ms_per_call": ms,
                      "allreduce_metric_GBps": 2 * n * count * 4 / (ms * 1e-3) / 1e9}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=12, help="model depth (12 = the workload; smaller for profiling)")
    ap.add_argument("--algo", default="ring", choices=["ring", "tree"],
                    help="ddp: the fold order of the headline step (ring, the default, or the double binary tree)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="headline only (configs 1, 3, 4, 5 left out)")
    ap.add_argument("--oracle-buckets", type=int, default=8)
    ap.add_argument("--kernel", default="ring", help="--workload kernel: stepped_ring, stepped_tree, "
                    "multiring<K>, reduce, rs, ag, ring, tree")
    ap.add_argument("--n", type=int, default=8, help="--workload kernel: simulated ranks")
    ap.add_argument("--mib", type=int, default=32, help="--workload kernel: MiB per rank")
    ap.add_argument("--workload", default="ddp", choices=["ddp", "zero", "moe", "sweep", "peer", "kernel"],
                    help="ddp = the headline step (plus every other config as rows at one GPU); zero, moe, sweep "
                         "= one config alone in detail; peer = the one-rank-per-GPU collective (the default at N > 1)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 or args.workload == "peer":
        return run_multi_gpu(args)
    if args.workload == "kernel":
        return run_kernel(args)
    if args.workload != "ddp":
        return run_rows(args)
    return run_headline(args)


def run_headline(args):
    """One GPU: the config-2 DDP step (N = 8 simulated ranks) as the headline, its end-to-end
    number through the host-buffer entry point, the oracle's CPU baseline, and configs 1, 3,
    4 and 5 as rows of the same line, each with its own clock record."""
    import torch
    import collective_communication_primitives_rank_b200 as cc

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    w = build_workload(torch, args.layers, SEED, pinned_inputs=True)
    bytes_step = 2 * N_SIM * w["total"] * 4
    stream = torch.cuda.current_stream()
    # scale: the library's mean; algo: the ring (the headline) unless --algo tree
    plan = cc.BucketAllreducePlan(w["dev_in"], w["dev_out"], cap_bytes=CAP, algo=args.algo)
    cuda_stream = stream.cuda_stream

    def step():
        plan.run(cuda_stream)

    launches_per_step = -(-len(w["numels"]) // 192)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        while not end.query():  # wait without holding the GIL, so the clock sampler runs meanwhile
            time.sleep(0.0005)
        torch.cuda.synchronize()
    ms_step = start.elapsed_time(end) / args.steps
    value = aggregate_gbps(1, bytes_step, ms_step)

    # end to end through the host-buffer entry point: H2D + fused allreduce + D2H per step
    host_out = [torch.empty(w["total"], dtype=torch.float32, pin_memory=True) for _ in range(N_SIM)]
    h_in = [w["views"](h) for h in w["host"]]
    h_out = [w["views"](h) for h in host_out]
    host_plan = cc.BucketAllreduceHostPlan(h_in, h_out, w["dev_in"], w["dev_out"], cap_bytes=CAP, algo=args.algo)
    host_plan.run(cuda_stream)
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(args.e2e_steps):
        host_plan.run(cuda_stream)
    e2.record(stream)
    torch.cuda.synchronize()
    e2e_value = aggregate_gbps(1, bytes_step, s2.elapsed_time(e2) / args.e2e_steps)

    peak, peak_kind = measured_peak()
    achieved = bytes_step / launches_per_step / (ms_step / launches_per_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "pct_of_8TBps": 100.0 * value / NOMINAL_HBM_GBS,
        "elems_per_s": N_SIM * w["total"] / (ms_step * 1e-3),
        "config": {"workload": workload_desc(args.layers, args.algo), "sim_ranks": N_SIM, "tensors": len(w["numels"]),
                   "elems_per_rank": w["total"], "bytes_per_step": bytes_step, "buckets": 17 if args.layers == 12 else None,
                   "l2": "inputs (3.5 GB) larger than L2 (126 MB); no flush", "parallelism": "replicas x1"},
        "roofline": dict(roofline_fields(achieved, peak, peak_kind), bound="hbm",
                         traffic=profile_traffic(DDP_PROFILES[args.algo]) if args.layers == 12 else None,
                         kernel=f"bucket_allreduce_kernel<{args.algo}>"),
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": N_SIM * w["total"] * 4,
                "d2h_bytes_per_step": N_SIM * w["total"] * 4},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        dt, moved, elems = oracle_sample_seconds(w["numels"], [h.numpy() for h in w["host"]], 0, args.oracle_buckets)
        line["cpu_baseline"] = {"value": moved / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": f"first {args.oracle_buckets} of 17 buckets ({elems} fp32 per rank, "
                                          f"{N_SIM} ranks), {dt:.1f} s single-threaded"}
    if not args.no_rows:
        it = max(3, args.steps // 2)
        # the same step with the double binary tree's fold order (config 2, the other algorithm)
        tree_plan = cc.BucketAllreducePlan(w["dev_in"], w["dev_out"], cap_bytes=CAP, algo="tree")
        tree_row = timed_row(torch, lambda: tree_plan.run(cuda_stream), it, bytes_step, launches_per_step, local=local,
                             kernel="bucket_allreduce_kernel<tree> (compiled 8-rank double binary tree)")
        config2 = {"workload": workload_desc(args.layers, "tree"),
                   "l2": "inputs larger than L2; no flush", "rows": {"bucket_allreduce_tree": tree_row}}
        del w, plan, tree_plan, host_plan, host_out, h_in, h_out
        torch.cuda.empty_cache()
        gen = torch.Generator(device="cuda")
        gen.manual_seed(SEED)
        cpu = not args.no_cpu_baseline
        line["rows"] = {"config2": config2,
                        "config1": rows_config1(torch, cc, local, cpu),
                        "config3": rows_config3(torch, cc, gen, local, it, cpu),
                        "config4": rows_config4(torch, cc, gen, local, it, cpu),
                        "config5": rows_config5(torch, cc, gen, local, cpu)}
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
