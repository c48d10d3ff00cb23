"""Benchmark: the fused DDP gradient-bucket allreduce of libcc on B200.

Workload (one step): N = 8 simulated ranks, each holding the fp32 gradients of a 12-layer
d = 768 transformer (147 tensors, 109,632,000 elements = 438.5 MB per rank, values
normal(0, 1e-3)), packed into 25 MiB buckets (17) in reverse registration order, ring
allreduce of every bucket with the 1/N scale, unflattened: one fused kernel launch
(cc_bucket_allreduce), inputs and outputs resident in HBM.

Metric: allreduce effective HBM GB/s = (N·T in + N·T out) / step time, T = 438.5 MB,
plus its share of ~8 TB/s and elements/s (N·count / step time).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--gpus N > 1 runs under torchrun, one process per GPU, each with its own replica of the
workload (independent problems: weak scaling); time is the max over ranks.
--impl reference times the oracle (the plain CPU message-passing simulator) on a bounded
sample of the same workload.
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


def workload_desc(layers):
    return (f"ddp_bucket_allreduce: N={N_SIM} simulated ranks on one GPU, fp32 gradients of a "
            f"{layers}-layer d=768 ffn=3072 vocab=32000 transformer, 25 MiB buckets in reverse "
            f"registration order, ring allreduce with scale 1/{N_SIM}, fused flatten/unflatten")


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def profile_traffic(name="bucket_allreduce_ddp.txt"):
    """DRAM bytes per launch of a line's dominant kernel from a committed ncu summary in
    profiles/, or None when the kernel's source file changed since the counters were taken
    (the summary records the file and its SHA-256)."""
    try:
        text = open(os.path.join(ROOT, "profiles", name)).read()
        lines = dict(l.split(":", 1) for l in text.splitlines() if ":" in l and not l.startswith(" "))
        src = os.path.join(ROOT, lines.get("kernel_source", os.path.relpath(KERNEL_SRC, ROOT)).strip())
        if lines.get("kernel_source_sha256", "").strip() != hashlib.sha256(open(src, "rb").read()).hexdigest():
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


# ---- the other hot-path rows (one JSON line each; not the headline) --------------------------------

def _event_time_ms(torch, fn, iters, flush=None):
    """Sum of per-iteration CUDA-event times of fn(); `flush` (outside the timed spans)
    evicts L2 between iterations when the working set would fit in it."""
    total = 0.0
    stream = torch.cuda.current_stream()
    for _ in range(iters):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    return total


def _prepared_allreduce(cc, x, y, algo, stream):
    """cc_allreduce with its arguments marshalled once, so that a timed span holds only the
    C call (the binding's per-call checks would otherwise sit between the events)."""
    fn = cc.get_lib().cc_allreduce
    a = (cc._ptrs(x), cc._ptrs(y), len(x), x[0].numel(), cc.CC_F32, cc.CC_F32, cc.CC_SUM,
         cc.CC_ALGO_RING if algo == "ring" else cc.CC_ALGO_TREE, 1.0, stream)

    def call():
        if fn(*a) != cc.CC_OK:
            raise RuntimeError("cc_allreduce failed")
    return call


def _prepared(cc, name, *args):
    """A C entry point with its arguments marshalled once (timed spans hold only the call)."""
    fn = getattr(cc.get_lib(), name)

    def call():
        st = fn(*args)
        if st != cc.CC_OK:
            raise RuntimeError(f"{name}: status {st}")
    return call


def _row_line(args, metric, value, unit, ms, config, roofline, launches, extra=None):
    peak, kind = measured_peak()
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": config.pop("dtype", "f32"), "data": "synthetic", "config": config,
            "roofline": dict(roofline, peak=peak, peak_kind=kind, unit="GB/s",
                             frac=roofline["achieved"] / peak, bound="hbm", traffic=roofline.get("traffic")),
            "gpu_launches": launches}
    if extra:
        line.update(extra)
    print(json.dumps(line))


def run_peer(args):
    """One rank per GPU (torchrun): a 256 MiB fp32 allreduce per rank through libcc's slice
    calls over CUDA IPC peer mappings (each rank folds its own chunk from every GPU and writes
    it to every GPU, ordered by host barriers), timed beside NCCL's all_reduce of the same
    buffer. Bus bandwidth = 2(N-1)/N * T / t per GPU (every byte of a rank's chunk leaves it
    once each way). Parity of the slice path is covered by the GPU tests."""
    import datetime
    import torch
    import torch.distributed as dist
    import collective_communication_primitives_rank_b200 as cc
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29531")
    os.environ.setdefault("RANK", str(rank))
    os.environ.setdefault("WORLD_SIZE", str(world))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    count = 64 * 1024 * 1024
    T = count * 4
    gen = torch.Generator(device="cuda")
    gen.manual_seed(replica_seed(rank))
    send = torch.randn(count, device="cuda", generator=gen)
    recv = torch.empty_like(send)
    stream = torch.cuda.current_stream()
    ar = cc.PeerAllreduce(send, recv, scale=1.0 / world)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        return max_over_ranks(dist, torch, a.elapsed_time(b) / args.steps, "cuda")

    with Clocks(local) as clocks:
        ms = timed(ar.run)
    x = send.clone()
    ms_nccl = timed(lambda: dist.all_reduce(x))
    ar.close()
    dist.barrier()
    factor = 2.0 * (world - 1) / world
    bus, bus_nccl = factor * T / (ms * 1e-3) / 1e9, factor * T / (ms_nccl * 1e-3) / 1e9
    if rank == 0:
        peak = 770.0  # measured peer copy per direction per GPU on this machine's NVLink 5
        print(json.dumps({
            "metric": "allreduce bus bandwidth per GPU, 2(N-1)/N * T / t (one rank per GPU over NVLink)",
            "value": bus, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "peer: 256 MiB fp32 per rank, one rank per GPU, ring-order one-shot allreduce "
                                   "(scale 1/N) through cc_allreduce_slice over CUDA IPC, host barriers included; "
                                   "NCCL all_reduce (sum) of the same buffer as the comparator",
                       "bytes_per_rank": T, "parallelism": f"ranks x{world}"},
            "algbw": T / (ms * 1e-3) / 1e9,
            "nccl": {"ms_per_step": ms_nccl, "busbw": bus_nccl, "algbw": T / (ms_nccl * 1e-3) / 1e9},
            "roofline": {"bound": "nvlink", "achieved": bus, "peak": peak, "unit": "GB/s",
                         "frac": bus / peak, "peak_kind": "measured peer copy (per direction)", "traffic": None,
                         "note": "no NVLink traffic at one GPU" if world == 1 else ""},
            "gpu_launches": args.steps, "clocks": clocks.summary()}))
    dist.destroy_process_group()
    return 0


def run_rows(args):
    import torch
    import collective_communication_primitives_rank_b200 as cc
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(SEED)
    iters = max(1, args.steps)
    if args.workload == "zero":
        # config 3: N = 8, 300M fp32 per rank normal(0, 1e-2): reduce-scatter to 1/8 shards, then
        # allgather of the shards; plus the bf16-input reduce-scatter with fp32 accumulation
        n, count = N_SIM, 300_000_000
        x = [torch.randn(count, device="cuda", generator=gen) * 1e-2 for _ in range(n)]
        shard = count // n
        rs = [torch.empty(shard, device="cuda") for _ in range(n)]
        ag = [torch.empty(count, device="cuda") for _ in range(n)]
        st = torch.cuda.current_stream().cuda_stream
        rs_call = _prepared(cc, "cc_reduce_scatter", cc._ptrs(x), cc._ptrs(rs), n, count, cc.CC_F32, cc.CC_F32,
                            cc.CC_SUM, cc.CC_ALGO_RING, 1.0, st)
        ag_call = _prepared(cc, "cc_allgather", cc._ptrs(rs), cc._ptrs(ag), n, count, cc.CC_F32, st)
        for _ in range(args.warmup):
            rs_call()
            ag_call()
        t_rs = _event_time_ms(torch, rs_call, iters) / iters
        t_ag = _event_time_ms(torch, ag_call, iters) / iters
        del ag, ag_call
        xb = [t.to(torch.bfloat16) for t in x]
        del x, rs_call
        bf_call = _prepared(cc, "cc_reduce_scatter", cc._ptrs(xb), cc._ptrs(rs), n, count, cc.CC_BF16, cc.CC_F32,
                            cc.CC_SUM, cc.CC_ALGO_RING, 1.0, st)
        for _ in range(args.warmup):
            bf_call()
        t_bf = _event_time_ms(torch, bf_call, iters) / iters
        T = count * 4
        ms = t_rs + t_ag
        value = 2 * n * T / (ms * 1e-3) / 1e9
        _row_line(args, METRIC, value, "GB/s", ms,
                  {"workload": "zero: N=8 simulated ranks, 300M fp32 per rank normal(0,1e-2), ring reduce-scatter "
                               "to 37.5M-element shards, then allgather of the shards (device-seeded inputs)",
                   "l2": "inputs larger than L2; no flush"},
                  {"achieved": (n + 1) * T / (t_rs * 1e-3) / 1e9, "kernel": "reduce_kernel<f32,sum,ring> (RS)",
                   "traffic": profile_traffic("reduce_scatter_allgather_zero.txt")},
                  2 * iters,
                  {"rows": {"reduce_scatter_f32": {"ms": t_rs, "bytes": (n + 1) * T, "GBps": (n + 1) * T / t_rs / 1e6},
                            "allgather_f32": {"ms": t_ag, "bytes": (n + 1) * T, "GBps": (n + 1) * T / t_ag / 1e6},
                            "reduce_scatter_bf16_in_f32_out": {"ms": t_bf, "bytes": n * T // 2 + T,
                                                               "GBps": (n * T // 2 + T) / t_bf / 1e6}}})
        return 0
    if args.workload == "moe":
        # config 4: N = 8, 8192 tokens x 4096 bf16 per rank, 64 experts (8 per rank), top-2
        n, tokens, hidden, epr, topk = N_SIM, 8192, 4096, 8, 2
        E = n * epr
        logits = [torch.randn(tokens, E, device="cuda", generator=gen) for _ in range(n)]
        toks = [torch.randn(tokens, hidden, device="cuda", generator=gen).to(torch.bfloat16) for _ in range(n)]
        ids = [torch.empty(tokens, topk, dtype=torch.int32, device="cuda") for _ in range(n)]
        cc.cc_route_topk(logits, ids)
        ws = torch.empty(cc.cc_alltoallv_workspace_size(n, tokens, topk, epr) // 4 + 64, dtype=torch.int32,
                         device="cuda")
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
        for _ in range(args.warmup):
            route()
            disp()
            comb()
        t_route = _event_time_ms(torch, route, iters) / iters
        t_d = _event_time_ms(torch, disp, iters) / iters
        t_c = _event_time_ms(torch, comb, iters) / iters
        b_d = n * tokens * row + rows_recv * row
        b_c = 2 * rows_recv * row
        ms = t_route + t_d + t_c
        _row_line(args, "alltoallv effective HBM GB/s (dispatch: tokens read once + routed rows written; "
                        "combine: routed rows read + written)", (b_d + b_c) / (ms * 1e-3) / 1e9, "GB/s", ms,
                  {"workload": "moe: N=8 simulated ranks, 8192 tokens x 4096 bf16 per rank, 64 experts (8 per rank), "
                               "top-2 routing from normal logits, dispatch then combine (device-seeded inputs)",
                   "dtype": "bf16 (bit copy)", "l2": "inputs larger than L2; no flush"},
                  {"achieved": b_d / (t_d * 1e-3) / 1e9, "kernel": "a2a dispatch (count + scan + base + copy)",
                   "traffic": profile_traffic("alltoallv_dispatch_moe.txt")},
                  iters * (1 + 4 + 4),
                  {"rows": {"route_topk": {"ms": t_route},
                            "dispatch": {"ms": t_d, "bytes": b_d, "GBps": b_d / t_d / 1e6},
                            "combine": {"ms": t_c, "bytes": b_c, "GBps": b_c / t_c / 1e6}}})
        return 0
    # config 5: ring vs double-binary-tree allreduce, N in {2..64}, 1 KiB .. 256 MiB per rank
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    table = []
    best = None
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
                call = _prepared_allreduce(cc, x, y, algo, torch.cuda.current_stream().cuda_stream)
                for _ in range(3):
                    call()
                ms = _event_time_ms(torch, call, reps, flush) / reps
                row[algo + "_us"] = ms * 1e3
                row[algo + "_GBps"] = 2 * n * size / (ms * 1e-3) / 1e9
                # the same result by the schedule's dependent steps (grid barrier per step)
                stepped = _prepared(cc, "cc_allreduce_stepped", cc._ptrs(x), cc._ptrs(y), n, count, cc.CC_F32,
                                    cc.CC_F32, cc.CC_SUM, cc.CC_ALGO_RING if algo == "ring" else cc.CC_ALGO_TREE,
                                    1.0, ws.data_ptr(), ws.numel() * 4, torch.cuda.current_stream().cuda_stream)
                for _ in range(2):
                    stepped()
                sreps = max(2, reps // 4)
                ms = _event_time_ms(torch, stepped, sreps, flush) / sreps
                row[algo + "_stepped_us"] = ms * 1e3
                row[algo + "_stepped_GBps"] = 2 * n * size / (ms * 1e-3) / 1e9
            if n == 8:
                bc = _prepared(cc, "cc_broadcast", x[0].data_ptr(), cc._ptrs(y), n, 0, count, cc.CC_F32,
                               torch.cuda.current_stream().cuda_stream)
                ms = _event_time_ms(torch, bc, reps, flush) / reps
                row["broadcast_GBps"] = (n + 1) * size / (ms * 1e-3) / 1e9
            table.append(row)
            if n == 8 and size == 256 * 1024 * 1024:
                best = row
            del x, y
    # hierarchical allreduce (8 ranks per node) at the large sizes
    hier = []
    for n, mib in ((16, 256), (64, 64)):
        count = mib * 1024 * 1024 // 4
        x = [torch.rand(count, device="cuda", generator=gen) * 2 - 1 for _ in range(n)]
        y = [torch.empty_like(t) for t in x]
        call = _prepared(cc, "cc_allreduce_hierarchical", cc._ptrs(x), cc._ptrs(y), n, 8, count, cc.CC_F32,
                         cc.CC_F32, cc.CC_SUM, 1.0, torch.cuda.current_stream().cuda_stream)
        for _ in range(3):
            call()
        ms = _event_time_ms(torch, call, 5) / 5
        hier.append({"n": n, "ranks_per_node": 8, "bytes_per_rank": count * 4, "us": ms * 1e3,
                     "GBps": 2 * n * count * 4 / (ms * 1e-3) / 1e9})
        del x, y
    cross, cross_stepped = {}, {}
    for n in (2, 4, 8, 16, 32, 64):
        pts = [r for r in table if r["n"] == n]
        for key, dst in (("", cross), ("_stepped", cross_stepped)):
            over = [r["bytes_per_rank"] for r in pts if r["ring" + key + "_GBps"] > 1.03 * r["tree" + key + "_GBps"]]
            under = [r["bytes_per_rank"] for r in pts if r["tree" + key + "_GBps"] > 1.03 * r["ring" + key + "_GBps"]]
            dst[str(n)] = {"ring_faster_by_3pct_at": over, "tree_faster_by_3pct_at": under}
    lat = min(r["ring_us"] for r in table)
    _row_line(args, METRIC, best["ring_GBps"], "GB/s", best["ring_us"] / 1e3,
              {"workload": "sweep: ring vs double-binary-tree allreduce, N in {2,4,8,16,32,64}, fp32 U[-1,1] "
                           "1 KiB..256 MiB per rank (powers of 4); headline value = N=8, 256 MiB, ring",
               "l2": "L2 flushed (256 MiB write) before every timed call whose working set fits in L2"},
              {"achieved": best["ring_GBps"], "kernel": "reduce_kernel<f32,sum,ring>"},
              len(table) * 2,
              {"sweep": table, "crossover": cross, "crossover_stepped": cross_stepped, "hierarchical": hier,
               "min_launch_latency_us": lat})
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=12, help="model depth (12 = the workload; smaller for profiling)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-buckets", type=int, default=8)
    ap.add_argument("--workload", default="ddp", choices=["ddp", "zero", "moe", "sweep", "peer"],
                    help="ddp = the headline step; zero, moe, sweep measure the remaining hot-path rows; "
                         "peer = one rank per GPU over NVLink against NCCL (run under torchrun)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "peer":
        return run_peer(args)
    if args.workload != "ddp":
        return run_rows(args)

    import torch
    import torch.distributed as dist
    import collective_communication_primitives_rank_b200 as cc

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    w = build_workload(torch, args.layers, replica_seed(rank), pinned_inputs=True)
    bytes_step = 2 * N_SIM * w["total"] * 4
    stream = torch.cuda.current_stream()

    plan = cc.BucketAllreducePlan(w["dev_in"], w["dev_out"], cap_bytes=CAP, scale=1.0 / N_SIM)
    cuda_stream = stream.cuda_stream

    def step():
        plan.run(cuda_stream)

    launches_per_step = -(-len(w["numels"]) // 192)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step()
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        barrier()
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        barrier()
    ms = start.elapsed_time(end)
    if world > 1:
        ms = max_over_ranks(dist, torch, ms, "cuda")
    ms_step = ms / args.steps
    value = aggregate_gbps(world, bytes_step, ms_step)

    # end to end through the host-buffer entry point: H2D + fused allreduce + D2H per step
    host_out = [torch.empty(w["total"], dtype=torch.float32, pin_memory=True) for _ in range(N_SIM)]
    h_in = [w["views"](h) for h in w["host"]]
    h_out = [w["views"](h) for h in host_out]

    host_plan = cc.BucketAllreduceHostPlan(h_in, h_out, w["dev_in"], w["dev_out"], cap_bytes=CAP, scale=1.0 / N_SIM)

    def e2e_step():
        host_plan.run(cuda_stream)

    e2e_step()
    barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e2.record(stream)
    barrier()
    ems = s2.elapsed_time(e2)
    if world > 1:
        ems = max_over_ranks(dist, torch, ems, "cuda")
    e2e_value = aggregate_gbps(world, bytes_step, ems / args.e2e_steps)

    peak, peak_kind = measured_peak()
    achieved = bytes_step / launches_per_step / (ms_step / launches_per_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "pct_of_8TBps": 100.0 * value / world / NOMINAL_HBM_GBS,
        "elems_per_s": world * N_SIM * w["total"] / (ms_step * 1e-3),
        "config": {"workload": workload_desc(args.layers), "sim_ranks": N_SIM, "tensors": len(w["numels"]),
                   "elems_per_rank": w["total"], "bytes_per_step": bytes_step, "buckets": 17 if args.layers == 12 else None,
                   "l2": "inputs (3.5 GB) larger than L2 (126 MB); no flush", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": profile_traffic() if args.layers == 12 else None,
                     "kernel": "bucket_allreduce_kernel<ring>"},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": N_SIM * w["total"] * 4,
                "d2h_bytes_per_step": N_SIM * w["total"] * 4},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, moved, elems = oracle_sample_seconds(w["numels"], [h.numpy() for h in w["host"]], 0,
                                                 args.oracle_buckets)
        line["cpu_baseline"] = {"value": moved / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": f"first {args.oracle_buckets} of 17 buckets ({elems} fp32 per rank, "
                                          f"{N_SIM} ranks), {dt:.1f} s single-threaded"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
