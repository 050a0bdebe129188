"""Benchmark of the ReAttention top-k span attention step on B200.

One step = one pass of the whole hot path over one batch: span scoring of the
middle of the pre-RoPE cache, top-k span selection, and attention over the
RoPE'd window (reatt_step through the C ABI).  Default workload: the
LLaMA3-8B-shaped 128K-context bf16 decode (B=1, 32/8 heads, d=128, G=32,
L=4096, S=32, k=64).  Inputs are seeded synthetic caches resident in HBM;
L2 is flushed (a 512 MiB read) before every timed step and the flush is
outside each step's CUDA-event interval.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica
sequence(s) -- the path has no cross-sequence exchange -- and rank 0 prints
the aggregate over ranks with the max per-rank time ("scaling": "weak").
`--impl reference` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ReAttention step latency (µs) and KV-scan GB/s vs HBM peak at 128K–4M context"
# committed ncu summaries holding the dominant kernel's per-launch DRAM traffic
PROFILE_SUMMARY = {
    "llama3_8b_128k": os.path.join(ROOT, "profiles", "scan_decode_llama3_8b_128k.md"),
    "llama3_8b_prefill_256k": os.path.join(ROOT, "profiles",
                                           "scan_prefill_tc_llama3_8b_prefill_256k.md"),
}


def step_bytes(w):
    """Algorithmic bytes one step must move: the middle keys once, the
    window's K/V rows once, q, the current K/V and the fp32 output."""
    e = w.elem_bytes
    M = max(0, w.T - w.G - w.L)
    scan = w.B * w.Hkv * M * w.d * e
    win_cached = min(w.G, w.T) + min(w.k * w.S, M) + (w.T - max(w.G, w.T - w.L) if w.T > w.G else 0)
    window = w.B * w.Hkv * win_cached * w.d * e * 2
    io = w.B * w.Hq * w.C * w.d * (e + 4) + w.B * w.Hkv * w.C * w.d * e * 2
    return scan, scan + window + io


def read_traffic(workload):
    """Per-launch DRAM traffic of the scan kernel from the committed ncu
    summary of this workload (a line 'traffic_bytes_per_launch: N', with the
    kernel build it was taken on); None if there is none."""
    path = PROFILE_SUMMARY.get(workload)
    if path is None:
        return None
    try:
        with open(path) as f:
            for line in f:
                if line.startswith("traffic_bytes_per_launch:"):
                    v = line.split(":", 1)[1].strip()
                    return None if v in ("null", "") else float(v)
    except OSError:
        pass
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) while
    the timed region runs."""

    def __init__(self, device, period_s=0.002):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:   # the same physical GPU as the CUDA device, whatever the visible-device map
                uuid = str(torch.cuda.get_device_properties(device).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reason_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _names(self, mask):
        nv = self.nv
        table = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        return {k for k, bit in table.items() if mask & bit}

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self._names(self._reason_fn(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def aggregate(world, step_b, steps, total_ms, e2e_ms, scan_ms, reduce_max=None):
    """Whole-job numbers: the slowest rank's times (max over ranks) and the
    bytes of every rank's replica over that time (weak scaling)."""
    if world > 1:
        total_ms, e2e_ms, scan_ms = reduce_max([total_ms, e2e_ms, scan_ms])
    return {"total_ms": total_ms, "e2e_ms": e2e_ms, "scan_ms": scan_ms,
            "value": world * step_b * steps / (total_ms * 1e-3) / 1e9,
            "e2e_value": world * step_b * steps / (e2e_ms * 1e-3) / 1e9}


def config_of(w, world):
    """The workload named by its sizes (both arms print the same dict)."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "C": w.C,
            "T": w.T, "G": w.G, "L": w.L, "S": w.S, "k": w.k, "rope_base": w.rope_base,
            "parallelism": f"replicas x{world}",
            "l2": "flushed before every step (512 MiB read); flush outside the step events"}


def dist_us(ms_list):
    """Median, p10 and p90 (µs) of a list of per-step times in ms."""
    v = sorted(ms_list)
    pick = lambda f: v[min(len(v) - 1, int(round(f * (len(v) - 1))))] * 1e3
    return {"median": round(pick(0.5), 2), "p10": round(pick(0.1), 2), "p90": round(pick(0.9), 2)}


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, kind): the measured copy bandwidth and
    cuBLAS bf16 throughput of this machine's B200s, else the earlier fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def scan_flops(w):
    """Algorithmic flops of the prefill scan in the summed-query form: one
    length-d dot product per (query position, middle token, KV head)."""
    M = max(0, w.T - w.G - w.L)
    return 2 * w.B * w.Hkv * w.C * M * w.d


def roofline(w, scan_b, scan_ms):
    """Roofline entry of the dominant kernel (the span scan): HBM-bound in
    decode, tensor-bound (tcgen05) for a bf16 prefill chunk."""
    hbm, tflops, kind = peaks()
    traffic = read_traffic(w.name)
    if w.C > 1 and w.dtype == "bf16" and 32 % w.S == 0:
        achieved = scan_flops(w) / (scan_ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": round(achieved, 1), "peak": tflops,
                "peak_kind": kind + " (bf16 burst)", "unit": "TFLOP/s",
                "frac": round(achieved / tflops, 4), "traffic": traffic,
                "kernel": "scan_prefill_tc_kernel", "flops_per_launch": scan_flops(w),
                "note": "issued MMA work is 2x (bf16 hi + lo query terms)"}
    achieved = scan_b / (scan_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "peak_kind": kind,
            "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic,
            "kernel": "scan_decode_kernel" if w.C == 1 else "scan_multi_kernel",
            "bytes_per_launch": scan_b}


def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from top_kv_span_b200 import reatt as R
    from top_kv_span_b200 import workloads as wl

    w = wl.WORKLOADS[args.workload]
    # weak scaling: rank r runs its own sequences (seed offset by rank)
    w = w.replace(seed=w.seed + 1000 * rank)
    x = wl.make_inputs(w, dev)
    d = R.dims_of(w)
    buf = R.alloc_outputs(d, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush.fill_(1)

    def do_flush():
        flush.sum(dtype=torch.int32)   # a full read: L2 ends up holding unrelated clean lines

    def step():
        R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], buf["sel"],
                     buf["out"], buf["ws"], stream)

    def scan_only():
        R.reatt_score_spans(d, x["q"], x["k_cache"], buf["span_scores"], buf["ws"], stream)

    # our kernels per step, counted once with the profiler (outside timing)
    from torch.profiler import ProfilerActivity, profile
    step()
    torch.cuda.synchronize(dev)
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        step()
        torch.cuda.synchronize(dev)
    per_step = sum(1 for e in prof.events()
                   if e.device_type.name == "CUDA" and "reatt" in e.name)

    for _ in range(args.warmup):
        do_flush()
        step()
    torch.cuda.synchronize(dev)
    assert R.reatt_workspace_status(buf["ws"], stream) == R.OK

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clk:
        for i in range(args.steps):
            do_flush()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)

    # dominant kernel (span scan) timed alone, same launch configuration
    for _ in range(3):
        do_flush()
        scan_only()
    sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        do_flush()
        sev[i][0].record(stream)
        scan_only()
        sev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    scan_list = [a.elapsed_time(b) for a, b in sev]
    scan_ms = statistics.mean(scan_list)

    # end to end through the C ABI with host buffers: per step the new
    # token's q / k / v go host->device from pinned memory and the output
    # comes back; the KV cache is device-resident state, as in decoding.  The
    # three inputs sit back to back in one pinned staging buffer (and one
    # device buffer), so a step needs one host->device copy.
    parts = [x["q"], x["k_cur"], x["v_cur"]]
    offs, off = [], 0
    for t in parts:
        offs.append(off)
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    hbuf = torch.empty(off, dtype=torch.uint8).pin_memory()
    dbuf = torch.empty(off, dtype=torch.uint8, device=dev)
    views = []
    for t, o in zip(parts, offs):
        n = t.numel() * t.element_size()
        hbuf[o:o + n].copy_(t.cpu().contiguous().view(torch.uint8).reshape(-1))
        views.append(dbuf[o:o + n].view(t.dtype).view(t.shape))
    x["q"], x["k_cur"], x["v_cur"] = views
    hout = torch.empty(buf["out"].shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in parts)
    d2h = hout.numel() * 4
    for _ in range(3):
        dbuf.copy_(hbuf, non_blocking=True)
        step()
    torch.cuda.synchronize(dev)
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        do_flush()
        eev[i][0].record(stream)
        dbuf.copy_(hbuf, non_blocking=True)
        step()
        hout.copy_(buf["out"], non_blocking=True)
        eev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(a.elapsed_time(b) for a, b in eev)

    def reduce_max(vals):
        t = torch.tensor(vals, dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return [float(v) for v in t.tolist()]

    scan_b, step_b = step_bytes(w)
    agg = aggregate(world, step_b, args.steps, total_ms, e2e_ms, scan_ms,
                    reduce_max if world > 1 else None)
    total_ms, e2e_ms, scan_ms = agg["total_ms"], agg["e2e_ms"], agg["scan_ms"]
    ms_per_step = total_ms / args.steps
    value, e2e_value = agg["value"], agg["e2e_value"]
    achieved = scan_b / (scan_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "step_us": round(ms_per_step * 1e3, 2),
        "scan_us": round(scan_ms * 1e3, 2),
        "scan_gbs": round(achieved, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded caches, per-channel sigma, planted needles)",
        "config": config_of(w, world),
        "roofline": roofline(w, scan_b, scan_ms),
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "us_per_step": round(e2e_ms / args.steps * 1e3, 2)},
        "gpu_launches": per_step * args.steps,
        "clocks": clk.summary(),
        # this rank's distribution over the timed steps (µs): median, p10, p90
        "step_dist_us": dist_us(step_ms),
        "scan_dist_us": dist_us(scan_list),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, x, seconds=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def oracle_sample(w, x, heads):
    """Host copies of the inputs restricted to the first `heads` KV heads of sequence 0."""
    from top_kv_span_b200 import workloads as wl
    g = w.Hq // w.Hkv
    sub = {"q": x["q"][:1, :heads * g], "k_cache": x["k_cache"][:1, :heads],
           "v_cache": x["v_cache"][:1, :heads], "k_cur": x["k_cur"][:1, :heads],
           "v_cur": x["v_cur"][:1, :heads]}
    return {n: wl.to_oracle(t) for n, t in sub.items()}, w.replace(B=1, Hkv=heads, Hq=heads * g)


def cpu_baseline(w, x, seconds=15.0, heads=None, single_seconds=5.0):
    """The oracle as it stands, on this host's cores, over a bounded sample of
    the workload (the first KV head(s) of sequence 0), repeated for ~seconds;
    then the same sample on one core for ~single_seconds."""
    import oracle
    heads = heads or 1
    xs, ws = oracle_sample(w, x, heads)
    _, sb = step_bytes(ws)

    def timed(limit):
        t0 = time.perf_counter()
        n = 0
        while True:
            oracle.step(**xs, G=ws.G, L=ws.L, S=ws.S, k=ws.k, rope_base=ws.rope_base,
                        want_scores=False)
            n += 1
            if time.perf_counter() - t0 > limit:
                break
        return (time.perf_counter() - t0) / n, n

    cores = oracle.max_threads()
    dt, n = timed(seconds)
    out = {"value": round(sb / dt / 1e9, 4), "unit": "GB/s", "cores": cores,
           "kind": "oracle", "sample": f"{w.name}: sequence 0, {heads} of {w.Hkv} KV heads "
                                       f"({heads * (w.Hq // w.Hkv)} query heads), {n} oracle steps",
           "sec_per_sample_step": round(dt, 4)}
    if single_seconds > 0:
        oracle.set_threads(1)
        try:
            dt1, n1 = timed(single_seconds)
        finally:
            oracle.set_threads(cores)
        out["single_thread"] = {"value": round(sb / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                                "sec_per_sample_step": round(dt1, 4), "steps": n1}
    return out


def run_reference(args):
    """The oracle timed as the reference arm (host cores), same metric/config."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    from top_kv_span_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    x = wl.make_inputs(w.replace(B=1), "cpu") if w.T <= (1 << 18) else None
    if x is None:
        # long caches: draw only the sampled head on the host
        ws = w.replace(B=1, Hkv=1, Hq=w.Hq // w.Hkv)
        x = wl.make_inputs(ws, "cpu")
        w_used, heads_total = ws, w.Hkv
    else:
        w_used, heads_total = w, w.Hkv
    import oracle
    xs, wsamp = oracle_sample(w_used, x, 1)
    _, sb = step_bytes(wsamp)
    for _ in range(args.warmup):
        oracle.step(**xs, G=wsamp.G, L=wsamp.L, S=wsamp.S, k=wsamp.k, rope_base=wsamp.rope_base,
                    want_scores=False)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.step(**xs, G=wsamp.G, L=wsamp.L, S=wsamp.S, k=wsamp.k, rope_base=wsamp.rope_base,
                    want_scores=False)
    dt = (time.perf_counter() - t0) / args.steps
    value = sb / dt / 1e9
    sample = f"{w.name}: sequence 0, 1 of {heads_total} KV heads per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, 1),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)
    del torch


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama3_8b_128k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
