"""Benchmark of the ReAttention top-k span attention step on B200.

One step = one pass of the whole hot path over one batch: span scoring of the
middle of the pre-RoPE cache, top-k span selection, and attention over the
RoPE'd window (reatt_step through the C ABI).  Headline workload: the
LLaMA3-8B-shaped 128K-context bf16 decode (B=1, 32/8 heads, d=128, G=32,
L=4096, S=32, k=64).  Inputs are seeded synthetic caches resident in HBM;
L2 is flushed (a 512 MiB read) before every timed step and the flush is
outside each step's CUDA-event interval.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference] [--extra NAMES] [--loops NAMES]
                  [--prefill-loop NAME]

At N=1 the same line also carries `per_workload` (the other workloads: the
tiny fp32 decode, the 1M x 4 and 4M decodes, the 2048-query prefill chunk),
each with its own timings, roofline and a parity sample, and `decode_loop`
(a graph-replayed decoding loop with its appends) and `prefill_loop` (a
128K-token prompt prefilled in the pages' chunks, each appended).  Parity comes from the
CPU leg, which runs the oracle on a bounded sample (KV head 0 of sequence 0)
and compares the GPU's selection (swap count) and outputs (max-abs) on it.

Multi-GPU: `--gpus N` starts N ranks of this script under
torch.distributed.run (one process per GPU) unless a launcher already did;
every rank runs its own replica sequence(s) -- the path has no
cross-sequence exchange -- and rank 0 prints the aggregate over ranks with
the max per-rank time ("scaling": "weak").  `--impl reference` times the CPU
oracle on the host cores instead.
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
                                           "scan_prefill_tcq_llama3_8b_prefill_64k.md"),
    "qwen2_1p5b_4m": os.path.join(ROOT, "profiles", "scan_decode_qwen2_1p5b_4m.md"),
    "llama3_8b_1m_x4": os.path.join(ROOT, "profiles", "scan_decode_llama3_8b_1m.md"),
    "tiny_f32_4k": os.path.join(ROOT, "profiles", "scan_decode_tiny_f32_4k.md"),
}
# key of the traffic line in a summary (a smaller capture scaled to the workload)
PROFILE_KEY = {"llama3_8b_prefill_256k": "traffic_bytes_per_launch_256k:",
               "llama3_8b_1m_x4": "traffic_bytes_per_launch_1m_x4:"}


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
    key = PROFILE_KEY.get(workload, "traffic_bytes_per_launch:")
    try:
        with open(path) as f:
            for line in f:
                if line.startswith(key):
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
                "kernel": "scan_prefill_tcq_kernel" if w.S == 32 else "scan_prefill_tc_kernel",
                "flops_per_launch": scan_flops(w),
                "note": "issued MMA work is 2x (bf16 hi + lo query terms)"}
    achieved = scan_b / (scan_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "peak_kind": kind,
            "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic,
            "kernel": "scan_decode_kernel" if w.C == 1 else "scan_multi_kernel",
            "bytes_per_launch": scan_b}


def dist_setup(cpu=False):
    """Rank, world and local rank from the launcher's environment; a process
    group over NCCL (one GPU per rank) or, for the CPU launch check, gloo."""
    import datetime

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        if cpu:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        else:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
    return world, rank, local


def host_cores():
    """Cores this process may run on (a launcher may have set OMP_NUM_THREADS=1)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def relaunch(n, argv):
    """`--gpus N` without a launcher around us: start N ranks of this script
    under torch.distributed.run (one process per GPU, rendezvous on
    127.0.0.1) and return the launcher's exit code."""
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def make_reduce_max(world, dev=None):
    import torch
    import torch.distributed as dist

    def reduce_max(vals):
        t = torch.tensor(vals, dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return [float(v) for v in t.tolist()]
    return reduce_max if world > 1 else None


def run_launch_check(args):
    """The multi-rank plumbing without a GPU (gloo): every rank reports its
    own replica times, rank 0 prints the job line (max time over ranks,
    bytes of every rank)."""
    import torch.distributed as dist
    world, rank, _ = dist_setup(cpu=True)
    total, e2e, scan = 10.0 + rank, 12.0 + 3 * rank, 5.0 - 0.5 * rank
    agg = aggregate(world, 1_000_000, args.steps, total, e2e, scan, make_reduce_max(world))
    if rank == 0:
        print(json.dumps({"launch_check": True, "n_gpus": world, "steps": args.steps,
                          "total_ms": agg["total_ms"], "e2e_ms": agg["e2e_ms"],
                          "scan_ms": agg["scan_ms"], "value": agg["value"]}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


class Timer:
    """Per-step device times with CUDA events on the launching stream, L2
    flushed (a 512 MiB read) before each step outside the events."""

    def __init__(self, dev, stream):
        import torch
        self.torch, self.dev, self.stream = torch, dev, stream
        self.flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.flush_buf.fill_(1)

    def flush(self):
        self.flush_buf.sum(dtype=self.torch.int32)   # a full read: L2 ends up holding unrelated lines

    def run(self, fn, steps, warmup=0, flush=True):
        torch = self.torch
        for _ in range(warmup):
            if flush:
                self.flush()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            if flush:
                self.flush()
            ev[i][0].record(self.stream)
            fn(i)
            ev[i][1].record(self.stream)
        torch.cuda.synchronize(self.dev)
        return [a.elapsed_time(b) for a, b in ev]


def launches_per_step(step):
    """Our kernels in one step, counted once with the profiler (outside timing)."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    step()
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        step()
        torch.cuda.synchronize()
    return sum(1 for e in prof.events() if e.device_type.name == "CUDA" and "reatt" in e.name)


def measure(w, args, dev, timer, world=1, rank=0, cpu_leg_seconds=0.0, single_seconds=0.0):
    """One workload: step, scan alone and end-to-end timings, roofline of the
    scan, and (rank 0) the CPU leg: the oracle on a bounded sample, which
    also yields the parity of that sample (selection swaps, max-abs)."""
    import torch
    from top_kv_span_b200 import reatt as R
    from top_kv_span_b200 import workloads as wl

    x = wl.make_inputs(w, dev)
    d = R.dims_of(w)
    buf = R.alloc_outputs(d, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i=0):
        R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], buf["sel"],
                     buf["out"], buf["ws"], stream)

    def scan_only(i=0):
        R.reatt_score_spans(d, x["q"], x["k_cache"], buf["span_scores"], buf["ws"], stream)

    per_step = launches_per_step(step)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clk:
        step_ms = timer.run(step, args.steps, warmup=args.warmup)
    if world > 1:
        dist.barrier()
    assert R.reatt_workspace_status(buf["ws"], stream) == R.OK
    gpu_sel = buf["sel"].cpu().numpy()
    gpu_out = buf["out"].cpu().numpy()
    scan_list = timer.run(scan_only, args.steps, warmup=3)

    # end to end through the C ABI with host buffers: per step the new
    # tokens' q / k / v go host->device from pinned memory and the output
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
    host_x = {n: x[n] for n in ("q", "k_cur", "v_cur")}
    x["q"], x["k_cur"], x["v_cur"] = views
    hout = torch.empty(buf["out"].shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in parts)
    d2h = hout.numel() * 4

    def e2e_step(i=0):
        dbuf.copy_(hbuf, non_blocking=True)
        step()
        hout.copy_(buf["out"], non_blocking=True)

    e2e_list = timer.run(e2e_step, args.steps, warmup=3)
    x.update(host_x)

    res = {"w": w, "x": x, "per_step": per_step, "clk": clk.summary(),
           "step_ms": step_ms, "scan_ms": scan_list, "e2e_ms": e2e_list,
           "h2d": h2d, "d2h": d2h}
    if rank == 0 and (cpu_leg_seconds >= 0):
        res["cpu"] = cpu_leg(w, x, gpu_sel, gpu_out, seconds=cpu_leg_seconds,
                             single_seconds=single_seconds)
    del buf
    return res


def summarise(res, world=1, steps=None, reduce_max=None):
    """JSON fields of one measured workload (times: max over ranks)."""
    w = res["w"]
    steps = steps or len(res["step_ms"])
    scan_b, step_b = step_bytes(w)
    agg = aggregate(world, step_b, steps, sum(res["step_ms"]), sum(res["e2e_ms"]),
                    statistics.mean(res["scan_ms"]), reduce_max)
    ms_per_step = agg["total_ms"] / steps
    out = {
        "value": round(agg["value"], 1),
        "unit": "GB/s",
        "ms_per_step": round(ms_per_step, 5),
        "step_us": round(ms_per_step * 1e3, 2),
        "scan_us": round(agg["scan_ms"] * 1e3, 2),
        "scan_gbs": round(scan_b / (agg["scan_ms"] * 1e-3) / 1e9, 1),
        "dtype": w.dtype,
        "config": config_of(w, world),
        "roofline": roofline(w, scan_b, agg["scan_ms"]),
        "step_roofline": step_roofline(w, ms_per_step),
        "e2e": {"value": round(agg["e2e_value"], 1), "unit": "GB/s",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                "us_per_step": round(agg["e2e_ms"] / steps * 1e3, 2)},
        "gpu_launches": res["per_step"] * steps,
        "clocks": res["clk"],
        # this rank's distribution over the timed steps (µs): median, p10, p90
        "step_dist_us": dist_us(res["step_ms"]),
        "scan_dist_us": dist_us(res["scan_ms"]),
    }
    if "cpu" in res:
        cpu = dict(res["cpu"])
        out["parity"] = cpu.pop("parity")
        if cpu.get("value") is not None:
            out["cpu_baseline"] = cpu
    return out


def step_roofline(w, ms_per_step):
    """The whole step against its bytes-over-HBM time (decode) or its
    flops-over-tensor time (bf16 prefill chunk)."""
    hbm, tflops, kind = peaks()
    _, step_b = step_bytes(w)
    if w.C > 1 and w.dtype == "bf16" and 32 % w.S == 0:
        fl = scan_flops(w) + attn_flops(w)
        t = fl / (tflops * 1e12)
        return {"bound": "tensor", "flops": fl, "roofline_us": round(t * 1e6, 2),
                "frac": round(t / (ms_per_step * 1e-3), 4), "peak_kind": kind}
    t = step_b / (hbm * 1e9)
    return {"bound": "hbm", "bytes": step_b, "roofline_us": round(t * 1e6, 2),
            "frac": round(t / (ms_per_step * 1e-3), 4), "peak_kind": kind}


def attn_flops(w):
    """Algorithmic flops of the window attention of a chunk: q.k and p.v over
    the causal window, 4*d per (query row, visible key)."""
    win_cached = min(w.G, w.T) + min(w.k * w.S, max(0, w.T - w.G - w.L)) + \
        (w.T - max(w.G, w.T - w.L) if w.T > w.G else 0)
    visible = w.C * win_cached + w.C * (w.C + 1) // 2
    return 4 * w.B * w.Hq * visible * w.d


def decode_loop(w, dev, timer, n_steps=16, reps=10):
    """NEXT step of a decoding loop, as a caller runs it: n_steps decode
    steps, each followed by the append of its token's K/V, captured once in
    a CUDA graph on caches with room to grow (T_cap = T + n_steps) and
    replayed.  Returns µs per step for the replayed graph and for the same
    loop launched eagerly (L2 flushed before each loop, not between its
    steps)."""
    import torch
    from top_kv_span_b200 import reatt as R
    from top_kv_span_b200 import workloads as wl

    x = wl.make_inputs(w, dev)
    cap = w.T + n_steps
    shape = (w.B, w.Hkv, cap, w.d)
    kc = torch.zeros(shape, dtype=w.torch_dtype, device=dev)
    vc = torch.zeros(shape, dtype=w.torch_dtype, device=dev)
    kc[:, :, :w.T] = x["k_cache"]
    vc[:, :, :w.T] = x["v_cache"]
    del x
    gen = torch.Generator(device=dev).manual_seed(w.seed + 77)
    rnd = lambda shp: torch.randn(shp, generator=gen, device=dev).to(w.torch_dtype)
    qs = [rnd((w.B, w.Hq, 1, w.d)) for _ in range(n_steps)]
    kn = [rnd((w.B, w.Hkv, 1, w.d)) for _ in range(n_steps)]
    vn = [rnd((w.B, w.Hkv, 1, w.d)) for _ in range(n_steps)]
    dims = [R.dims_of(w, T=w.T + i, T_cap=cap) for i in range(n_steps)]
    ws = torch.zeros(max(R.reatt_workspace_bytes(dd) for dd in dims), dtype=torch.uint8,
                     device=dev)
    outs = [torch.empty((w.B, w.Hq, 1, w.d), dtype=torch.float32, device=dev)
            for _ in range(n_steps)]
    sels = [torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device=dev)
            for _ in range(n_steps)]
    st = torch.cuda.Stream(dev)

    def loop(stream):
        for i in range(n_steps):
            R.reatt_step(dims[i], qs[i], kc, vc, kn[i], vn[i], sels[i], outs[i], ws,
                         stream=stream)
            R.reatt_append_kv(dims[i], kc, vc, kn[i], vn[i], stream=stream)

    with torch.cuda.stream(st):
        loop(st)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=st):
            loop(st)
        t = Timer(dev, st)
        g_ms = t.run(lambda i=0: graph.replay(), reps, warmup=3)
        e_ms = t.run(lambda i=0: loop(st), reps, warmup=3)
    assert R.reatt_workspace_status(ws, st) == R.OK
    del graph
    return {"steps_per_loop": n_steps, "T_first": w.T,
            "graph_us_per_step": round(statistics.median(g_ms) * 1e3 / n_steps, 2),
            "eager_us_per_step": round(statistics.median(e_ms) * 1e3 / n_steps, 2),
            "note": "median over replays; one L2 flush before each loop of steps"}


def prefill_loop(w, dev, timer, prompt=131072, chunk=512, reps=3):
    """NEXT step of a prefill as the pages run it: a first chunk of G+L
    tokens over an empty cache, then chunks of `chunk` tokens (chunk_size=512
    in the OpenReview discussion's NIAH settings), each attending over the
    cache built so far (span selection on its middle) and then appended in
    place (caches with T_cap = prompt rows).  Launched eagerly; L2 flushed
    before each prompt, not between its chunks."""
    import torch
    from top_kv_span_b200 import reatt as R

    first = w.G + w.L
    n = max(0, (prompt - first) // chunk)
    sizes = [first] + [chunk] * n
    P = sum(sizes)
    gen = torch.Generator(device=dev).manual_seed(w.seed + 91)
    rnd = lambda shp: torch.randn(shp, generator=gen, device=dev).to(w.torch_dtype)
    # per-chunk contiguous operands: [B, Hq, c, d] queries, [B, Hkv, c, d] K/V
    qs = [rnd((w.B, w.Hq, c, w.d)) for c in sizes]
    kn = [rnd((w.B, w.Hkv, c, w.d)) for c in sizes]
    vn = [rnd((w.B, w.Hkv, c, w.d)) for c in sizes]
    kc = torch.zeros((w.B, w.Hkv, P, w.d), dtype=w.torch_dtype, device=dev)
    vc = torch.zeros_like(kc)
    dims, t = [], 0
    for c in sizes:
        dims.append(R.dims_of(w, T=t, C=c, T_cap=P))
        t += c
    ws = torch.zeros(max(R.reatt_workspace_bytes(dd) for dd in dims), dtype=torch.uint8,
                     device=dev)
    outs = {c: torch.empty((w.B, w.Hq, c, w.d), dtype=torch.float32, device=dev)
            for c in set(sizes)}
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device=dev)
    st = timer.stream

    def one_prompt(i=0):
        for j, c in enumerate(sizes):
            R.reatt_step(dims[j], qs[j], kc, vc, kn[j], vn[j], sel, outs[c], ws, stream=st)
            R.reatt_append_kv(dims[j], kc, vc, kn[j], vn[j], stream=st)

    ms = timer.run(one_prompt, reps, warmup=1)
    assert R.reatt_workspace_status(ws, st) == R.OK
    med = statistics.median(ms)
    return {"workload": w.name, "prompt_tokens": P, "first_chunk": first, "chunk": chunk,
            "chunks": len(sizes), "ms_per_prompt": round(med, 3),
            "tokens_per_s": round(P / (med * 1e-3), 1),
            "us_per_chunk": round(med * 1e3 / len(sizes), 2),
            "note": "eager launches; median over prompts; one L2 flush before each prompt"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_setup()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from top_kv_span_b200 import workloads as wl

    stream = torch.cuda.current_stream(dev)
    timer = Timer(dev, stream)
    w = wl.WORKLOADS[args.workload]
    # weak scaling: rank r runs its own sequences (seed offset by rank)
    w = w.replace(seed=w.seed + 1000 * rank)
    head = measure(w, args, dev, timer, world, rank,
                   cpu_leg_seconds=-1 if (world > 1 or args.no_cpu_baseline) else args.cpu_seconds,
                   single_seconds=args.cpu_single_seconds)
    line = summarise(head, world, args.steps, make_reduce_max(world, dev))
    result = {"metric": METRIC, "value": line.pop("value"), "unit": line.pop("unit"),
              "n_gpus": world, "steps": args.steps, "warmup": args.warmup}
    result.update({k: line[k] for k in ("ms_per_step", "step_us", "scan_us", "scan_gbs")})
    result.update({"higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                   "dtype": line["dtype"],
                   "data": "synthetic (seeded caches, per-channel sigma, planted needles)"})
    for k in ("config", "roofline", "step_roofline", "e2e", "gpu_launches", "clocks",
              "step_dist_us", "scan_dist_us", "parity", "cpu_baseline"):
        if k in line:
            result[k] = line[k]
    del head
    if world == 1 and args.extra:
        per = {}
        for name in args.extra.split(","):
            name = name.strip()
            if not name or name == args.workload:
                continue
            torch.cuda.empty_cache()
            r = measure(wl.WORKLOADS[name], args, dev, timer, cpu_leg_seconds=0.0)
            per[name] = summarise(r)
            del r
        result["per_workload"] = per
    if world == 1 and args.loops:
        torch.cuda.empty_cache()
        result["decode_loop"] = {name: decode_loop(wl.WORKLOADS[name], dev, timer)
                                 for name in args.loops.split(",") if name}
    if world == 1 and args.prefill_loop:
        torch.cuda.empty_cache()
        result["prefill_loop"] = prefill_loop(wl.WORKLOADS[args.prefill_loop], dev, timer)
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


def _swaps(ora_scores, ora_sel, gpu_sel, k):
    """Selection of each sampled head against the oracle's: exact, or
    differing only by swaps among spans within 1e-3 relative of the oracle's
    k-th score.  Returns (swaps, ok)."""
    import numpy as np
    swaps, ok = 0, True
    for idx in np.ndindex(ora_sel.shape[:2]):
        sc = ora_scores[idx]
        keff = min(k, sc.size)
        g = gpu_sel[idx]
        ok &= bool((g[keff:] == -1).all() and (np.diff(g[:keff]) > 0).all())
        O, Gs = set(ora_sel[idx][:keff].tolist()), set(g[:keff].tolist())
        if O == Gs:
            continue
        kth = np.sort(sc)[::-1][keff - 1]
        for sp in O ^ Gs:
            ok &= bool(0 <= sp < sc.size and abs(sc[sp] - kth) <= 1e-3 * abs(kth))
        swaps += len(O - Gs)
    return swaps, ok


def cpu_leg(w, x, gpu_sel, gpu_out, seconds=15.0, single_seconds=0.0, heads=1):
    """The CPU leg: the oracle as it stands on this host's cores over a
    bounded sample of the workload (the first KV head of sequence 0).  Its
    first run also gives the parity of that sample: the GPU's selection
    against the oracle's (swap rule) and the max-abs output error of the
    sample's query heads (for a prefill chunk: spans and queries sampled).
    With seconds > 0 the run repeats for ~seconds (cpu_baseline), then for
    ~single_seconds on one core."""
    import numpy as np

    import oracle
    oracle.set_threads(host_cores())
    tol = 1e-4 if w.dtype == "f32" else 2e-2
    xs, ws = oracle_sample(w, x, heads)
    _, sb = step_bytes(ws)
    g = w.Hq // w.Hkv
    gsel = gpu_sel[:1, :heads]
    gout = gpu_out[:1, :heads * g].astype(np.float64)
    t0 = time.perf_counter()
    if w.C == 1:
        ref = oracle.step(**xs, G=ws.G, L=ws.L, S=ws.S, k=ws.k, rope_base=ws.rope_base)
        swaps, ok = _swaps(ref["scores"], ref["sel"], gsel, w.k)
        if not np.array_equal(ref["sel"], gsel):
            ref = oracle.step(**xs, G=ws.G, L=ws.L, S=ws.S, k=ws.k, rope_base=ws.rope_base,
                              sel=gsel)
        err = float(np.abs(gout - ref["out"]).max())
        parity = {"sample": f"sequence 0, KV heads 0..{heads - 1} of {w.Hkv}: every span "
                            "scored, full selection and output", "swaps": swaps,
                  "selection_ok": ok, "max_abs": err, "tol": tol, "ok": ok and err <= tol}
    else:
        # prefill chunk: the chosen spans with the lowest oracle scores must
        # not lose to unchosen ones (sampled), and sampled queries' outputs
        rng = np.random.default_rng(0)
        mask = np.zeros(max(1, (w.T - w.G - w.L + w.S - 1) // w.S), bool)
        NS = mask.size if w.T > w.G + w.L else 0
        ok, swaps = True, 0
        if NS and w.k:
            chosen = gsel[0, 0][gsel[0, 0] >= 0]
            mask[chosen] = True
            ch, un = np.flatnonzero(mask), np.flatnonzero(~mask)
            pick = np.concatenate([rng.choice(ch, min(8, ch.size), replace=False),
                                   rng.choice(un, min(8, un.size), replace=False)])
            pairs = np.stack([np.zeros_like(pick), pick], 1)
            sc = oracle.span_scores_list(xs["q"], xs["k_cache"], ws.G, ws.L, ws.S, pairs)
            sel_sc, un_sc = sc[:min(8, ch.size)], sc[min(8, ch.size):]
            lo = sel_sc.min() if sel_sc.size else np.inf
            ok = bool(un_sc.size == 0 or un_sc.max() <= lo + 1e-3 * abs(lo))
        c_list = sorted({0, w.C - 1, *rng.choice(w.C, 14, replace=False).tolist()})
        ref = oracle.step(**xs, G=ws.G, L=ws.L, S=ws.S, k=ws.k, rope_base=ws.rope_base,
                          sel=gsel, c_list=c_list)
        err = float(np.abs(gout[:, :, c_list] - ref["out"][:, :, c_list]).max())
        parity = {"sample": f"sequence 0, KV head 0: 16 sampled spans (8 chosen, 8 not) "
                            f"and {len(c_list)} sampled queries", "swaps": swaps,
                  "selection_ok": ok, "max_abs": err, "tol": tol, "ok": ok and err <= tol}
    first = time.perf_counter() - t0
    out = {"parity": parity}
    if seconds <= 0 or w.C != 1:
        return out

    def timed(limit):
        t1 = time.perf_counter()
        n = 0
        while True:
            oracle.step(**xs, G=ws.G, L=ws.L, S=ws.S, k=ws.k, rope_base=ws.rope_base,
                        want_scores=False)
            n += 1
            if time.perf_counter() - t1 > limit:
                break
        return (time.perf_counter() - t1) / n, n

    cores = oracle.max_threads()
    dt, n = timed(seconds)
    out.update({"value": round(sb / dt / 1e9, 4), "unit": "GB/s", "cores": cores,
                "kind": "oracle", "sample": f"{w.name}: sequence 0, {heads} of {w.Hkv} KV heads "
                                            f"({heads * g} query heads), {n} oracle steps",
                "sec_per_sample_step": round(dt, 4), "first_run_s": round(first, 3)})
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
    oracle.set_threads(host_cores())
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


DEFAULT_EXTRA = "tiny_f32_4k,llama3_8b_1m_x4,llama3_8b_prefill_256k,qwen2_1p5b_4m"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama3_8b_128k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--cpu-single-seconds", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra", default=DEFAULT_EXTRA,
                    help="comma-separated workloads measured after the headline one (N=1 only); "
                         "'' for none")
    ap.add_argument("--loops", default="tiny_f32_4k,llama3_8b_128k",
                    help="workloads whose graph-replayed decoding loop is timed (N=1 only)")
    ap.add_argument("--prefill-loop", default="llama3_8b_128k",
                    help="workload whose heads time a chunked 128K-token prefill "
                         "(first chunk G+L, then 512-token chunks with appends); '' skips it")
    ap.add_argument("--launch-check", action="store_true",
                    help="multi-rank plumbing only, on CPU ranks (gloo), no GPU work")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args.gpus, sys.argv[1:]))
    if args.launch_check:
        run_launch_check(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
