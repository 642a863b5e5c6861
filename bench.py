#!/usr/bin/env python3
"""Benchmark of the sm_100a exact attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-per-workload]

One step = one attention forward (the whole hot path) over one batch of the
workload: by default the 40x40 YOLO neck attention, B=16, H=4, Nq=Nk=1600,
d=64, fp16, non-causal.  Inputs are seeded synthetic N(0,1) tensors resident
in HBM; L2 (126 MB) is flushed by a 256 MiB write before every timed step
because these inputs are smaller than L2.  Each step is timed with CUDA
events on the launching stream; the timed region is bracketed by a barrier
and a device synchronisation, and multi-GPU runs report the max over ranks.
With N > 1 (torchrun), every rank runs its own copy of the workload over
its own (batch, head) slice -- the method has no exchange step, so there is
no collective on the data path (weak scaling).

Rank 0 prints one JSON line.  ``--impl reference`` times the float64 CPU
oracle instead (the slow baseline), on a bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOPS & % of B200 roofline; µs/call at YOLO shapes"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
DEFAULT_WORKLOAD = "yolo_neck_40x40_b16"
FLUSH_BYTES = 256 << 20
KERNEL_SOURCES = ["exact_attention_153_b200/csrc/attn_fwd_sm100.cuh",
                  "exact_attention_153_b200/csrc/sm100_ptx.cuh",
                  "exact_attention_153_b200/csrc/attn_api.cu"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_kernel_traffic.json")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    p = dict(FALLBACK_PEAKS)
    p["source"] = "fallback"
    return p


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if still current."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        doc = json.load(f)
    ent = doc.get("workloads", {}).get(workload)
    if not ent or doc.get("kernel_source_sha") != kernel_source_sha():
        return None
    return ent.get("dram_bytes_per_launch")


def roofline(w, t_s, peaks, sustained=False):
    """Which roof bounds this workload and how close one launch gets to it."""
    flops_peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * 1e12
    bw_peak = peaks["hbm_gbs"] * 1e9
    if w.flops / w.bytes >= flops_peak / bw_peak:
        achieved = w.flops / t_s / 1e12
        peak = flops_peak / 1e12
        return {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4)}
    achieved = w.bytes / t_s / 1e9
    peak = bw_peak / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": round(peak, 1),
            "unit": "GB/s", "frac": round(achieved / peak, 4)}


class ClockSampler(threading.Thread):
    """Polls SM clock and clock-event reasons through NVML during the timed region."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._halt = threading.Event()
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report it, keep benchmarking
            self.nv = None
            self.error = repr(e)

    def run(self):
        if self.nv is None:
            return
        nv = self.nv
        while not self._halt.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception as e:
                self.error = repr(e)
                return
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)

    def summary(self):
        reasons = [name for bit, name in self.REASONS.items() if self.reasons & bit]
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
               "source": "nvml"}
        if self.error:
            out["error"] = self.error
        return out


L2_NOTE = "flushed before every timed call (256 MiB write)"
GRAPH_CALLS = {"yolo_c2psa_20x20": 2000, "yolo_neck_40x40_b16": 200,
               "yolo_highres_80x80_b16": 20, "llm_causal_2048": 20, "long_context_32k": 5}


def bench_config(w, world: int) -> dict:
    """The config dict of the JSON line; both arms print exactly this for the same workload."""
    return dict(w.as_config(), l2=L2_NOTE,
                parallelism=f"dp{world} over (batch, head) slices, no collective")


def percentiles(values):
    """Median, p10, p90 and mean of a list of per-call times."""
    import numpy as np
    a = np.asarray(values, dtype=np.float64)
    return {"median": float(np.median(a)), "p10": float(np.percentile(a, 10)),
            "p90": float(np.percentile(a, 90)), "mean": float(a.mean())}


def rank_seed(w, rank: int) -> int:
    """Seed of rank ``rank``'s own copy of the workload (weak scaling: one slice per rank)."""
    return w.seed + 1000 * rank


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank timing over all ranks (the slowest rank sets the job time)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_step: float, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every rank ran ``steps`` steps of its own slice."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def time_oracle_sample(w, q, k, v, budget_s=12.0, max_heads=None):
    """Run the float64 oracle over whole (batch, head) slices until the budget is spent."""
    import numpy as np
    import oracle
    rows = np.arange(w.Nq)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    if max_heads is not None:
        heads = heads[:max_heads]
    done = 0
    t0 = time.perf_counter()
    for b, h in heads:
        oracle.attention_head_rows(q[b, h], k[b, h], v[b, h], w.scale, w.causal, rows)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    flops = w.flops * done / len(heads) if max_heads is None else w.flops * done / (w.B * w.H)
    return flops, dt, done


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:
        return None


def run_reference(args, w):
    """The oracle as it stands, on the host cores: each step one bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from seeded_inputs import make_workload_qkv
    q, k, v = make_workload_qkv(w)
    heads_per_step = max(1, min(w.B * w.H, 8))
    for _ in range(args.warmup):
        time_oracle_sample(w, q, k, v, budget_s=1e9, max_heads=heads_per_step)
    tot_flops = tot_t = 0.0
    for _ in range(args.steps):
        f, dt, _ = time_oracle_sample(w, q, k, v, budget_s=1e9, max_heads=heads_per_step)
        tot_flops += f
        tot_t += dt
    value = tot_flops / tot_t / 1e12
    cores = blas_threads() or cpu_cores()
    sample = (f"{heads_per_step} of {w.B * w.H} (batch, head) slices per step, all "
              f"{w.Nq} query rows each, float64 numpy")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": int(os.environ.get("WORLD_SIZE", args.gpus)), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1))",
        "config": bench_config(w, int(os.environ.get("WORLD_SIZE", args.gpus))),
        "reference_run": "float64 oracle on the host cores of rank 0; other ranks do no work",
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the context timings of the other workloads")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of float64 oracle work for cpu_baseline")
    ap.add_argument("--part", choices=["forward", "backward", "block", "fp8"], default="forward",
                    help="with --kernel-only: which path to run (for ncu captures)")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time only the device loop (no e2e, CPU baseline or context timings);"
                         " used for ncu captures")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from seeded_inputs import workload
    w = workload(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.kernel_only and args.part != "forward":
        return run_part(args, w)

    import torch
    import torch.distributed as dist
    import exact_attention_153_b200 as attn
    from seeded_inputs import Workload, make_qkv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    peaks = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    # each rank: its own seeded copy of the workload (weak scaling over (batch, head))
    q, k, v = make_qkv(w.B, w.H, w.Nq, w.Nk, w.d, w.dtype, rank_seed(w, rank), w.qk_scale)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    od = torch.empty_like(qd)
    ld = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    code = attn.ATTN_BF16 if w.dtype == "bf16" else attn.ATTN_FP16
    sh = stream.cuda_stream
    # split-mode workspace (allocated once, outside the timed region; None when unused)
    ws = attn.workspace_for(qd, kd, w.causal)
    ws_ptr = ws.data_ptr() if ws is not None else None
    ws_bytes = ws.numel() if ws is not None else 0

    def step():
        st = attn.attn_fwd_ws(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                              ld.data_ptr(), w.B, w.H, w.Nq, w.Nk, w.d, w.scale, w.causal, code,
                              ws_ptr, ws_bytes, sh)
        if st != 0:
            raise attn.AttnError(st)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    kernel_ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    total_ms = max_over_ranks(sum(kernel_ms), dist if world > 1 else None, dev)
    st, word = attn.attn_get_device_status(sh)
    if st != 0:
        raise attn.AttnError(st, f"device status {word:#x}")
    if args.kernel_only:
        if rank == 0:
            ms = total_ms / args.steps
            print(json.dumps({"workload": w.name, "us_per_call": round(ms * 1e3, 2),
                              "tflops": round(world * w.flops / (ms * 1e-3) / 1e12, 2),
                              "n_gpus": world, "steps": args.steps}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    # ---------------------------------------------------------------- end to end
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32).pin_memory()

    def e2e_step():
        st = attn.attn_fwd_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), oh.data_ptr(),
                                lh.data_ptr(), qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                od.data_ptr(), ld.data_ptr(), ws_ptr, ws_bytes, w.B, w.H, w.Nq,
                                w.Nk, w.d, w.scale, w.causal, code, sh)
        if st != 0:
            raise attn.AttnError(st, "attn_fwd_host")

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), dist if world > 1 else None, dev)

    ms_per_step = total_ms / args.steps
    value = job_tflops(world, w.flops, args.steps, total_ms)
    e2e_value = job_tflops(world, w.flops, args.steps, e2e_ms)
    per_launch_s = ms_per_step * 1e-3
    roof = roofline(w, per_launch_s, peaks)
    roof["peak_source"] = peaks["source"]
    roof["traffic"] = recorded_traffic(w.name)
    roof["algorithmic_flops_per_launch"] = w.flops
    roof["algorithmic_bytes_per_launch"] = w.bytes

    per_workload = None
    backward = None
    blocks = None
    fp8 = None
    cpu = None
    if rank == 0 and world == 1 and not args.no_per_workload:
        per_workload = context_timings(attn, torch, dev, peaks, steps=args.steps,
                                       warmup=args.warmup, device_index=local)
        backward = backward_timings(attn, torch, dev, peaks, warmup=args.warmup)
        blocks = block_timings(attn, torch, dev, peaks, warmup=args.warmup)
        fp8 = fp8_timings(attn, torch, dev, peaks, warmup=args.warmup)
    if rank == 0:
        flops, dt, done = time_oracle_sample(w, q, k, v, budget_s=args.cpu_budget)
        cpu = {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": blas_threads() or cpu_cores(),
               "kind": "oracle",
               "sample": f"{done} of {w.B * w.H} (batch, head) slices of {w.name}, all "
                         f"{w.Nq} rows each, float64 numpy, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "us_per_call": round(ms_per_step * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded N(0,1), recipe in seeded_inputs)",
            "config": bench_config(w, world),
            "us_per_call_stats": {k: round(v * 1e3, 2) for k, v in percentiles(kernel_ms).items()},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOPS",
                    "h2d_bytes_per_step": int(q.numel() + k.numel() + v.numel()) * 2,
                    "d2h_bytes_per_step": int(q.numel()) * 2 + w.B * w.H * w.Nq * 4,
                    "ms_per_step": round(e2e_ms / args.steps, 4),
                    "path": "attn_fwd_host: pinned host -> device, kernel, device -> host"},
            "gpu_launches": args.steps,
            "split_mode": ws is not None,
            "clocks": sampler.summary(),
            "kernel_source_sha": kernel_source_sha(),
        }
        if per_workload is not None:
            line["per_workload"] = per_workload
        if backward is not None:
            line["backward"] = backward
        if blocks is not None:
            line["block"] = blocks
        if fp8 is not None:
            line["fp8"] = fp8
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def backward_flops(w) -> float:
    """Algorithmic FLOPs of the backward: five N x N x d contractions (S, dP, dV, dK, dQ)."""
    f = 10.0 * w.B * w.H * w.Nq * w.Nk * w.d
    return f / 2.0 if w.causal else f


def backward_timings(attn, torch, dev, peaks, steps=20, warmup=3):
    """µs/call (L2 flushed before each call; median, p10, p90) and TFLOP/s of attn_bwd
    (row pass, main pass, dQ conversion) on every workload."""
    from seeded_inputs import WORKLOADS, make_grad_out, make_workload_qkv
    out = {}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for w in WORKLOADS:
        q, k, v = (t.to(dev) for t in make_workload_qkv(w))
        do = make_grad_out(w.B, w.H, w.Nq, w.d, w.dtype, w.seed).to(dev)
        o, lse = attn.forward(q, k, v, causal=w.causal)
        ws = torch.empty(attn.attn_bwd_workspace_size(w.B, w.H, w.Nq, w.Nk, w.d),
                         dtype=torch.uint8, device=dev)
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        for _ in range(max(3, warmup)):
            attn.backward(q, k, v, o, lse, do, causal=w.causal, workspace=ws, out=grads)
        torch.cuda.synchronize()
        times = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            attn.backward(q, k, v, o, lse, do, causal=w.causal, workspace=ws, out=grads)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3)
        st = percentiles(times)
        us = st["median"]
        tf = backward_flops(w) / (us * 1e-6) / 1e12
        out[w.name] = {"us_per_call": round(us, 2), "us_p10": round(st["p10"], 2),
                       "us_p90": round(st["p90"], 2), "tflops": round(tf, 2),
                       "frac": round(tf / peaks["bf16_tflops"], 4), "bound": "tensor",
                       "launches": 3}
        del q, k, v, do, o, lse, ws, grads
        torch.cuda.empty_cache()
    return out


FP8_CONFIGS = [
    # name, B, H, N, causal, qk_scale: the d = 128 workload, and the 80x80 map's 256
    # channels as two heads of d = 128
    ("long_context_32k", 1, 32, 32768, True, 0.5),
    ("yolo_highres_80x80_b16_d128", 16, 2, 6400, False, 1.0),
]


def fp8_config(name):
    for c in FP8_CONFIGS:
        if c[0] == name:
            return c
    raise KeyError(name)


def fp8_timings(attn, torch, dev, peaks, steps=20, warmup=3):
    """µs/call (L2 flushed before each call; median, p10, p90) of the e4m3 forward, next to
    the bf16 forward on inputs of the same shape.  Its roofline peak is the measured bf16
    GEMM rate times 2, the nominal e4m3 / bf16 tensor-rate ratio (4.5 / 2.25 PFLOP/s)."""
    from seeded_inputs import make_fp8_qkv, make_qkv
    out = {}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peak = 2.0 * peaks["bf16_tflops"]

    def timed(fn):
        for _ in range(max(3, warmup)):
            fn()
        torch.cuda.synchronize()
        times = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3)
        return percentiles(times)

    for name, B, H, N, causal, qk in FP8_CONFIGS:
        q8, k8, vt8, ds = make_fp8_qkv(B, H, N, N, 128, seed=1005, qk_scale=qk)
        q8, k8, vt8 = q8.to(dev), k8.to(dev), vt8.to(dev)
        ws = attn.workspace_for(q8, k8, causal)
        o = torch.empty((B, H, N, 128), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        st8 = timed(lambda: attn.forward_fp8(q8, k8, vt8, ds, causal=causal, out=o, lse=lse,
                                             workspace=ws))
        del q8, k8, vt8
        q, k, v = (t.to(dev) for t in make_qkv(B, H, N, N, 128, "bf16", seed=1005, qk_scale=qk))
        ws16 = attn.workspace_for(q, k, causal)
        st16 = timed(lambda: attn.forward(q, k, v, causal=causal, out=o, lse=lse,
                                          workspace=ws16))
        flops = 4.0 * B * H * N * N * 128 * (0.5 if causal else 1.0)
        tf = flops / (st8["median"] * 1e-6) / 1e12
        out[name] = {"B": B, "H": H, "N": N, "d": 128, "causal": causal,
                     "us_per_call": round(st8["median"], 2), "us_p10": round(st8["p10"], 2),
                     "us_p90": round(st8["p90"], 2), "tflops": round(tf, 2),
                     "frac": round(tf / peak, 4), "peak": round(peak, 1),
                     "peak_source": "measured bf16 x 2 (nominal e4m3 / bf16 ratio)",
                     "bf16_us_per_call": round(st16["median"], 2),
                     "speedup_vs_bf16": round(st16["median"] / st8["median"], 3)}
        del q, k, v, o, lse, ws, ws16
        torch.cuda.empty_cache()
    return out


BLOCK_CONFIGS = [
    # name, B, N, H, d, dtype, causal: the attention block around two of the workloads
    ("yolo_neck_40x40_b16_block", 16, 1600, 4, 64, "fp16", False),
    ("llm_causal_2048_block", 32, 2048, 16, 64, "fp16", True),
]


def block_timings(attn, torch, dev, peaks, steps=20, warmup=3):
    """µs per attn_block_fwd call (qkv GEMM, attention, output GEMM; L2 flushed before each
    call) and the time of each of its three kernels alone."""
    from seeded_inputs import make_block_inputs
    out = {}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for name, B, N, H, d, dtype, causal in BLOCK_CONFIGS:
        C = H * d
        x, w_qkv, b_qkv, w_o, b_o = (t.to(dev) if t is not None else None
                                     for t in make_block_inputs(B, N, H, d, C, dtype, seed=7))
        q, k, v, o = (torch.empty((B, H, N, d), dtype=x.dtype, device=dev) for _ in range(4))
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        y = torch.empty_like(x)
        code = attn.ATTN_BF16 if dtype == "bf16" else attn.ATTN_FP16
        sh = torch.cuda.current_stream().cuda_stream
        calls = {
            "block": lambda: attn.attn_block_fwd(
                x.data_ptr(), w_qkv.data_ptr(), None, w_o.data_ptr(), b_o.data_ptr(),
                q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                y.data_ptr(), B, N, H, d, C, 1.0 / math.sqrt(d), causal, code, sh),
            "qkv_proj": lambda: attn.attn_qkv_proj(x.data_ptr(), w_qkv.data_ptr(), None,
                                                   q.data_ptr(), k.data_ptr(), v.data_ptr(), B,
                                                   N, H, d, code, sh),
            "attention": lambda: attn.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                               o.data_ptr(), lse.data_ptr(), B, H, N, N, d,
                                               1.0 / math.sqrt(d), causal, code, sh),
            "out_proj": lambda: attn.attn_out_proj(o.data_ptr(), w_o.data_ptr(), b_o.data_ptr(),
                                                   y.data_ptr(), B, N, H, d, C, code, sh),
        }
        res = {"B": B, "N": N, "H": H, "d": d, "C": C, "dtype": dtype, "causal": causal}
        for part, fn in calls.items():
            for _ in range(max(3, warmup)):
                assert fn() == 0
            times = []
            for _ in range(steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                assert fn() == 0
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1) * 1e3)
            res[part + "_us"] = round(percentiles(times)["median"], 2)
        gemm_flops = 2.0 * B * N * C * 3 * C + 2.0 * B * N * C * C
        attn_flops = 4.0 * B * H * N * N * d / (2.0 if causal else 1.0)
        res["tflops"] = round((gemm_flops + attn_flops) / (res["block_us"] * 1e-6) / 1e12, 2)
        res["qkv_proj_tflops"] = round(2.0 * B * N * C * 3 * C / (res["qkv_proj_us"] * 1e-6) / 1e12, 2)
        res["out_proj_tflops"] = round(2.0 * B * N * C * C / (res["out_proj_us"] * 1e-6) / 1e12, 2)
        out[name] = res
        del x, w_qkv, w_o, b_o, q, k, v, o, lse, y
        torch.cuda.empty_cache()
    return out


def graph_per_call_us(attn, torch, w, q, k, v, o, lse, ws, calls: int, replays: int = 10):
    """Per-call µs of ``calls`` back-to-back forwards captured in one CUDA graph (L2 warm).

    Launch overhead is amortised over the graph; each call is still its own
    kernel launch (nothing is merged).  Returns the median over ``replays``.
    """
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream, outside the graph
        for _ in range(3):
            attn.forward(q, k, v, causal=w.causal, out=o, lse=lse, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(calls):
            attn.forward(q, k, v, causal=w.causal, out=o, lse=lse, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(replays):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3 / calls)
    del g
    return statistics.median(times)


def run_part(args, w):
    """--kernel-only for the backward or the block: W warm-up and K timed calls on one GPU."""
    import torch
    import exact_attention_153_b200 as attn
    from seeded_inputs import make_block_inputs, make_grad_out, make_workload_qkv
    dev = torch.device("cuda", 0)
    if args.part == "fp8":
        from seeded_inputs import make_fp8_qkv
        _, B, H, N, causal, qk = fp8_config(w.name if w.d == 128 else "yolo_highres_80x80_b16_d128")
        q8, k8, vt8, ds = (x.to(dev) if hasattr(x, "to") else x
                           for x in make_fp8_qkv(B, H, N, N, 128, seed=1005, qk_scale=qk))
        ws = attn.workspace_for(q8, k8, causal)
        fn = lambda: attn.forward_fp8(q8, k8, vt8, ds, causal=causal, workspace=ws)
        flops = 4.0 * B * H * N * N * 128 * (0.5 if causal else 1.0)
    elif args.part == "backward":
        q, k, v = (t.to(dev) for t in make_workload_qkv(w))
        do = make_grad_out(w.B, w.H, w.Nq, w.d, w.dtype, w.seed).to(dev)
        o, lse = attn.forward(q, k, v, causal=w.causal)
        ws = torch.empty(attn.attn_bwd_workspace_size(w.B, w.H, w.Nq, w.Nk, w.d),
                         dtype=torch.uint8, device=dev)
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        fn = lambda: attn.backward(q, k, v, o, lse, do, causal=w.causal, workspace=ws, out=grads)
        flops = backward_flops(w)
    else:
        C = w.H * w.d
        x, w_qkv, b_qkv, w_o, b_o = (t.to(dev) if t is not None else None
                                     for t in make_block_inputs(w.B, w.Nq, w.H, w.d, C, w.dtype, 7))
        fn = lambda: attn.block_forward(x, w_qkv, b_qkv, w_o, b_o, w.H, causal=w.causal)
        flops = 8.0 * w.B * w.Nq * C * C + w.flops
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"workload": w.name, "part": args.part, "us_per_call": round(ms * 1e3, 2),
                      "tflops": round(flops / (ms * 1e-3) / 1e12, 2), "steps": args.steps}),
          flush=True)
    return 0


def context_timings(attn, torch, dev, peaks, steps=50, warmup=5, device_index=0):
    """Every workload: cold single-call µs (L2 flushed each call; median, p10, p90), TFLOPS and
    roofline fraction of the median, the clocks seen meanwhile, and a CUDA-graph-replayed warm
    per-call figure."""
    from seeded_inputs import WORKLOADS, make_workload_qkv
    out = {}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for w in WORKLOADS:
        q, k, v = (t.to(dev) for t in make_workload_qkv(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        ws = attn.workspace_for(q, k, w.causal)
        for _ in range(max(3, warmup)):
            flush.zero_()
            attn.forward(q, k, v, causal=w.causal, out=o, lse=lse, workspace=ws)
        torch.cuda.synchronize()
        sampler = ClockSampler(device_index)
        sampler.start()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record()
            attn.forward(q, k, v, causal=w.causal, out=o, lse=lse, workspace=ws)
            e1.record()
        torch.cuda.synchronize()
        times = [e0.elapsed_time(e1) * 1e3 for e0, e1 in evs]
        calls = GRAPH_CALLS.get(w.name, 20)
        graph_us = graph_per_call_us(attn, torch, w, q, k, v, o, lse, ws, calls)
        sampler.stop()
        st = percentiles(times)
        us = st["median"]
        r = roofline(w, us * 1e-6, peaks)
        out[w.name] = {"us_per_call": round(us, 2),
                       "us_p10": round(st["p10"], 2), "us_p90": round(st["p90"], 2),
                       "calls": steps, "split": ws is not None,
                       "tflops": round(w.flops / (us * 1e-6) / 1e12, 2),
                       "bound": r["bound"], "frac": r["frac"],
                       "frac_of_sustained": roofline(w, us * 1e-6, peaks, sustained=True)["frac"],
                       "graph_warm_us_per_call": round(graph_us, 2), "graph_calls": calls,
                       "graph_warm_frac": roofline(w, graph_us * 1e-6, peaks)["frac"],
                       "clocks": sampler.summary()}
        del q, k, v, o, lse
        torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    sys.exit(main())
