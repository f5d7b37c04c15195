#!/usr/bin/env python
"""Benchmark of one MLA decode step over a paged latent KV cache on B200.

A step is one call of the C ABI's mla_decode_run on one batch: the absorb
kernel, the split-KV latent decode kernel and the LSE-combine + W_UV kernel.
Default workload: the DeepSeek-V3 attention shape at 32K context (B=32,
128 heads, r=512, rope 64, bf16), the shape the metric is quoted on.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle as the reference arm

Prints ONE JSON line on rank 0. Under torchrun (N > 1) every rank decodes its
own replica of the workload (the path shards over independent sequences:
weak scaling, no collective on the data path); value = the cache bytes of all
ranks / the slowest rank's time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import random
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")
METRIC = "MLA decode: KV-cache GB/s & TFLOP/s vs B200 roofline; µs/step at 32K ctx"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="deepseek_v3")
    ap.add_argument("--kernel", choices=["auto", "simt", "tcgen05"], default="auto")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="oracle work for the cpu_baseline sample")
    ap.add_argument("--blasst", type=float, default=None, metavar="LOG2",
                    help="decode with threshold skipping of key groups below the running max + LOG2 (<= 0)")
    ap.add_argument("--tpla-shard", action="store_true",
                    help="TPLA workloads on one GPU: time one GPU's latent shard of the multi-GPU form "
                         "(no all-reduce: the other shards live on other GPUs)")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling cases)")
    ap.add_argument("--context", type=int, default=0, help="override every length (profiling cases)")
    return ap.parse_args()


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
# algorithmic work of one step: cache bytes (r + d_rope elements per cached
# token), absorbed-query bytes (one query row per sequence and head), weight and
# output bytes, and the FLOPs of the absorb, QK, PV and up-projection
# contractions
# ----------------------------------------------------------------------------
def step_work(wl, lens):
    elt = 4 if wl.dtype == "fp32" else 2
    B, Lq, H = len(lens), wl.q_len, wl.heads
    r, dr, dn, dv, S = wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim, wl.latent_shards
    sum_l = int(sum(lens))
    rows = H * Lq
    # FP8 cache: r code bytes, the bf16 RoPE key and an fp32 scale per token
    cache = sum_l * (r + dr * 2 + 4) if wl.dtype == "fp8" else sum_l * (r + dr) * elt
    q_full = B * rows * (r + dr) * elt
    weights = H * dn * r * elt + H * r * dv * elt
    io = B * rows * (dn + dr) * elt + B * rows * dv * elt
    qk = 2 * rows * sum_l * (r + S * dr)
    pv = 2 * rows * sum_l * r
    absorb = 2 * B * rows * dn * r
    upproj = 2 * B * rows * r * dv
    return dict(cache_bytes=cache, step_bytes=cache + weights + io,
                step_flops=qk + pv + absorb + upproj,
                decode_bytes=cache + q_full, decode_flops=qk + pv,
                exps=rows * sum_l * S)


# The sources a recorded traffic figure depends on: the decode kernel's own
# headers and the file that configures its launch (files of other kernels do
# not change what this one reads and writes).
_DECODE_SOURCES = ["common.cuh", "sm100_ptx.cuh", "tc_decode.cuh", "mla_decode_api.cu"]
TRAFFIC_SOURCES = {"bf16": _DECODE_SOURCES, "fp8": _DECODE_SOURCES + ["tc_decode_f8.cuh"]}


def kernel_source_digest(dtype="bf16"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_latent_kv_21_b200", "csrc")
    for fn in sorted(TRAFFIC_SOURCES.get(dtype, os.listdir(csrc))):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel, dtype="bf16"):
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(workload, {}).get(kernel)
    if not ent or ent.get("source_digest") != kernel_source_digest(dtype):
        return None
    return ent.get("bytes_per_launch")


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU while the timed region
    runs: NVML queries from a thread every 5 ms (read-only), or nvidia-smi
    -lms 50 where NVML is not available."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.rows = []  # (time, sm_mhz, max_mhz, power_w, set of reasons)
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            self.nvml = (pynvml, h)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.gpu_id], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _poll_nvml(self):
        nv, h = self.nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                mask = int(get_reasons(h))
                rs = {name for name, bit in self.REASONS if mask & bit}
                self.rows.append((time.time(), sm, self.max_mhz, pw, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def _read_smi(self):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.strip().split(",")]
            if len(parts) < 10:
                continue
            rs = {name for (name, _), val in zip(self.REASONS, parts[6:10])
                  if val.lower().startswith("active")}
            self.rows.append((time.time(), num(parts[2]), num(parts[3]), num(parts[4]), rs))

    def stop(self):
        self.stop_flag.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        inside = [r for r in self.rows if t0 <= r[0] <= t1]
        if not inside:
            inside = [r for r in self.rows if r[0] >= t0][:1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [r[1] for r in inside if r[1] is not None]
        reasons = set()
        for r in inside:
            reasons |= r[4]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": inside[0][2], "reasons": sorted(reasons),
                "power_w_max": max((r[3] or 0.0) for r in inside),
                "samples": len(inside), "source": "nvml" if self.nvml else "nvidia-smi"}


# ----------------------------------------------------------------------------
# raw CUDA events (driver API) handed to the library for timing its decode kernel
# ----------------------------------------------------------------------------
class DriverEvents:
    def __init__(self):
        import ctypes
        self.ct = ctypes
        self.cu = ctypes.CDLL("libcuda.so.1")
        self.cu.cuEventCreate.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_uint]
        self.cu.cuEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p,
                                               ctypes.c_void_p]
        self.cu.cuEventDestroy_v2.argtypes = [ctypes.c_void_p]
        self.events = []

    def create(self) -> int:
        ev = self.ct.c_void_p()
        rc = self.cu.cuEventCreate(self.ct.byref(ev), 0)  # CU_EVENT_DEFAULT: timing enabled
        if rc != 0:
            raise RuntimeError(f"cuEventCreate failed ({rc})")
        self.events.append(ev.value)
        return ev.value

    def elapsed_ms(self, a: int, b: int) -> float:
        ms = self.ct.c_float()
        rc = self.cu.cuEventElapsedTime(self.ct.byref(ms), a, b)
        if rc != 0:
            raise RuntimeError(f"cuEventElapsedTime failed ({rc})")
        return float(ms.value)

    def destroy(self):
        for e in self.events:
            self.cu.cuEventDestroy_v2(e)
        self.events = []


# ----------------------------------------------------------------------------
# distributed plumbing (one process per GPU)
# ----------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    """The largest value of x over all ranks (each rank times its own GPU)."""
    if not dist:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tpla_layout(world: int, tp: int) -> dict:
    """Ranks of a TPLA run across GPUs: consecutive groups of tp ranks (one
    latent shard per rank, an all-reduce inside each group), the groups
    decoding independent replicas of the batch."""
    if tp < 1 or world % tp:
        raise ValueError(f"{world} ranks do not split into groups of {tp}")
    groups = [list(range(i, i + tp)) for i in range(0, world, tp)]
    return {"groups": groups, "tp_rank": [r % tp for r in range(world)],
            "group_of": [r // tp for r in range(world)]}


def whole_job_value(world: int, bytes_per_rank: float, ms_per_step: float) -> float:
    """GB/s of the whole job: every rank processes its own full batch (weak
    scaling, replicas), timed by the slowest rank."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e9


def emit(line: dict, rank: int) -> None:
    """Rank 0 alone prints the JSON line."""
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# oracle timing (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------
def oracle_threads():
    try:
        import threadpoolctl
        n = [i["num_threads"] for i in threadpoolctl.threadpool_info() if i["user_api"] == "blas"]
        if n:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle_sample(wl, inputs, pairs, tokens):
    """Runs the oracle on (sequence, head) pairs over their first `tokens` keys
    (Lq = 1 workloads) or full length; returns (seconds, outputs)."""
    import numpy as np
    from mla_workloads import logical_cache, stored_rows_fp8
    from oracle import fp8_cache, mla_oracle
    qn = inputs["q_nope"].double().numpy()
    qr = inputs["q_rope"].double().numpy()
    wuk = inputs["w_uk"].double().numpy()
    wuv = inputs["w_uv"].double().numpy()
    outs = []
    t0 = time.perf_counter()
    for b, h in pairs:
        if wl.dtype == "fp8":
            codes, rope, scale = stored_rows_fp8(inputs, b, wl)
            c, k = fp8_cache.logical_cache_fp8(codes.numpy(), rope.double().numpy(), scale.double().numpy())
        else:
            c, k = logical_cache(inputs, b, wl)
            c, k = c.double().numpy(), k.double().numpy()
        n = min(tokens, c.shape[0]) if tokens else c.shape[0]
        outs.append(mla_oracle.mla_decode(qn, qr, {b: c[:n]}, {b: k[:n]}, wuk, wuv,
                                          wl.softmax_scale, wl.latent_shards, [b], [h]))
    return time.perf_counter() - t0, outs


def compare_sample(gpu_out, oracle_outs, pairs, dtype):
    """max-abs / rel-Frobenius of the GPU output against the oracle's sampled rows."""
    import numpy as np
    got = np.concatenate([gpu_out[b, :, h].double().numpy().ravel() for b, h in pairs])
    ref = np.concatenate([o[0, :, 0].ravel() for o in oracle_outs])
    d = got - ref
    return {"max_abs": float(np.abs(d).max()),
            "rel_fro": float(np.linalg.norm(d) / np.linalg.norm(ref)),
            "pairs": [list(p) for p in pairs],
            # FP8 cache: 1.5x the rms relative error its rounding steps give
            # (2.79e-3), and no absolute bound (its element-wise bound scales
            # with |out|); bf16: the stated bounds
            "tolerance": ({"rel_fro": 1e-5} if dtype == "fp32"
                          else {"rel_fro": 4.19e-3} if dtype == "fp8"
                          else {"max_abs": 2e-2, "rel_fro": 5e-3})}


def reference_arm(args, wl, world, rank):
    """The CPU oracle as it stands, timed on host cores (rank 0 only)."""
    if rank != 0:
        return
    from mla_workloads import generate
    inputs = generate(wl)
    lens = inputs["seq_lens"].tolist()
    work = step_work(wl, lens)
    B, H = len(lens), wl.heads
    # calibrate: seconds per (head x token) on a small sample
    t_cal, _ = time_oracle_sample(wl, inputs, [(0, 0)], 2048)
    per_token = t_cal / 2048
    budget = min(2.0, 150.0 / max(1, args.steps + args.warmup))
    tokens = int(max(256, min(min(lens), budget / max(per_token, 1e-9))))
    pairs = [(i % B, (7 * i) % H) for i in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        time_oracle_sample(wl, inputs, [pairs[i]], tokens)
    total, done_tokens = 0.0, 0
    for i in range(args.warmup, args.warmup + args.steps):
        dt, _ = time_oracle_sample(wl, inputs, [pairs[i]], tokens)
        total += dt
        done_tokens += min(tokens, lens[pairs[i][0]])
    frac = done_tokens / (sum(lens) * H)          # share of the step's (token, head) work
    value = work["cache_bytes"] * frac / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": B, "heads": H, "q_len": wl.q_len,
                   "context": wl.context, "latent_rank": wl.latent_rank,
                   "rope_dim": wl.rope_dim, "latent_shards": wl.latent_shards},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle_threads(),
                         "kind": "oracle",
                         "sample": f"per step one (sequence, head) pair over its first "
                                   f"{tokens} keys; throughput scaled by the pair's share "
                                   f"of the step's (token x head) work"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
PREFILL_METRIC = "MLA-form prefill: TFLOP/s vs B200 bf16 tensor roofline"


def prefill_work(wl, lens):
    """FLOPs of one causal prefill: the up-projection (K_nope and V of every
    token and head) and the attention (query t of a prompt sees t + 1 keys:
    QK over d_nope + d_rope, PV over d_v); bytes it must move at least."""
    H, r, dr, dn, dv = wl.heads, wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim
    T = int(sum(lens))
    pairs = sum(int(L) * (int(L) + 1) // 2 for L in lens)
    uproj = 2 * T * r * (dn + dv) * H
    attn = 2 * pairs * H * (dn + dr + dv)
    io = 2 * (T * H * (dn + dr + dv) + T * (r + dr) + H * r * (dn + dv))
    return {"flops": uproj + attn, "uproj_flops": uproj, "attn_flops": attn, "bytes": io}


def prefill_main(args, wl, world, rank, local):
    """One step = one MLA-form prefill of the workload's prompts (the prefill
    row of the method; the headline metric is the decode step)."""
    import torch
    import mla_latent_kv_21_b200 as M
    from mla_workloads import generate_prefill
    dist = init_dist(world)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    peaks, peaks_kind = load_peaks()
    inputs = generate_prefill(wl)
    lens = inputs["seq_lens"].tolist()
    work = prefill_work(wl, lens)
    dev = {k: v.to(device) for k, v in inputs.items()}
    dims = M.dims_for(wl.heads, wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim, 1, wl.softmax_scale,
                      wl.dtype, 1, wl.page_size)
    plan = M.PrefillPlan(dims, lens).allocate_workspace(device)
    T = sum(lens)
    out = torch.empty((T, wl.heads, wl.v_dim), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def step(d=dev, o=out, events=None):
        plan.run(d["q_nope"], d["q_rope"], d["kv_rows"], d["cu_seqlens"], d["w_uk"], d["w_uv"], o,
                 stream.cuda_stream, events)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    if plan.read_status() != 0:
        raise SystemExit("device status after warm-up: " + M.mla_status_string(plan.read_status()))
    K = args.steps
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    w0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    w_head = time.time()
    drv = DriverEvents()
    ev = [(drv.create(), drv.create()) for _ in range(K)]
    for i in range(K):
        step(events=ev[i])
    torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / K, dist, device)
    attn_s = statistics.mean(drv.elapsed_ms(a, b) for a, b in ev) * 1e-3
    drv.destroy()
    if plan.read_status() != 0:
        raise SystemExit("device status after timing")
    # end to end with host buffers: the prompts' inputs in, the output back, every step
    host = {k: inputs[k].pin_memory() for k in ("q_nope", "q_rope", "kv_rows", "cu_seqlens")}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()
    dset = {k: torch.empty_like(dev[k]) for k in host}
    Ke = max(1, min(K, 10))
    torch.cuda.synchronize(device)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(Ke):
        for k, t in host.items():
            dset[k].copy_(t, non_blocking=True)
        step(d={**dev, **dset})
        out_host.copy_(out, non_blocking=True)
    x1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(x0.elapsed_time(x1) / Ke, dist, device)
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    value = world * work["flops"] / (ms * 1e-3) / 1e12
    achieved = work["attn_flops"] / attn_s / 1e12
    line = {
        "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "batch": len(lens), "prompt_tokens": lens, "heads": wl.heads,
                   "latent_rank": wl.latent_rank, "rope_dim": wl.rope_dim, "nope_dim": wl.nope_dim,
                   "v_dim": wl.v_dim, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"K_nope / V workspace {plan.workspace_bytes / 1e9:.2f} GB, larger than L2"},
        "step_tflop": work["flops"] / 1e12,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "kernel": "prefill attention",
                     "peak_source": f"{peaks_kind} (bf16 sustained: a multi-ms kernel timed in a loop)",
                     "attn_us": attn_s * 1e6, "attn_launches_timed": K},
        "e2e": {"value": world * work["flops"] / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "us_per_step": e2e_ms * 1e3,
                "steps": Ke},
        "gpu_launches": 2 * K,
        "clocks": sampler.summary(w0, w_head),
    }
    emit(line, rank)
    plan.close()
    if dist:
        dist.destroy_process_group()


def main():
    args = parse_args()
    world, rank, local = dist_env()
    from mla_workloads import PREFILL_WORKLOADS, WORKLOADS, generate
    if args.workload in PREFILL_WORKLOADS:
        if args.impl == "reference":
            emit({"impl": "reference", "unavailable": "the oracle arm times the decode step; prefill has no "
                  "reference arm"}, rank)
            return
        pwl = PREFILL_WORKLOADS[args.workload]
        if args.batch:
            pwl = pwl.with_(batch=args.batch)
        if args.context:
            pwl = pwl.with_(context=args.context)
        prefill_main(args, pwl, world, rank, local)
        return
    wl = WORKLOADS[args.workload]
    if args.batch:
        wl = wl.with_(batch=args.batch)
    if args.context:
        wl = wl.with_(context=args.context, context_min=0)
    if args.impl == "reference":
        reference_arm(args, wl, world, rank)
        return

    import torch
    import mla_latent_kv_21_b200 as M

    dist = init_dist(world)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    peaks, peaks_kind = load_peaks()

    inputs = generate(wl)
    lens = inputs["seq_lens"].tolist()
    kernel = {"auto": M.MLA_KERNEL_AUTO, "simt": M.MLA_KERNEL_SIMT,
              "tcgen05": M.MLA_KERNEL_TCGEN05}[args.kernel]
    dims = M.dims_for(wl.heads, wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim, wl.q_len,
                      wl.softmax_scale, wl.dtype, wl.latent_shards, wl.page_size)
    # TPLA on more than one GPU: groups of latent_shards ranks, one latent shard
    # per rank, the shard outputs summed by one all-reduce per step (the
    # method's exchange step); every other workload runs replicas
    tp = wl.latent_shards if ((dist or args.tpla_shard) and wl.latent_shards > 1) else 1
    if tp > 1:
        from mla_workloads import tpla_shard_inputs
        if dist:
            lay = tpla_layout(world, tp)
            groups = [dist.new_group(g) for g in lay["groups"]]
            tp_rank, group = lay["tp_rank"][rank], groups[lay["group_of"][rank]]
        else:
            tp_rank, group = 0, None
        inputs = tpla_shard_inputs(inputs, wl, tp, tp_rank)
        plan = M.TplaShardPlan(dims, lens, tp=tp, group=group).allocate_workspace(device)
        if not dist:
            plan.run = plan.run_shard  # one GPU holds one shard here: nothing to sum
        work = step_work(wl.with_(latent_rank=wl.latent_rank // tp, latent_shards=1), lens)
    else:
        plan = M.DecodePlan(dims, lens, kernel=kernel).allocate_workspace(device)
        work = step_work(wl, lens)
    dev = {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in inputs.items()}
    B = len(lens)
    out = torch.empty((B, wl.q_len, wl.heads, wl.v_dim), dtype=wl.torch_dtype, device=device)
    stream = torch.cuda.current_stream(device)

    def run_plan(q_nope, q_rope, block_table, seq_lens, o, events=None):
        if wl.dtype == "fp8":
            plan.run_fp8(q_nope, q_rope, dev["kv_codes"], dev["kv_rope"], dev["kv_scale"], block_table,
                         seq_lens, dev["w_uk"], dev["w_uv"], o, stream.cuda_stream, events)
        elif args.blasst is not None:
            plan.run_blasst(q_nope, q_rope, dev["kv_pool"], block_table, seq_lens, dev["w_uk"], dev["w_uv"], o,
                            args.blasst, stream.cuda_stream, events)
        else:
            plan.run(q_nope, q_rope, dev["kv_pool"], block_table, seq_lens, dev["w_uk"], dev["w_uv"], o,
                     stream.cuda_stream, events)

    def step(events=None):
        run_plan(dev["q_nope"], dev["q_rope"], dev["block_table"], dev["seq_lens"], out, events)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    status = plan.read_status()
    if status != 0:
        raise SystemExit(f"device status after warm-up: {M.mla_status_string(status)}")

    K = args.steps
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    w0 = time.time()
    # headline: K uninstrumented steps (consecutive kernels may overlap their
    # launch and prologue with the previous kernel's tail)
    t_start.record(stream)
    for i in range(K):
        step()
    t_stop.record(stream)
    torch.cuda.synchronize(device)
    w_head = time.time()
    # the decode kernel alone: events recorded on the launch stream around it
    Kd = min(K, 200)
    drv = DriverEvents()
    ev = [(drv.create(), drv.create()) for _ in range(Kd)]
    for i in range(Kd):
        step(ev[i])
    torch.cuda.synchronize(device)
    w1 = time.time()
    if dist:
        dist.barrier()
    sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_stop)
    decode_ms = [drv.elapsed_ms(a, b) for a, b in ev]
    drv.destroy()
    elapsed_ms = max_over_ranks(elapsed_ms, dist, device)
    status = plan.read_status()
    if status != 0:
        raise SystemExit(f"device status after timing: {M.mla_status_string(status)}")

    # ---- end to end through the public API: host buffers, copies in the timed region.
    # A serving loop: every step copies its inputs from pinned host memory and
    # its output back; two device buffer sets and two copy streams let step i's
    # input copy and step i-1's output copy overlap step i-1's / step i's compute.
    host = {k: inputs[k].pin_memory() for k in ("q_nope", "q_rope", "block_table", "seq_lens")}
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    Ke = max(1, min(K, 200))
    dsets = [{k: torch.empty_like(dev[k]) for k in host} for _ in range(2)]
    douts = [torch.empty_like(out) for _ in range(2)]
    h2d_stream = torch.cuda.Stream(device)
    d2h_stream = torch.cuda.Stream(device)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "comp", "d2h")}

    def e2e_steps(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                h2d_stream.wait_event(ev["comp"][b])   # step i-2 is done reading set b
            with torch.cuda.stream(h2d_stream):
                for k, t in host.items():
                    dsets[b][k].copy_(t, non_blocking=True)
                ev["h2d"][b].record(h2d_stream)
            stream.wait_event(ev["h2d"][b])
            if i >= 2:
                stream.wait_event(ev["d2h"][b])        # out b of step i-2 has been copied out
            d = dsets[b]
            run_plan(d["q_nope"], d["q_rope"], d["block_table"], d["seq_lens"], douts[b])
            ev["comp"][b].record(stream)
            d2h_stream.wait_event(ev["comp"][b])
            with torch.cuda.stream(d2h_stream):
                out_host[b].copy_(douts[b], non_blocking=True)
                ev["d2h"][b].record(d2h_stream)
        stream.wait_stream(d2h_stream)

    e2e_steps(4)
    torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_stream(stream)
    d2h_stream.wait_stream(stream)
    e2e_steps(Ke)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dist, device)
    if not torch.equal(out_host[(Ke - 1) % 2], out.cpu()):
        raise SystemExit("end-to-end output differs from the device-resident run")

    ms_step = elapsed_ms / K
    value = whole_job_value(world, work["cache_bytes"], ms_step)
    e2e_value = whole_job_value(world, work["cache_bytes"], e2e_ms / Ke)
    info = plan.info
    kname = {M.MLA_KERNEL_TCGEN05: "tcgen05"}.get(
        info.kernel, "simt")
    dec_s = statistics.mean(decode_ms) * 1e-3
    hbm_peak = peaks["hbm_gbs"]
    if kname.startswith("tcgen05") and wl.dtype == "fp8":
        # e4m3 / e5m2 MMAs: the fp8 dense rate is twice bf16's (nominal ratio);
        # the two-term operand splits execute 2x the algorithmic FLOPs there
        flop_peak = 2 * peaks["bf16_tflops"]
        flop_kind = "fp8 tensor = 2 x measured bf16"
    elif kname.startswith("tcgen05"):
        flop_peak = peaks["bf16_tflops"]
        flop_kind = "bf16 tensor"
    else:
        # CUDA-core fp32 FMA: 148 SMs x 128 lanes x 2 flops x max SM clock
        flop_peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        flop_kind = "fp32 FMA (ALU)"
    t_bytes = work["decode_bytes"] / (hbm_peak * 1e9)
    t_flops = work["decode_flops"] / (flop_peak * 1e12)
    if t_bytes >= t_flops:
        roof = {"bound": "hbm", "achieved": work["decode_bytes"] / dec_s / 1e9, "peak": hbm_peak,
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor" if kname.startswith("tcgen05") else "alu",
                "achieved": work["decode_flops"] / dec_s / 1e12, "peak": flop_peak,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(wl.name, kname, wl.dtype)
    roof["kernel"] = f"decode_{kname}"
    roof["peak_source"] = f"{peaks_kind} ({flop_kind} for FLOPs)"
    roof["decode_us"] = dec_s * 1e6
    roof["decode_launches_timed"] = Kd
    fp8_dec = work["decode_flops"] if wl.dtype == "fp8" else 0
    step_roof_s = max(work["step_bytes"] / (hbm_peak * 1e9),
                      (work["step_flops"] - fp8_dec) / (peaks["bf16_tflops"] * 1e12)
                      + fp8_dec / (2 * peaks["bf16_tflops"] * 1e12))

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "batch": B, "heads": wl.heads, "q_len": wl.q_len,
                   "context": wl.context, "latent_rank": wl.latent_rank,
                   "rope_dim": wl.rope_dim, "nope_dim": wl.nope_dim, "v_dim": wl.v_dim,
                   "latent_shards": wl.latent_shards, "page_size": wl.page_size,
                   "kernel": kname, "workers": info.num_workers,
                   "parallelism": (f"tpla: {world // tp} groups x {tp} latent shards, all-reduce"
                                   if tp > 1 and dist else
                                   f"one latent shard of {tp} (the per-GPU work of TPLA across GPUs)"
                                   if tp > 1 else f"replicas{world}" if world > 1 else "single"),
                   "l2": f"inputs larger than L2 (cache {work['cache_bytes'] / 1e9:.2f} GB)"},
        "us_per_step": ms_step * 1e3,
        "tflops": work["step_flops"] / (ms_step * 1e-3) / 1e12,
        "step_roofline_us": step_roof_s * 1e6,
        "step_roofline_frac": step_roof_s / (ms_step * 1e-3),
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "us_per_step": e2e_ms / Ke * 1e3, "steps": Ke,
                "pipeline": "2 buffer sets; H2D and D2H on their own streams overlap compute"},
        "gpu_launches": info.launches_per_run * K,
        "clocks": sampler.summary(w0, w_head),
    }
    if args.blasst is not None:
        # skip counters of the last step (every step of a plan makes the same decisions)
        skipped, groups = plan.skip_counts()
        line["blasst"] = {"skip_log2": args.blasst, "skipped_groups": skipped, "groups": groups,
                          "sparsity": skipped / max(1, groups),
                          "note": "threshold skipping: the result is the attention over the kept key groups"}
        line["config"]["kernel"] += "+threshold_skipping"

    if rank == 0 and world == 1 and tp == 1 and not args.no_cpu_baseline:
        # the oracle as it stands on the host cores, bounded sample; its sampled
        # outputs double as a parity spot check of this run's GPU output
        # seeded (sequence, head) pairs at full length until about
        # --cpu-seconds of oracle work have been spent
        rng = random.Random(12345)
        order = [(0, 0), (B - 1, wl.heads - 1)] + [
            (rng.randrange(B), rng.randrange(wl.heads)) for _ in range(4 * B * wl.heads)]
        pairs, outs, dt = [], [], 0.0
        for pr in order:
            if dt >= args.cpu_seconds or len(pairs) >= B * wl.heads:
                break
            if pr in pairs:
                continue
            t1, o = time_oracle_sample(wl, inputs, [pr], 0)
            pairs.append(pr)
            outs.extend(o)
            dt += t1
        done = sum(lens[b] for b, _ in pairs)
        frac = done / (sum(lens) * wl.heads)
        line["cpu_baseline"] = {
            "value": work["cache_bytes"] * frac / dt / 1e9, "unit": "GB/s",
            "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{len(pairs)} seeded (sequence, head) pairs at full length, fp64 numpy, "
                      f"scaled by their share of the step's (token x head) work; {dt:.1f} s"}
        line["parity_sample"] = compare_sample(out.cpu(), outs, pairs, wl.dtype)
    emit(line, rank)
    plan.close()
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
