#!/usr/bin/env python
"""Benchmark of the flex-attention hot path on B200.

One step = one flex forward over the long-context workload (B=2, H=Hkv=32,
S=8192, D=128, bf16, no_mod) followed by one decode over the dynamic KV cache
workload (B=16, H=Hkv=32, cap=8192, D=128, f16, kv_len ~ U[1, 8192], 10% -inf
additive mask).  Inputs are seeded synthetic tensors made on the device; every
input is larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun every rank runs the same workload
on its own GPU (independent replicas, weak scaling; no collective in the data
path) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "flex-attn fwd TFLOPS (B2 H32 D128 S8192 bf16); decode KV-read HBM GB/s"
FWD = dict(B=2, H=32, Hkv=32, S=8192, D=128, sigma=0.5, seed=4000)
DEC = dict(B=16, H=32, Hkv=32, cap=8192, D=128, scale=0.08837890625, seed=3032, mask_p=0.1)
# FlyDSL flex_attention on MI300X, no_mod, B=2 H=32 D=128 S=8192 (context, other hardware)
PAGES_NO_MOD_8192_TFLOPS = 470.1
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# dram read+write bytes per launch from ncu, keyed by the hash of the kernel sources
# they were measured on (a changed kernel reports null until it is captured again)
MEASURED_TRAFFIC = {
    # flex_fwd_kernel<128,bf16,none,none> (one CTA per unit), B2 H32 S8192 D128:
    # 402,722,816 B read + 114,174,720 B written (profiles/flex_fwd_kernel_bf16_nomod_S8192.md)
    "35374352ecfe85fe": 516897536,
}
MEASURED_DECODE_TRAFFIC = {
    # decode_split_kernel<128,f16,1,128>, B16 H32 Hkv32 cap8192, the bench's lengths and
    # mask: 868,650,240 B read + 5,617,152 B written
    # (profiles/decode_split_kernel_f16_hkv32_bench.md)
    "c56b25081c3bff63": 874267392,
}
# the forward kernel's sources: the roofline traffic below belongs to that kernel
KERNEL_SOURCES = ["attention_flex_attn_b200/csrc/flex_fwd_sm100.cuh",
                  "attention_flex_attn_b200/csrc/ptx_sm100.cuh",
                  "attention_flex_attn_b200/csrc/mask_rules.cuh"]
DECODE_SOURCES = ["attention_flex_attn_b200/csrc/flex_decode.cuh",
                  "attention_flex_attn_b200/csrc/flex_decode_launch.cu",
                  "attention_flex_attn_b200/csrc/ptx_sm100.cuh"]


def kernel_hash(sources=None) -> str:
    h = hashlib.sha256()
    for f in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def fwd_flops(B, H, Sq, Skv, D):
    return 4.0 * B * H * Sq * Skv * D


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings (every rank gets the result).  Ranks run
    independent replicas, so the job takes as long as its slowest rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(world, flops_per_rank, seconds):
    """Whole-job throughput of `world` replicas that each did flops_per_rank in `seconds`
    (the max over ranks)."""
    return world * flops_per_rank / seconds / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"]))}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0), "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]), "reasons": reasons,
                "samples": len(rows)}


def make_inputs(dev):
    import torch
    import synth
    f = FWD
    q, k, v = synth.qkv(f["B"], f["H"], f["Hkv"], f["S"], f["S"], f["D"], seed=f["seed"], sigma=f["sigma"],
                        device=dev)
    d = DEC
    qd = synth.normal_tensor((d["B"], d["H"], 1, d["D"]), d["seed"] * 8 + 1, dtype="f16", device=dev)
    kc = synth.normal_tensor((d["B"], d["Hkv"], d["cap"], d["D"]), d["seed"] * 8 + 2, dtype="f16", device=dev)
    vc = synth.normal_tensor((d["B"], d["Hkv"], d["cap"], d["D"]), d["seed"] * 8 + 3, dtype="f16", device=dev)
    lens = synth.kv_lengths(d["B"], d["cap"], d["seed"] * 8 + 4).to(dev)
    mask = synth.bernoulli_neg_inf_mask((d["B"], d["H"], 1, d["cap"]), d["mask_p"], d["seed"] * 8 + 5,
                                        dtype="f16").to(dev)
    return (q, k, v), (qd, kc, vc, lens, mask)


def decode_bytes(lens, H, Hkv, D, with_mask):
    """Algorithmic bytes of one decode: K and V rows read for every valid position,
    mask entries for valid positions, Q read, O (f16) and LSE (fp32) written."""
    tot = int(sum(int(x) for x in lens))
    b = tot * Hkv * D * 2 * 2
    if with_mask:
        b += tot * H * 2
    B = len(lens)
    b += B * H * D * 2 * 2 + B * H * 4
    return b


def cpu_oracle_sample(q, k, v, target_s=15.0):
    """Times the fp64 oracle on a bounded row sample of the forward workload."""
    import numpy as np
    import oracle
    B, H, S, D = q.shape
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    threads = oracle.default_threads()
    rng = np.random.default_rng(0)
    n = max(threads, 8)
    rows = np.sort(rng.choice(B * H * S, size=n, replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    oracle.fwd(qc, kc, vc, scale=1 / math.sqrt(D), rows=rows, threads=threads)
    dt = time.perf_counter() - t0
    n2 = int(min(B * H * S, max(n, n * target_s / max(dt, 1e-3))))
    rows = np.sort(rng.choice(B * H * S, size=n2, replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    oracle.fwd(qc, kc, vc, scale=1 / math.sqrt(D), rows=rows, threads=threads)
    dt = time.perf_counter() - t0
    flops = 4.0 * n2 * S * D
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": f"{n2} random query rows of the B2 H32 S8192 D128 no_mod forward (8192 keys each), "
                      f"fp64, {dt:.1f} s"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: bounded row samples on the host cores."""
    import numpy as np
    import torch
    import oracle
    import synth
    if rank != 0:
        return 0
    f = FWD
    q, k, v = synth.qkv(f["B"], f["H"], f["Hkv"], f["S"], f["S"], f["D"], seed=f["seed"], sigma=f["sigma"])
    B, H, S, D = q.shape
    threads = oracle.default_threads()
    rng = np.random.default_rng(1)
    probe = np.sort(rng.choice(B * H * S, size=max(threads, 8), replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    oracle.fwd(q, k, v, scale=1 / math.sqrt(D), rows=probe, threads=threads)
    per_row = (time.perf_counter() - t0) / probe.size
    budget = args.ref_seconds / (args.steps + args.warmup)
    n = int(max(threads, min(B * H * S, budget / max(per_row, 1e-6))))
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(B * H * S, size=n, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.fwd(q, k, v, scale=1 / math.sqrt(D), rows=rows, threads=threads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    dt = sum(times)
    flops = 4.0 * n * S * D * len(times)
    val = flops / dt / 1e12
    line = {"metric": METRIC, "value": val, "unit": "TFLOPS", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "flex fwd B2 H32 Hkv32 S8192 D128 no_mod, oracle row sample per step",
                       "rows_per_step": n},
            "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                             "sample": f"{n} random query rows per step (8192 keys each), fp64"},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="reference arm: host seconds of oracle work over all warm-up and timed steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the per-case and e2e measurements")
    ap.add_argument("--profile", choices=["fwd", "fwd8192", "fwd_blocks", "bwd", "fp8", "decode", "decode_bench"],
                    default=None,
                    help="run only a few launches of one kernel (for ncu captures) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.profile:
        return profile_case(args.profile)

    import torch
    import torch.distributed as dist
    import attention_flex_attn_b200 as fa

    fa.load_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    (q, k, v), (qd, kc, vc, lens, mask) = make_inputs(dev)
    f, d = FWD, DEC
    scale = 1.0 / math.sqrt(f["D"])
    o = torch.empty_like(q)
    lse = torch.empty((f["B"], f["H"], f["S"]), dtype=torch.float32, device=dev)
    od = torch.empty_like(qd)
    lsed = torch.empty((d["B"], d["H"], 1), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.decode_workspace_size(d["B"], d["H"], d["Hkv"], d["cap"], d["D"]), dtype=torch.uint8,
                     device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        fa.fwd(q, k, v, scale=scale, out=o, lse_out=lse)
        if ev is not None:
            ev[1].record()
        fa.decode(qd, kc, vc, lens, d["scale"], mask=mask, out=od, lse_out=lsed, workspace=ws)
        if ev is not None:
            ev[2].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.15)
    start.record()
    for i in range(args.steps):
        step(evs[i])
    end.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms, fwd_sum, dec_sum = max_over_ranks([total_ms, sum(fwd_ms), sum(dec_ms)], device=dev)
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the timed steps")

    flops = fwd_flops(f["B"], f["H"], f["S"], f["S"], f["D"])
    fwd_avg_s = fwd_sum / args.steps / 1e3
    dec_avg_s = dec_sum / args.steps / 1e3
    dbytes = decode_bytes(lens.tolist(), d["H"], d["Hkv"], d["D"], True)
    value = whole_job_tflops(world, flops, fwd_avg_s)  # max-over-ranks time
    peaks, peak_kind = load_peaks()
    achieved = flops / fwd_avg_s / 1e12
    traffic = MEASURED_TRAFFIC.get(kernel_hash())

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": value / world / PAGES_NO_MOD_8192_TFLOPS,
        "vs_baseline_ref": "FlyDSL flex_attention no_mod on MI300X, 470.1 TFLOPS (other hardware, context)",
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "flex fwd B2 H32 Hkv32 S8192 D128 bf16 no_mod + decode B16 H32 Hkv32 cap8192 "
                               "D128 f16 kv_len~U[1,8192] mask10%",
                   "global_batch": f["B"] * world, "seq_len": f["S"], "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (forward Q/K/V 384 MiB, decode caches 2 GiB); no flush"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 burst", "kernel": "flex_fwd_kernel<128,bf16,none,none>"},
        "decode": {"gbs": dbytes / dec_avg_s / 1e9, "ms": dec_avg_s * 1e3, "bytes": dbytes,
                   "roofline": {"bound": "hbm", "achieved": dbytes / dec_avg_s / 1e9, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": dbytes / dec_avg_s / 1e9 / peaks["hbm_gbs"],
                                "traffic": MEASURED_DECODE_TRAFFIC.get(kernel_hash(DECODE_SOURCES)),
                                "peak_source": peak_kind, "kernel": "decode_split_kernel<128,f16,1,128>"}},
        "fwd_ms": fwd_avg_s * 1e3,
        "fwd_stats": _spread(fwd_ms), "decode_stats": _spread(dec_ms),
        "protocol": "headline step: per-step CUDA events over the K timed steps; cases: "
                    f"{PROTOCOL['warmup']} warm-up, {PROTOCOL['samples']} samples x {PROTOCOL['iters']} iterations",
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
        "kernel_hash": kernel_hash(),
    }

    if not args.no_extras:
        line["cases"] = per_case(fa, q, k, v, scale, o, lse, args)
        line["decode_cases"] = decode_cases(fa, dev, args)
        line["e2e"] = e2e(fa, q, k, v, scale, args, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(q, k, v)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# The pages' timing protocol (FlyDSL PR 931, Performance Report header): 10 warm-up runs,
# then 12 samples of 100 back-to-back iterations each; mean +- std over the samples.
PROTOCOL = dict(warmup=10, samples=12, iters=100)


class NvmlClockPoll:
    """SM clock of this process's GPU, read through NVML by a background thread every
    10 ms while a measurement runs (median over the samples; None without NVML)."""

    def __init__(self):
        self.handle, self.vals, self.thread, self.stop_flag = None, [], None, False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
        except Exception:  # NVML missing or the device not found: no clock record
            self.handle = None

    def _run(self):
        while not self.stop_flag:
            try:
                self.vals.append(self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM))
            except Exception:
                return
            time.sleep(0.01)

    def __enter__(self):
        import threading
        if self.handle is not None:
            self.vals, self.stop_flag = [], False
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join()
            self.thread = None

    def median(self):
        return statistics.median(self.vals) if self.vals else None


_CLOCKS = None


def _time_stats(fn, samples=None, iters=None, warm=None):
    """Seconds per call: mean, std and coefficient of variation over `samples` samples,
    each the CUDA-event time of `iters` back-to-back calls divided by `iters`; plus the
    median SM clock seen meanwhile (long runs settle under the board's power cap)."""
    import torch
    global _CLOCKS
    if _CLOCKS is None:
        _CLOCKS = NvmlClockPoll()
    samples = samples or PROTOCOL["samples"]
    iters = iters or PROTOCOL["iters"]
    warm = PROTOCOL["warmup"] if warm is None else warm
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(samples + 1)]
    with _CLOCKS:
        ev[0].record()
        for s in range(samples):
            for _ in range(iters):
                fn()
            ev[s + 1].record()
        torch.cuda.synchronize()
    per = [ev[s].elapsed_time(ev[s + 1]) / iters / 1e3 for s in range(samples)]
    mean = statistics.fmean(per)
    std = statistics.stdev(per) if len(per) > 1 else 0.0
    return {"mean": mean, "std": std, "cv_pct": 100.0 * std / mean if mean > 0 else 0.0, "samples": samples,
            "iters": iters, "sm_mhz": _CLOCKS.median(), "min_us": min(per) * 1e6}


def _case_row(st, flops=None, key="tflops"):
    """A per-case row: time in us with its spread, and TFLOPS from the mean time."""
    row = {"us": st["mean"] * 1e6, "std_us": st["std"] * 1e6, "cv_pct": st["cv_pct"], "min_us": st["min_us"],
           "sm_mhz": st["sm_mhz"]}
    if flops is not None:
        row[key] = flops / st["mean"] / 1e12
    return row


def _spread(ms):
    """mean, std and CV% of per-step times in ms (this rank's steps)."""
    mean = statistics.fmean(ms)
    std = statistics.stdev(ms) if len(ms) > 1 else 0.0
    return {"mean_ms": mean, "std_ms": std, "cv_pct": 100.0 * std / mean if mean > 0 else 0.0, "steps": len(ms)}


def per_case(fa, q, k, v, scale, o, lse, args):
    """TFLOPS of the other hook cases on the same inputs (BASELINE convention: causal halved)."""
    B, H, S, D = q.shape
    dense = fwd_flops(B, H, S, S, D)
    W = 1024
    useful_window = 4.0 * D * B * H * (W * (W + 1) // 2 + (S - W) * W)
    cases = {"no_mod": dict(), "alibi": dict(score_mod="alibi"),
             "sliding_window_1024": dict(mask_mod="sliding_window", window=W),
             "causal_via_mask": dict(mask_mod="causal"), "causal_fast": dict(mask_mod="causal_fast")}
    out = {}
    for name, mods in cases.items():
        st = _time_stats(lambda: fa.fwd(q, k, v, scale=scale, out=o, lse_out=lse, **mods))
        t = st["mean"]
        causal = "causal" in name
        out[name] = _case_row(st, dense * (0.5 if causal else 1.0))
        out[name]["tflops_dense_equiv"] = dense / t / 1e12
        if name.startswith("sliding"):
            out[name]["tflops_useful"] = useful_window / t / 1e12
    out.update(mha2048_cases(fa))
    out.update(block_cases(fa, q, k, v, scale, o, lse))
    out.update(captured_cases(fa, q, k, v, scale, o, lse))
    out.update(bwd_cases(fa, q, k, v, scale))
    out.update(fp8_cases(fa, q, k, v, scale))
    return out


def mha2048_cases(fa):
    """The MHA configuration at S=2048 (B2 H32 D128 bf16, N(0, 1) inputs, scale 1/sqrt(128)):
    no_mod, alibi, sliding window 256 (causal), causal via mask_mod, causal=True.  These
    inputs (96 MiB) fit in L2, so iterations run L2-warm; the kernel is tensor-bound."""
    import torch
    import synth
    dev = torch.device("cuda")
    B, H, S, D = 2, 32, 2048, 128
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=synth.case_seed(1, 0), device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    dense = fwd_flops(B, H, S, S, D)
    W = 256
    useful_window = 4.0 * D * B * H * (W * (W + 1) // 2 + (S - W) * W)
    cases = {"s2048_no_mod": dict(), "s2048_alibi": dict(score_mod="alibi"),
             "s2048_sliding_window_256": dict(mask_mod="sliding_window", window=W),
             "s2048_causal_via_mask": dict(mask_mod="causal"), "s2048_causal_fast": dict(mask_mod="causal_fast")}
    out = {}
    for name, mods in cases.items():
        st = _time_stats(lambda: fa.fwd(q, k, v, out=o, lse_out=lse, **mods))
        if "sliding" in name:
            out[name] = _case_row(st, useful_window, "tflops_useful")
        else:
            out[name] = _case_row(st, dense * (0.5 if "causal" in name else 1.0))
        out[name]["l2"] = "warm"
    return out


def fp8_cases(fa, q, k, v, scale):
    """8-bit forward (flex_attn_fwd_fp8) on the forward inputs rounded to e4m3 (descales 1),
    including its V transpose pre-pass; TFLOPS as for the 16-bit forward."""
    import torch
    B, H, S, D = q.shape
    q8, k8, v8 = (t.float().to(torch.float8_e4m3fn) for t in (q, k, v))
    ws = torch.empty(fa.load_library().flex_attn_fwd_fp8_workspace_size(B, k.shape[1], S, D), dtype=torch.uint8,
                     device=q.device)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    res = {}
    for name, mods in (("fp8_no_mod", {}), ("fp8_causal", dict(mask_mod="causal"))):
        st = _time_stats(lambda: fa.fwd_fp8(q8, k8, v8, scale=scale, out=o, lse_out=lse, workspace=ws, **mods))
        res[name] = _case_row(st, fwd_flops(B, H, S, S, D) * (0.5 if "causal" in name else 1.0))
    return res


def bwd_cases(fa, q, k, v, scale):
    """Backward (flex_attn_bwd: prep + dQ + dK/dV launches) on the forward inputs, with
    dO ~ N(0, 1) (seed 4103): TFLOPS count the five algorithmic products of the backward,
    10 * B * H * Sq * Skv * D (halved for causal), not the two the kernels recompute."""
    import torch
    import synth
    B, H, S, D = q.shape
    res = {}
    dout = synth.normal_tensor(tuple(q.shape), 4103, dtype="bf16", device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.bwd_workspace_size(B, H, S), dtype=torch.uint8, device=q.device)
    for name, mods in (("bwd_no_mod", {}), ("bwd_causal", dict(mask_mod="causal"))):
        o, lse = fa.fwd(q, k, v, scale=scale, **mods)
        st = _time_stats(lambda: fa.bwd(q, k, v, o, lse, dout, scale=scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                                        **mods))
        res[name] = _case_row(st, 2.5 * fwd_flops(B, H, S, S, D) * (0.5 if "causal" in name else 1.0))
    return res


def captured_cases(fa, q, k, v, scale, o, lse):
    """Tensor-capturing mods on the forward inputs: alibi with a captured slope tensor
    (TFLOPS as no_mod), and packed documents whose boundaries fall off the 128 grid
    (lengths 200..3000, per-batch draws, seed 4102), plain and causal; useful TFLOPS =
    4 * D * kept pairs."""
    import numpy as np
    import torch
    B, H, S, D = q.shape
    dev = q.device
    res = {}
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32, device=dev)
    st = _time_stats(lambda: fa.fwd(q, k, v, scale=scale, score_mod="alibi", alibi_slopes=slopes, out=o,
                                    lse_out=lse))
    res["alibi_slope_tensor"] = _case_row(st, fwd_flops(B, H, S, S, D))
    rng = np.random.default_rng(4102)
    bounds = []
    for _ in range(B):
        cuts, pos = [0], 0
        while pos < S:
            pos = min(S, pos + int(rng.integers(200, 3001)))
            cuts.append(pos)
        bounds.append(cuts)
    n = max(len(c) for c in bounds)
    off = np.array([c + [S] * (n - len(c)) for c in bounds], np.int32)  # repeats = empty documents
    doff = torch.from_numpy(off).to(dev)
    for mask in ("document", "document_causal"):
        st = _time_stats(lambda: fa.fwd(q, k, v, scale=scale, mask_mod=mask, doc_offsets=doff, out=o, lse_out=lse))
        pairs = 0.0
        for b in range(B):
            for a, e in zip(off[b, :-1], off[b, 1:]):
                L = float(e - a)
                pairs += L * (L + 1) / 2 if mask == "document_causal" else L * L
        res[f"{mask}_packed"] = _case_row(st, 4.0 * D * H * pairs, "tflops_useful")
        res[f"{mask}_packed"]["documents"] = [len(c) - 1 for c in bounds]
    return res


def block_lists(sel):
    """[B, H, nq, nk] boolean block selection -> (counts, indices) int32, selected first."""
    import numpy as np
    num = sel.sum(-1).astype(np.int32)
    idx = np.argsort(~sel, axis=-1, kind="stable").astype(np.int32)
    return num, idx


def block_cases(fa, q, k, v, scale, o, lse):
    """Block-mask forward (flex_attn_fwd_block_sparse) on the forward inputs: causal given
    as lists (diagonal blocks partial, the rest full); causal attention inside documents
    of 4..24 whole tiles (useful TFLOPS = 4 * D * kept pairs); random per-head lists with
    half of the key blocks of every query tile full (TFLOPS count the listed blocks whole,
    4 * D * 128 * 128 per block).  The causal case halves the dense count as above."""
    import numpy as np
    import torch
    B, H, S, D = q.shape
    nq = nk = S // 128
    dev = q.device
    res = {}
    diag = np.eye(nq, nk, dtype=bool)
    below = np.tril(np.ones((nq, nk), dtype=bool), -1)
    kn, ki = block_lists(np.broadcast_to(diag, (1, 1, nq, nk)))
    fn, fi = block_lists(np.broadcast_to(below, (1, 1, nq, nk)))
    lists = [torch.from_numpy(a).to(dev) for a in (kn, ki, fn, fi)]
    st = _time_stats(lambda: fa.fwd_block_sparse(q, k, v, *lists, scale=scale, mask_mod="causal", out=o,
                                                 lse_out=lse))
    res["block_causal_lists"] = _case_row(st, 0.5 * fwd_flops(B, H, S, S, D))
    # documents of 4..24 whole tiles (512..3072 tokens), causal inside each document:
    # the diagonal block partial, earlier blocks of the same document full
    rng = np.random.default_rng(4101)
    starts, t = [], 0
    while t < nq:
        starts.append(t)
        t += int(rng.integers(4, 25))
    doc_start = np.zeros(nq, np.int64)
    for s0 in starts:
        doc_start[s0:] = s0
    part = np.zeros((1, 1, nq, nk), bool)
    full = np.zeros((1, 1, nq, nk), bool)
    for qt in range(nq):
        part[0, 0, qt, qt] = True
        full[0, 0, qt, doc_start[qt]:qt] = True
    kn, ki = block_lists(part)
    fn, fi = block_lists(full)
    lists = [torch.from_numpy(a).to(dev) for a in (kn, ki, fn, fi)]
    st = _time_stats(lambda: fa.fwd_block_sparse(q, k, v, *lists, scale=scale, mask_mod="causal", out=o,
                                                 lse_out=lse))
    pairs = 0.0  # kept (query, key) pairs per (b, h)
    ends = starts[1:] + [nq]
    for s0, e0 in zip(starts, ends):
        n = (e0 - s0) * 128
        pairs += n * (n + 1) / 2
    res["block_document_causal"] = _case_row(st, 4.0 * D * B * H * pairs, "tflops_useful")
    res["block_document_causal"]["documents"] = len(starts)
    rng = np.random.default_rng(4100)
    sel = rng.random((B, H, nq, nk)) < 0.5
    fn, fi = block_lists(sel)
    lists = [torch.from_numpy(a).to(dev) for a in (fn, fi)]
    st = _time_stats(lambda: fa.fwd_block_sparse(q, k, v, None, None, *lists, scale=scale, out=o, lse_out=lse))
    res["block_random_half_full"] = _case_row(st, 4.0 * D * 128 * 128 * float(sel.sum()))
    res["block_random_half_full"]["density"] = float(sel.mean())
    return res


def decode_cases(fa, dev, args):
    """Decode GB/s for the other rows of the decode configuration."""
    import torch
    import synth
    d = DEC
    res = {}
    for Hkv in (32, 8):
        for long_kv in (False, True):
            seed = 3300 + Hkv
            qd = synth.normal_tensor((d["B"], d["H"], 1, d["D"]), seed * 8 + 1, dtype="f16", device=dev)
            kc = synth.normal_tensor((d["B"], Hkv, d["cap"], d["D"]), seed * 8 + 2, dtype="f16", device=dev)
            vc = synth.normal_tensor((d["B"], Hkv, d["cap"], d["D"]), seed * 8 + 3, dtype="f16", device=dev)
            lens = (torch.full((d["B"],), d["cap"], dtype=torch.int32) if long_kv
                    else synth.kv_lengths(d["B"], d["cap"], seed * 8 + 4))
            mask = synth.bernoulli_neg_inf_mask((d["B"], d["H"], 1, d["cap"]), 0.1, seed * 8 + 5, dtype="f16").to(dev)
            lens_d = lens.to(dev)
            ws = torch.empty(fa.decode_workspace_size(d["B"], d["H"], Hkv, d["cap"], d["D"]), dtype=torch.uint8,
                             device=dev)
            for with_mask in (False, True):
                st = _time_stats(lambda: fa.decode(qd, kc, vc, lens_d, d["scale"], mask=mask if with_mask else None,
                                                   workspace=ws))
                by = decode_bytes(lens.tolist(), d["H"], Hkv, d["D"], with_mask)
                key = f"Hkv{Hkv}_{'long' if long_kv else 'random'}_{'mask' if with_mask else 'nomask'}"
                res[key] = _case_row(st, by * 1e3, "gbs")  # bytes / s / 1e9 = (by * 1e3) / s / 1e12
            del qd, kc, vc, mask, ws
    return res


def e2e(fa, q, k, v, scale, args, dev, world):
    """Forward through the public API with host buffers (flex_attn_fwd_host): Q/K/V read
    from pinned host memory and O/LSE written back to it, the library pipelining the
    copies of chunks of kv heads with the kernels; all inside the timed region, which
    ends once the results are in host memory."""
    import torch
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    hl = torch.empty(q.shape[:3], dtype=torch.float32).pin_memory()
    B, H, S, D = q.shape
    Hkv = k.shape[1]
    flops = fwd_flops(B, H, S, S, D)
    ws = torch.empty(fa.fwd_host_workspace_size(B, H, Hkv, S, S, D), dtype=torch.uint8, device=dev)

    def once():
        fa.fwd_host(hq, hk, hv, scale=scale, out=ho, lse_out=hl, workspace=ws, device=dev)

    # each call moves 512 MiB over PCIe: 4 samples of up to 5 calls
    st = _time_stats(once, samples=4, iters=max(2, min(args.steps, 5)), warm=2)
    t = st["mean"]
    h2d = 3 * q.numel() * q.element_size()
    d2h = q.numel() * q.element_size() + hl.numel() * 4
    return {"value": world * flops / t / 1e12, "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "cv_pct": st["cv_pct"],
            "what": "flex_attn_fwd_host: Q/K/V in pinned host memory, O/LSE back to it, copies pipelined "
                    "with the kernels by chunks of kv heads"}


def profile_case(which):
    """A few launches of one kernel on a case larger than L2 but a few GB at most:
    fwd = B2 H32 S4096 D128 bf16 no_mod (192 MiB of Q/K/V); fwd8192 = the full forward
    workload; fwd_blocks = the S4096 inputs with random per-head block lists, half of the
    key blocks of every query tile full; bwd = forward + backward at B2 H32 S4096 D128,
    no_mod then causal; fp8 = the S4096 inputs rounded to e4m3, 8-bit forward; decode = B16 H32 Hkv8 cap8192 all-full f16 with mask (537 MB of cache);
    decode_bench = the benchmark step's decode (B16 H32 Hkv32 cap8192, kv_len ~ U[1, 8192],
    10 % -inf mask; 2.1 GB of cache)."""
    import torch
    import synth
    import attention_flex_attn_b200 as fa
    fa.load_library()
    dev = torch.device("cuda", 0)
    if which == "fp8":
        S = 4096
        q, k, v = synth.qkv(2, 32, 32, S, S, 128, seed=4000, sigma=0.5, device=dev)
        q8, k8, v8 = (t.float().to(torch.float8_e4m3fn) for t in (q, k, v))
        for _ in range(4):
            fa.fwd_fp8(q8, k8, v8)
    elif which == "bwd":
        S = 4096
        q, k, v = synth.qkv(2, 32, 32, S, S, 128, seed=4000, sigma=0.5, device=dev)
        dout = synth.normal_tensor(tuple(q.shape), 4103, dtype="bf16", device=dev)
        for mask in ("none", "causal"):
            o, lse = fa.fwd(q, k, v, mask_mod=mask)
            fa.bwd(q, k, v, o, lse, dout, mask_mod=mask)
    elif which == "fwd_blocks":
        import numpy as np
        S, nq = 4096, 32
        q, k, v = synth.qkv(2, 32, 32, S, S, 128, seed=4000, sigma=0.5, device=dev)
        sel = np.random.default_rng(4100).random((2, 32, nq, nq)) < 0.5
        fn, fi = (torch.from_numpy(a).to(dev) for a in block_lists(sel))
        for _ in range(4):
            fa.fwd_block_sparse(q, k, v, None, None, fn, fi)
    elif which.startswith("fwd"):
        S = 8192 if which == "fwd8192" else 4096
        q, k, v = synth.qkv(2, 32, 32, S, S, 128, seed=4000, sigma=0.5, device=dev)
        for _ in range(4):
            fa.fwd(q, k, v)
    elif which == "decode_bench":
        _, (qd, kc, vc, lens, mask) = make_inputs(dev)
        ws = torch.empty(fa.decode_workspace_size(16, 32, 32, 8192, 128), dtype=torch.uint8, device=dev)
        for _ in range(4):
            fa.decode(qd, kc, vc, lens, DEC["scale"], mask=mask, workspace=ws)
    else:
        qd = synth.normal_tensor((16, 32, 1, 128), 11, dtype="f16", device=dev)
        kc = synth.normal_tensor((16, 8, 8192, 128), 12, dtype="f16", device=dev)
        vc = synth.normal_tensor((16, 8, 8192, 128), 13, dtype="f16", device=dev)
        lens = torch.full((16,), 8192, dtype=torch.int32, device=dev)
        mask = synth.bernoulli_neg_inf_mask((16, 32, 1, 8192), 0.1, 14, dtype="f16").to(dev)
        for _ in range(4):
            fa.decode(qd, kc, vc, lens, 0.08837890625, mask=mask)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    print(f"profile {which} ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
