#!/usr/bin/env python3
"""Benchmark: exact attention forward + backward on B200 through the fa C ABI.

One step = the whole hot path on one batch: fa_fwd, then fa_bwd's three kernels
(preprocess, main, dQ finish). Default workload: the sequence-length sweep's
N=4096 point (16k tokens, hidden 2048 -> B=4, H=16, d=128), non-causal, bf16 N(0,1)
inputs from the seeded generator. Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--seqlen N] [--headdim d]
                    [--causal] [--block-sparse [--block-density P]] [--dtype bf16|f16]
                    [--impl reference] [--sweep] [--density-sweep] [--decode NQ] [--forward-only]

Metric: fwd+bwd TFLOPS with FLOPs counted as 4*B*H*N^2*d for the forward (halved for causal,
scaled by block density for block-sparse) and 2.5x that for the backward.
--gpus N (under torchrun): every rank runs the same per-GPU workload on its own (b, h) shard
(no data-path collective: heads are independent), value = all ranks' FLOPs / max time.
--impl reference: the fp64 CPU oracle, timed on this host's cores on a bounded sample of
the same workload (whole heads), reported in the same metric.
"""
from __future__ import annotations

import argparse
import functools
import json
import math
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

TOKENS, HIDDEN = 16384, 2048
METRIC = "attention fwd / fwd+bwd TFLOPS and % of B200 dense BF16 peak vs seq len"
UNIT = "TFLOPS"


# ----------------------------------------------------------------------------- host logic
def workload(seqlen: int, headdim: int, causal: bool, block_sparse: bool, p_on: float = 0.25):
    if block_sparse:
        return dict(B=4, H=16, N=4096, d=64, causal=False, block_sparse=True, p_on=p_on,
                    name=f"block-sparse B=4 H=16 N=4096 d=64, 128x128 blocks Bernoulli({p_on:g}), diagonal on")
    B, H = TOKENS // seqlen, HIDDEN // headdim
    return dict(B=B, H=H, N=seqlen, d=headdim, causal=causal, block_sparse=False,
                name=f"seq-len sweep (16k tokens, hidden 2048): N={seqlen} d={headdim} B={B} H={H} "
                     f"{'causal' if causal else 'non-causal'}")


def fwd_flops(B, H, N, d, causal=False, density=1.0) -> float:
    f = 4.0 * B * H * N * N * d * density
    return f * 0.5 if causal else f


def shard_heads(BH: int, world: int, rank: int):
    """Contiguous (b, h) shard of a rank. Every head is independent, so no exchange is needed."""
    per = (BH + world - 1) // world
    lo = min(BH, rank * per)
    return lo, min(BH, lo + per)


def reduce_max(value: float, dist_on: bool, device=None) -> float:
    """Max over ranks (timing convention: the slowest rank defines the step time)."""
    if not dist_on:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def kernel_source_hash() -> str:
    """Hash of the backward kernel's code (its source and the PTX wrappers) with comments and
    whitespace removed, so that a comment edit does not retire a traffic record."""
    import hashlib
    import re
    m = hashlib.sha256()
    for f in ("exact_attention_110_b200/csrc/fa_bwd.cu", "exact_attention_110_b200/csrc/ptx.cuh"):
        text = (ROOT / f).read_text()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)  # block comments
        text = re.sub(r"//[^\n]*", " ", text)                 # line comments
        m.update(" ".join(text.split()).encode())
    return m.hexdigest()[:16]


def recorded_traffic(key: str):
    """DRAM bytes per launch from the last ncu capture, or None if the kernel changed since."""
    tfile = ROOT / "profiles" / "traffic.json"
    if not tfile.exists():
        return None
    rec = json.loads(tfile.read_text()).get(key)
    if not rec or rec.get("source_hash") != kernel_source_hash():
        return None
    return rec["bytes"]


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return dict(bf16_tflops=float(d["bf16_tflops"]), bf16_tflops_sustained=float(d["bf16_tflops_sustained"]),
                    hbm_gbs=float(d["hbm_gbs"]), source="measured")
    return dict(bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, hbm_gbs=6650.0, source="fallback")


def physical_gpu(local_rank: int) -> str:
    """nvidia-smi index (or UUID) of this rank's GPU, honouring CUDA_VISIBLE_DEVICES."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.proc = None
        self.gpu_index = gpu_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [ln.split(", ") for ln in (self.out or "").strip().splitlines() if ln.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_sample(wl, nheads: int, seed: int, dtype: str = "bf16"):
    """Times the fp64 oracle (fwd + bwd) on `nheads` whole heads of the workload."""
    import numpy as np
    import oracle
    import synth
    B, H, N, d = wl["B"], wl["H"], wl["N"], wl["d"]
    mask = synth.block_mask_for(N, p=wl.get("p_on", 0.25)) if wl["block_sparse"] else None
    n = nheads * N * d
    q, k, v, do = (synth.bits_to_f32(synth.normal_bits(seed + i, n, dtype), dtype).astype(np.float64)
                   .reshape(1, nheads, N, d) for i in range(4))
    scale = 1.0 / math.sqrt(d)
    t0 = time.perf_counter()
    oracle.attention_fwd(q, k, v, scale, causal=wl["causal"], mask=mask)
    oracle.attention_bwd(q, k, v, do, scale, causal=wl["causal"], mask=mask)
    dt = time.perf_counter() - t0
    density = float(mask.mean()) if mask is not None else 1.0
    flops = 3.5 * fwd_flops(1, nheads, N, d, wl["causal"], density)
    return flops, dt, oracle.num_threads()


def heads_for_seconds(wl, target_s: float, rate_gflops: float = 50.0) -> int:
    per_head = 3.5 * fwd_flops(1, 1, wl["N"], wl["d"], wl["causal"],
                               wl.get("p_on", 0.25) + 0.03 if wl["block_sparse"] else 1.0)
    return max(1, min(wl["B"] * wl["H"], int(target_s * rate_gflops * 1e9 / per_head)))


def run_reference(args, wl, rank, world):
    if rank != 0:
        return 0
    nh = heads_for_seconds(wl, 2.0)
    for _ in range(args.warmup):
        oracle_sample(wl, nh, 1000, args.dtype)
    tot_f, tot_t, cores = 0.0, 0.0, 1
    for s in range(args.steps):
        f, t, cores = oracle_sample(wl, nh, 2000 + 10 * s, args.dtype)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    sample = f"{nh} whole head(s) of {wl['N']}x{wl['d']} per step (fwd+bwd, fp64), of {wl['B'] * wl['H']} heads"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl["name"]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def fwd_kernel_name(d: int, nq: int) -> str:
    """The forward kernel the library launches for nq query rows at head dimension d (a label
    for the roofline object; the choice itself is made in the library)."""
    nb = -(-nq // 128)
    if d == 256 or (d == 128 and nb == 1):
        return "fa_fwd_kernel (one tile per CTA)"
    if nb <= 8:
        return "fa_fwd_solo_kernel" + (" (query rows copied per lane quarter)" if d == 64 and nq <= 64 else "")
    return "fa_fwd_kernel"


# ----------------------------------------------------------------------------- decode arm
def run_decode(args, rank, world, local_rank, dist_on):
    """Decode-shaped forward: args.decode queries per head against --seqlen keys, B=8, H=16
    (hidden 2048 at d=128), split over the key range and merged. HBM-bound: the metric is the
    K/V bytes read per second against the measured HBM copy bandwidth."""
    import torch
    import exact_attention_110_b200 as fa
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, H, nq, nk, d = 8, HIDDEN // args.headdim, args.decode, args.seqlen, args.headdim
    seed = synth.BASE_SEED + 97 * rank
    q = synth.to_torch(_stream(seed + synth.SEED_Q, B * H * nq * d, args.dtype).reshape(B, H, nq, d), args.dtype, dev)
    k, v = (synth.to_torch(_stream(seed + o, B * H * nk * d, args.dtype).reshape(B, H, nk, d), args.dtype, dev)
            for o in (synth.SEED_K, synth.SEED_V))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, nq), device=dev, dtype=torch.float32)
    need = int(fa.library().fa_fwd_decode_workspace_bytes(B, H, nq, nk, d, 0))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fa.forward_decode(q, k, v, causal=args.causal, out=o, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    with ClockSampler(physical_gpu(local_rank)) as clk:
        time.sleep(0.3)
        start.record()
        for _ in range(args.steps):
            fa.forward_decode(q, k, v, causal=args.causal, out=o, lse=lse, workspace=ws)
        end.record()
        torch.cuda.synchronize()
    if fa.last_device_status(dev) != 0:
        raise RuntimeError("device wait timed out")
    ms = reduce_max(start.elapsed_time(end), dist_on, dev) / args.steps
    kv_bytes = 2 * B * H * nk * d * 2
    peaks = load_peaks()
    gbs = world * kv_bytes / (ms * 1e-3) / 1e9
    line = {"metric": "decode forward K/V read bandwidth", "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
            "config": {"workload": f"decode B={B} H={H} Nq={nq} Nk={nk} d={d} "
                                   f"{'causal' if args.causal else 'non-causal'}, split keys (library's choice)",
                       "workspace_bytes": need},
            "tflops": world * fwd_flops(B, H, 1, d) * nq * nk / (ms * 1e-3) / 1e12,
            "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / world / peaks["hbm_gbs"], "traffic": None, "kernel": fwd_kernel_name(d, nq)},
            "gpu_launches": args.steps * (2 if need > 0 else 1), "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_forward_only(args, wl, rank, world, local_rank, dist_on):
    """Forward pass alone on the sweep's workload. Metric: forward TFLOPS (4·N²·d per head,
    halved when causal) against the measured dense bf16 peak."""
    import torch
    import exact_attention_110_b200 as fa
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, H, N, d, causal = wl["B"], wl["H"], wl["N"], wl["d"], wl["causal"]
    seed = synth.BASE_SEED + 97 * rank
    q, k, v = (synth.to_torch(_stream(seed + o, B * H * N * d, args.dtype).reshape(B, H, N, d), args.dtype, dev)
               for o in (synth.SEED_Q, synth.SEED_K, synth.SEED_V))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    scale = 1.0 / math.sqrt(d)
    for _ in range(args.warmup):
        fa.forward(q, k, v, causal=causal, scale=scale, out=o, lse=lse)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    with ClockSampler(physical_gpu(local_rank)) as clk:
        time.sleep(0.3)
        start.record()
        for _ in range(args.steps):
            fa.forward(q, k, v, causal=causal, scale=scale, out=o, lse=lse)
        end.record()
        torch.cuda.synchronize()
    if fa.last_device_status(dev) != 0:
        raise RuntimeError("device wait timed out")
    ms = reduce_max(start.elapsed_time(end), dist_on, dev) / args.steps
    tflops = fwd_flops(B, H, N, d, causal) / (ms * 1e-3) / 1e12
    peaks = load_peaks()
    line = {"metric": "attention forward TFLOPS", "value": world * tflops, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
            "config": {"workload": wl["name"] + ", forward only", "B": B, "H": H, "N": N, "d": d,
                       "causal": causal},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops"], "traffic": None, "kernel": fwd_kernel_name(d, N)},
            "gpu_launches": args.steps, "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
@functools.lru_cache(maxsize=4)
def _stream(seed: int, n: int, dtype: str = "bf16"):
    """Seeded N(0,1) bf16 (or fp16) bits (same bytes as synth.attention_inputs); every sweep
    point has the same element count, so the streams are generated once."""
    import synth
    return synth.normal_bits(seed, n, dtype)


SWEEP_POINTS = [(n, dd, c) for dd in (64, 128) for c in (False, True) for n in (512, 1024, 2048, 4096, 8192, 16384)]
# The other configurations the metric is quoted on (block-sparse: diagonal on, others Bernoulli(0.25)).
NAMED_CONFIGS = {
    "bert_large_shape": dict(B=16, H=16, N=512, d=64, causal=False, block_sparse=False),
    "gpt2_shape_causal": dict(B=8, H=12, N=1024, d=64, causal=True, block_sparse=False),
    "block_sparse": dict(B=4, H=16, N=4096, d=64, causal=False, block_sparse=True),
    # the same 16k tokens x hidden 2048 at head dimension 256
    "head_dim_256": dict(B=4, H=8, N=4096, d=256, causal=False, block_sparse=False),
    "head_dim_256_causal": dict(B=4, H=8, N=4096, d=256, causal=True, block_sparse=False),
}


def time_kernels(fa, t, shape, causal, mask, scale, steps, warmup, min_warm_s=0.0, min_timed_s=0.0):
    """Per-kernel CUDA-event times (ms, mean over the timed steps) of one fwd+bwd step on the
    views in `t` (q, k, v, do, o, dq, dk, dv of `shape`; lse; ws), after at least `warmup` untimed
    steps and `min_warm_s` seconds of them, and the whole-loop time per step. At least `steps`
    steps are timed, more when that takes under `min_timed_s` (short steps from an idle GPU
    would otherwise be timed while the clocks ramp up)."""
    import torch
    q, k, v, do, o, dq, dk, dv = (t[x] for x in ("q", "k", "v", "do", "o", "dq", "dk", "dv"))
    lse, ws = t["lse"], t["ws"]

    def step(evs=None):
        if evs is not None:
            evs[0].record()
        fa.forward(q, k, v, causal=causal, block_mask=mask, scale=scale, out=o, lse=lse)
        if evs is not None:
            evs[1].record()
        fa.bwd_preprocess(o, do, lse, scale=scale, workspace=ws)
        if evs is not None:
            evs[2].record()
        fa.bwd_main(q, k, v, do, ws, causal=causal, block_mask=mask, scale=scale, dk=dk, dv=dv)
        if evs is not None:
            evs[3].record()
        fa.bwd_dq_finish(ws, shape, q.device, dq=dq)
        if evs is not None:
            evs[4].record()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    n_warm, t0 = warmup, time.perf_counter()
    while time.perf_counter() - t0 < min_warm_s:
        step()
        torch.cuda.synchronize()
        n_warm += 1
    if min_warm_s > 0 and n_warm > warmup:
        per_step = (time.perf_counter() - t0) / (n_warm - warmup)
        steps = max(steps, math.ceil(min_timed_s / per_step))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for e in evs:
        step(e)
    end.record()
    torch.cuda.synchronize()
    k_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / steps for i in range(4)]
    return k_ms, start.elapsed_time(end) / steps


# Each sweep point: at least 10 ms of warm-up steps, then at least `--sweep-steps` steps and
# 10 ms timed (a point's step takes 0.2 to 8 ms): short steps are no longer timed while the
# clocks ramp up from idle, and long ones see about the load of the headline's timed region
# (30 + 20 ms put the N >= 4096 points under the power cap).
SWEEP_WARM_S, SWEEP_TIMED_S = 0.01, 0.01


def run_sweep(fa, dev, dtype, steps, warmup, peaks):
    """The metric's curve: every sequence-length sweep point (16k tokens, hidden 2048; N x d x
    causal) and the named configurations, each timed on its own with CUDA events. All sweep
    points have 16384 x 2048 elements per tensor, so one set of device buffers serves them all
    (viewed as [B, H, N, d]); the named configurations use prefixes of the same buffers."""
    import torch
    import synth
    n = TOKENS * HIDDEN
    base = {x: synth.to_torch(_stream(synth.BASE_SEED + off, n, dtype), dtype, dev)
            for x, off in (("q", synth.SEED_Q), ("k", synth.SEED_K), ("v", synth.SEED_V), ("do", synth.SEED_DO))}
    for x in ("o", "dq", "dk", "dv"):
        base[x] = torch.empty_like(base["q"])
    lse_all = torch.empty(n // 64, dtype=torch.float32, device=dev)
    ws_all = torch.empty(max(fa.bwd_workspace_bytes(TOKENS // N, HIDDEN // dd, N, dd) for N, dd, _ in SWEEP_POINTS),
                         dtype=torch.uint8, device=dev)

    def views(B, H, N, d):
        m = B * H * N * d
        t = {x: base[x][:m].view(B, H, N, d) for x in ("q", "k", "v", "do", "o", "dq", "dk", "dv")}
        t["lse"] = lse_all[:B * H * N].view(B, H, N)
        t["ws"] = ws_all
        return t

    def entry(B, H, N, d, causal, mask_np):
        time.sleep(0.25)  # each point starts from an idle GPU, as a burst measurement does
        mask = None if mask_np is None else torch.from_numpy(mask_np).to(dev)
        density = float(mask_np.mean()) if mask_np is not None else 1.0
        (f_ms, p_ms, m_ms, d_ms), step_ms = time_kernels(fa, views(B, H, N, d), (B, H, N, d), causal, mask,
                                                          1.0 / math.sqrt(d), steps, warmup, SWEEP_WARM_S,
                                                          SWEEP_TIMED_S)
        ff = fwd_flops(B, H, N, d, causal, density)
        fwd_t = ff / (f_ms * 1e-3) / 1e12
        fb_t = 3.5 * ff / (step_ms * 1e-3) / 1e12
        return {"B": B, "H": H, "N": N, "d": d, "causal": causal, "block_density": round(density, 4),
                "fwd_ms": round(f_ms, 4), "bwd_ms": round(p_ms + m_ms + d_ms, 4), "step_ms": round(step_ms, 4),
                "fwd_tflops": round(fwd_t, 1), "fwd_bwd_tflops": round(fb_t, 1),
                "bwd_main_tflops": round(2.5 * ff / (m_ms * 1e-3) / 1e12, 1),
                "pct_of_peak_fwd": round(100 * fwd_t / peaks["bf16_tflops"], 2),
                "pct_of_peak_fwd_bwd": round(100 * fb_t / peaks["bf16_tflops"], 2)}

    points = []
    for (N, d, c) in SWEEP_POINTS:
        points.append(entry(TOKENS // N, HIDDEN // d, N, d, c, None))
    named = {}
    for name, c in NAMED_CONFIGS.items():
        mask_np = synth.block_mask_for(c["N"]) if c["block_sparse"] else None
        named[name] = entry(c["B"], c["H"], c["N"], c["d"], c["causal"], mask_np)
    if fa.last_device_status(dev) != 0:
        raise RuntimeError("device wait timed out in the sweep")
    return points, named


def run_gpu(args, wl, rank, world, local_rank, dist_on):
    import numpy as np
    import torch
    import exact_attention_110_b200 as fa
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fa.library()
    B, H, N, d, causal = wl["B"], wl["H"], wl["N"], wl["d"], wl["causal"]
    shape = (B, H, N, d)
    seed = synth.BASE_SEED + 97 * rank
    offs = (synth.SEED_Q, synth.SEED_K, synth.SEED_V, synth.SEED_DO)
    q, k, v, do = (synth.to_torch(_stream(seed + o, B * H * N * d, args.dtype).reshape(B, H, N, d), args.dtype, dev)
                   for o in offs)
    mask_np = synth.block_mask_for(N, p=wl.get("p_on", 0.25)) if wl["block_sparse"] else None
    mask = None if mask_np is None else torch.from_numpy(mask_np).to(dev)
    density = float(mask_np.mean()) if mask_np is not None else 1.0
    scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)

    def step(evs=None):
        if evs is not None:
            evs[0].record()
        fa.forward(q, k, v, causal=causal, block_mask=mask, scale=scale, out=o, lse=lse)
        if evs is not None:
            evs[1].record()
        fa.bwd_preprocess(o, do, lse, scale=scale, workspace=ws)
        if evs is not None:
            evs[2].record()
        fa.bwd_main(q, k, v, do, ws, causal=causal, block_mask=mask, scale=scale, dk=dk, dv=dv)
        if evs is not None:
            evs[3].record()
        fa.bwd_dq_finish(ws, shape, dev, dq=dq)
        if evs is not None:
            evs[4].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.last_device_status(dev) != 0:
        raise RuntimeError("device wait timed out during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(physical_gpu(local_rank)) as clk:
        time.sleep(0.3)  # let the sampler start
        start.record()
        for s in range(args.steps):
            step(evs[s])
        end.record()
        torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    if fa.last_device_status(dev) != 0:
        raise RuntimeError("device wait timed out in the timed region")
    total_ms = reduce_max(start.elapsed_time(end), dist_on, dev)
    k_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i in range(4)]
    fwd_ms, pre_ms, main_ms, fin_ms = (reduce_max(x, dist_on, dev) for x in k_ms)
    ms = total_ms / args.steps
    f_fwd = fwd_flops(B, H, N, d, causal, density)
    value = world * 3.5 * f_fwd / (ms * 1e-3) / 1e12
    peaks = load_peaks()

    # ---- end to end through the public API with pinned host buffers
    # Every step copies its inputs (q, k, v, dO) in from pinned host memory and its results
    # (o, lse, dq, dk, dv) back out. Steps are pipelined over three streams with two sets of
    # device buffers, as a training loop would overlap its transfers: step k's compute runs while
    # step k+1's inputs arrive and step k-1's results leave; events order each buffer's reuse.
    e2e = None
    if not args.no_e2e:
        hin = [t.cpu().pin_memory() for t in (q, k, v, do)]
        hout = [torch.empty(shape, dtype=q.dtype).pin_memory() for _ in range(4)] + \
               [torch.empty((B, H, N), dtype=torch.float32).pin_memory()]
        din = [[torch.empty_like(t) for t in (q, k, v, do)] for _ in range(2)]
        dout = [[torch.empty_like(q) for _ in range(4)] + [torch.empty((B, H, N), device=dev, dtype=torch.float32)]
                for _ in range(2)]
        s_in, s_c, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_c = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        issued = [False, False]

        def e2e_step(i):
            b = i % 2
            xq, xk, xv, xdo = din[b]
            xo, xdq, xdk, xdv, xl = dout[b]
            with torch.cuda.stream(s_in):
                if issued[b]:
                    s_in.wait_event(ev_c[b])  # the compute two steps back has read these inputs
                for dst, src in zip(din[b], hin):
                    dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_c):
                s_c.wait_event(ev_in[b])
                if issued[b]:
                    s_c.wait_event(ev_out[b])  # the results two steps back have left
                fa.forward(xq, xk, xv, causal=causal, block_mask=mask, scale=scale, out=xo, lse=xl)
                fa.backward(xq, xk, xv, xo, xdo, xl, causal=causal, block_mask=mask, scale=scale, workspace=ws,
                            dq=xdq, dk=xdk, dv=xdv)
                ev_c[b].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[b])
                for dst, src in zip(hout, (xo, xdq, xdk, xdv, xl)):
                    dst.copy_(src, non_blocking=True)
                ev_out[b].record(s_out)
            issued[b] = True

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist_on:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0.record(s_in)
        for i in range(args.steps):
            e2e_step(i)
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_c)
        e1.record(s_out)
        torch.cuda.synchronize()
        if fa.last_device_status(dev) != 0:
            raise RuntimeError("device wait timed out in the end-to-end loop")
        e2e_ms = reduce_max(e0.elapsed_time(e1), dist_on, dev) / args.steps
        nb = B * H * N * d * 2
        e2e = {"value": world * 3.5 * f_fwd / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 4 * nb, "d2h_bytes_per_step": 4 * nb + B * H * N * 4,
               "ms_per_step": e2e_ms,
               "pipeline": "3 streams (copy in, compute, copy out), 2 device buffer sets, pinned host memory"}

    # ---- roofline of the dominant kernel (bwd main: 5 of the 7 matmuls of a step)
    main_flops = 2.5 * f_fwd
    achieved = main_flops / (main_ms * 1e-3) / 1e12
    traffic = recorded_traffic(f"bwd_main N={N} d={d} causal={int(causal)} bs={int(wl['block_sparse'])}"
                               + (f" p={wl['p_on']:g}" if wl["block_sparse"] and wl["p_on"] != 0.25 else "")
                               + ("" if args.dtype == "bf16" else f" {args.dtype}"))
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": traffic, "kernel": "fa_bwd_kernel",
                "peak_kind": f"bf16 dense burst ({peaks['source']})" + (
                    "; fp16 has the same nominal dense rate (ratio 1)" if args.dtype == "f16" else ""),
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]}

    kernels = {
        "fwd": {"ms": fwd_ms, "tflops": f_fwd / (fwd_ms * 1e-3) / 1e12},
        "bwd_preprocess": {"ms": pre_ms, "gbs": (4 * B * H * N * d + 8 * B * H * N + 4 * B * H * N * d + 4 * B * H * N)
                           / (pre_ms * 1e-3) / 1e9},
        "bwd_main": {"ms": main_ms, "tflops": achieved},
        "bwd_dq_finish": {"ms": fin_ms, "gbs": (4 * B * H * N * d + 2 * B * H * N * d) / (fin_ms * 1e-3) / 1e9},
    }
    bwd_ms = pre_ms + main_ms + fin_ms
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": args.dtype,
        "data": "synthetic",
        "config": {"workload": wl["name"], "B": B, "H": H, "N": N, "d": d, "causal": causal,
                   "block_density": density, "global_batch_heads": world * B * H,
                   "l2": "no flush: the step's tensors (q,k,v,o,do,dq,dk,dv = 8 x "
                         f"{B * H * N * d * 2 / 2**20:.0f} MiB) exceed the 126 MB L2",
                   "parallelism": f"dp{world} over (b,h) shards, no collective"},
        "fwd_tflops": world * f_fwd / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": world * 2.5 * f_fwd / (bwd_ms * 1e-3) / 1e12,
        "pct_of_peak_fwd_bwd": 100.0 * value / world / peaks["bf16_tflops"],
        "pct_of_peak_fwd": 100.0 * f_fwd / (fwd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "kernels": kernels,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": 4 * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_sweep:
        with ClockSampler(physical_gpu(local_rank)) as sclk:
            time.sleep(0.3)
            points, named = run_sweep(fa, dev, args.dtype, args.sweep_steps, args.warmup, peaks)
        line["sweep"] = {"unit": UNIT, "peak": peaks["bf16_tflops"],
                         "peak_kind": f"bf16 dense burst ({peaks['source']})",
                         "steps": args.sweep_steps, "warmup": args.warmup, "dtype": args.dtype,
                         "timing": f"per point: >= {args.warmup} warm-up steps and >= {SWEEP_WARM_S * 1e3:.0f} ms "
                                   f"of them, then >= {args.sweep_steps} steps and >= "
                                   f"{SWEEP_TIMED_S * 1e3:.0f} ms timed",
                         "workload": "16k tokens, hidden 2048: B = 16384/N, H = 2048/d, bf16 N(0,1); "
                                     "per-GPU figures on this rank",
                         "points": points, "configs": named, "clocks": sclk.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # one head first to measure this host's rate, then enough heads for ~12 s of oracle work
        f1, t1, _ = oracle_sample(wl, 1, 2999, args.dtype)
        nh = max(1, min(B * H, int(12.0 / max(t1, 1e-3))))
        f, t, cores = oracle_sample(wl, nh, 3000, args.dtype)
        line["cpu_baseline"] = {"value": f / t / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{nh} whole head(s) of {N}x{d} (fwd+bwd, fp64) of {B * H} heads; "
                                          f"{t:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--seqlen", type=int, default=4096)
    ap.add_argument("--headdim", type=int, default=128)
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--block-sparse", action="store_true")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the sequence-length curve (24 points + named configs) in the headline line")
    ap.add_argument("--sweep-steps", type=int, default=5, help="timed steps per point of that curve")
    ap.add_argument("--sweep", action="store_true", help="one JSON line per sweep point (N x d x causal)")
    ap.add_argument("--block-density", type=float, default=0.25,
                    help="with --block-sparse: probability that an off-diagonal 128x128 block is on")
    ap.add_argument("--density-sweep", action="store_true",
                    help="block-sparse config at densities 0.05..1: runtime should follow the blocks that are on")
    ap.add_argument("--decode", type=int, default=0, metavar="NQ",
                    help="decode-shaped forward: NQ queries per head against --seqlen keys (B=8)")
    ap.add_argument("--forward-only", action="store_true", help="time the forward alone")
    ap.add_argument("--dtype", choices=["bf16", "f16"], default="bf16",
                    help="element type of q, k, v, o, dO and the gradients (fp32 accumulation either way)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    if args.impl == "reference":
        wl = workload(args.seqlen, args.headdim, args.causal, args.block_sparse, args.block_density)
        return run_reference(args, wl, rank, world)
    if dist_on:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.decode > 0:
            return run_decode(args, rank, world, local_rank, dist_on)
        if args.forward_only:
            return run_forward_only(args, workload(args.seqlen, args.headdim, args.causal, False),
                                    rank, world, local_rank, dist_on)
        if args.density_sweep:
            args.no_cpu_baseline, args.no_e2e, args.no_sweep = True, True, True
            for p_on in (0.05, 0.1, 0.25, 0.5, 1.0):
                run_gpu(args, workload(args.seqlen, args.headdim, False, True, p_on), rank, world, local_rank, dist_on)
            return 0
        points = ([(n, dd, c) for dd in (64, 128) for c in (False, True) for n in (512, 1024, 2048, 4096, 8192, 16384)]
                  if args.sweep else [(args.seqlen, args.headdim, args.causal)])
        for (n, dd, c) in points:
            wl = workload(n, dd, c, args.block_sparse, args.block_density)
            if args.sweep:
                args.no_cpu_baseline, args.no_e2e, args.no_sweep = True, True, True
            run_gpu(args, wl, rank, world, local_rank, dist_on)
    finally:
        if dist_on:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
