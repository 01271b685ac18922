"""Benchmark of the VC-Attention forward (V-Smooth prep + ExpCast-FP8 attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mid_32k_d128] [--no-cpu-baseline]

One step is one pass of the whole hot path over the workload: V-Smooth prep
(k-means, regroup, K/V quantisation) and the attention forward, on inputs
resident in HBM.  The metric is attention TFLOPS, 4*B*H*N^2*d over the step
time.  Rank 0 prints one JSON line.

Multi-GPU (torchrun, one process per GPU): every (b, h) problem is
independent, so each rank runs its own copy of the workload with no data-path
collective (weak scaling); the step time is the max over ranks.

--impl reference times the CPU oracle (the only other implementation of the
method there is) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_fp8_attention_smooth_b200 import synth  # noqa: E402

BETA = 64
METRIC = "attn fwd TFLOPS (4*B*H*N^2*d/t) at N=32K, d=128; % of B200 FP8 tensor peak"
FP8_PER_BF16 = 2.0  # nominal dense fp8 : bf16 tensor ratio on B200


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def kernel_code_hash() -> str:
    """First 16 hex digits of sha256 over vc_attn.cu and vc_device.cuh with
    // comments and blank lines removed: the code the profiled kernel was
    built from, indifferent to edits of its comments."""
    import hashlib

    csrc = os.path.join(ROOT, "bit_fp8_attention_smooth_b200", "csrc")
    h = hashlib.sha256()
    for name in ("vc_attn.cu", "vc_device.cuh"):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            lines = (line.split("//", 1)[0].rstrip() for line in f.read().splitlines())
            h.update("\n".join(line for line in lines if line).encode())
    return h.hexdigest()[:16]


def attn_traffic_bytes(heads: int, kernel: str = "vc_attn_kernel", N=None, d=None, block=None):
    """DRAM bytes (read + write) of one attention-kernel launch over `heads`
    heads, from the ncu capture recorded in profiles/attn_traffic.json; None
    when there is no record for the kernel, its code has changed since the
    capture (the counters no longer apply), or the record names the shape it
    was captured on (N, d, block) and the launch's shape differs (the bytes a
    head grow with N)."""
    try:
        with open(os.path.join(ROOT, "profiles", "attn_traffic.json")) as f:
            rec = json.load(f).get(kernel)
        code = kernel_code_hash()
    except (OSError, ValueError):
        return None
    if not rec or rec.get("sources_sha256_16") != code:
        return None
    for key, val in (("N", N), ("d", d), ("block", block)):
        if key in rec and val is not None and int(rec[key]) != int(val):
            return None
    return int(rec["dram_bytes_per_head"]) * heads


# ----------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU oracle
def oracle_sample(w, rows: int, threads: int, smooth: bool = True):
    """Time the oracle (prep of one head + replay of `rows` query rows over all
    keys) and extrapolate to the per-head attention throughput in TFLOPS."""
    import oracle

    q, k, v = (synth.head_bits(w, t, 0, 0) for t in "qkv")
    sel = np.linspace(0, w.N - 1, rows).astype(np.int64)
    t0 = time.perf_counter()
    rf = resid_fmt_of(w)
    prep = oracle.prep_head(k, v, C=w.C, iters=w.iters, bk=w.block, smooth=smooth, resid_fmt=rf)
    t1 = time.perf_counter()
    oracle.forward_head(q, k, v, sel, C=w.C, iters=w.iters, bk=w.block, beta=BETA, smooth=smooth, resid_fmt=rf,
                        prep=prep, threads=threads)
    t2 = time.perf_counter()
    head_s = (t1 - t0) + (t2 - t1) * (w.N / rows)
    head_flops = 4.0 * float(w.N) ** 2 * w.d
    return dict(value=head_flops / head_s / 1e12, prep_s=t1 - t0, rows_s=t2 - t1, head_s=head_s)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------- arms
def run_reference(args, w):
    """The oracle as it stands, timed on the host cores.  One step is one
    bounded sample of the workload: the full prep of head 0 plus the replay of
    `--ref-rows` strided query rows over all keys.  ms_per_step is the measured
    time of that sample; value is the workload's attention flops over the time
    the sample extrapolates to (the head's prep plus all its rows, times the
    heads)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cores = cpu_cores()
    rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(w, max(8, rows // 8), cores, args.smooth)
    samples = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        samples.append(oracle_sample(w, rows, cores, args.smooth))
    wall = time.perf_counter() - t0
    head_s = statistics.median(r["head_s"] for r in samples)
    full_s = head_s * w.B * w.H
    value = w.attn_flops / full_s / 1e12
    sample = (f"head 0 of {w.name}: full k-means/regroup/quantise prep + replay of {rows} strided query rows "
              f"over all {w.N} keys; value extrapolates to all {w.N} rows of each of the {w.B * w.H} heads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 emulation of e4m3",
        "data": "synthetic", "config": config_of(w, args.smooth),
        "sample_s": {"prep": statistics.median(r["prep_s"] for r in samples),
                     "rows": statistics.median(r["rows_s"] for r in samples)},
        "extrapolated_head_s": head_s, "extrapolated_step_s": full_s,
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def resid_fmt_of(w) -> int:
    """1 for the 4-bit (NVFP4) residual workload, else 0 (E4M3)."""
    return 1 if w.resid_fmt == "nvfp4" else 0


def config_of(w, smooth: bool):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "C": w.C, "kmeans_iters": w.iters,
            "block": w.block, "beta": BETA, "v_smooth": smooth,
            "residual": "nvfp4 (E2M1 + UE4M3 per 16)" if resid_fmt_of(w) else "e4m3",
            "l2": l2_note(w)}


def l2_note(w) -> str:
    gb = 3 * w.B * w.H * w.N * w.d * 2 / 1e9
    if gb > 0.126:
        return f"inputs {gb:.2f} GB per step > 126 MB L2 (no flush needed)"
    return f"inputs {gb * 1e3:.1f} MB per step fit in the 126 MB L2 (a parity-size case, not a throughput workload)"


def prep_roofline(w, prep_ms: float, peaks, timed_s: float) -> dict:
    """The V-Smooth prep against its floor.  Compulsory bytes per head: K and
    V read as bf16 (4Nd); the quantised K (Tp d) and V residual (Tp d, or half
    plus the 16-token block scales on the 4-bit path) written; perm (4N),
    block means (4Td), K block scales (4T) and channel scales (4d).  Flops: the
    k-means assignment, 2 N C d per pass.  The floor is the slower of the
    bytes at the HBM copy rate and the flops at the bf16 tensor rate."""
    T = -(-w.N // w.block)
    Tp = T * w.block
    fp4 = resid_fmt_of(w) == 1
    resid = Tp * w.d // 2 + T * w.d * (w.block // 16) if fp4 else Tp * w.d
    per_head = 4 * w.N * w.d + Tp * w.d + resid + 4 * w.N + 4 * T * w.d + 4 * T + 4 * w.d
    nbytes = per_head * w.B * w.H
    flops = 2.0 * w.N * w.C * w.d * w.iters * w.B * w.H
    tensor, _ = tensor_peak(peaks, timed_s)
    t_bytes = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_flops = flops / (tensor * 1e12)
    floor_s = max(t_bytes, t_flops)
    t = prep_ms * 1e-3
    return {"bound": "hbm" if t_bytes >= t_flops else "tensor", "bytes": nbytes, "flops": flops,
            "achieved_gbs": nbytes / t / 1e9, "peak_gbs": peaks["hbm_gbs"], "peak_bf16_tflops": tensor,
            "floor_ms": floor_s * 1e3, "frac": floor_s / t}


def launches_per_step(p) -> int:
    """Kernels of the library one step launches (the launch list in profiles/
    shows the same sequence).  V-Smooth with C <= 64: km_init; per k-means
    pass km_pass and km_refine; between passes km_finalize; after the last,
    km_scan and km_scatter.  With C > 64: km_init; per pass km_assign,
    km_refine, km_scan, km_scatter; between passes km_update, km_finalize.
    Then prep_kv_block and prep_v_quant.  V-Smooth off (smooth 0):
    identity_order, prep_kv_block, prep_v_quant (plus a memset).  A kept
    regroup (smooth 2): prep_kv_block and prep_v_quant.  Every step then
    launches quant_q and the attention kernel."""
    if p.smooth == 1 and p.C <= 64:
        prep = 1 + 2 * p.iters + (p.iters - 1) + 2 + 2
    elif p.smooth == 1:
        prep = 1 + 4 * p.iters + 2 * (p.iters - 1) + 2
    else:
        prep = 3 if p.smooth == 0 else 2
    return prep + 2


def accuracy_vs_exact(q, k, v, out, heads, rows: int = 64) -> dict:
    """Error of the output against exact attention softmax(q k^T / sqrt(d)) v
    on the bf16 inputs, computed in fp64 with torch on sampled query rows of
    the given heads (the benchmark spec's rel-L2 and PSNR, plus cosine)."""
    B, H, N, d = q.shape
    sel = torch.unique(torch.cat([torch.linspace(0, N - 1, rows).long(), torch.tensor([N - 1])])).to(q.device)
    num, den, dot, nrm_o, peak, sq, cnt = 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0
    for h in heads:
        qh = q[0, h, sel].double()
        kh, vh = k[0, h].double(), v[0, h].double()
        ref = torch.softmax(qh @ kh.T / d ** 0.5, dim=-1) @ vh
        got = out[0, h, sel].double()
        e = got - ref
        num += float((e * e).sum())
        den += float((ref * ref).sum())
        dot += float((got * ref).sum())
        nrm_o += float((got * got).sum())
        peak = max(peak, float(ref.abs().max()))
        sq += float((e * e).sum())
        cnt += e.numel()
    rmse = (sq / cnt) ** 0.5
    return {"vs": "exact softmax attention on the bf16 inputs (fp64)", "heads": list(heads), "rows_per_head": len(sel),
            "rel_l2": (num / den) ** 0.5, "cos": dot / (den * nrm_o) ** 0.5,
            "psnr_db": 20.0 * float(np.log10(peak / rmse)) if rmse > 0 else float("inf")}


def tensor_peak(peaks, timed_s: float):
    """The measured bf16 tensor rate that applies to a kernel timed inside a
    region of timed_s seconds: the burst figure for a short region (the clocks
    stay near max), the power-capped sustained one for a region of seconds."""
    if timed_s < 2.0 or not peaks.get("bf16_sustained"):
        return peaks["bf16"], "burst"
    return peaks["bf16_sustained"], "sustained"


def run_ours(args, w):
    import bit_fp8_attention_smooth_b200 as vc

    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    vc.lib()
    full = w
    if args.split_heads:  # strong scaling: this rank takes its share of the heads
        if world > w.H:
            raise SystemExit(f"--split-heads needs at most {w.H} ranks")
        h0, h1 = vc.head_range(rank, world, w.H)
        w = dataclasses.replace(w, H=h1 - h0)
    params = vc.Params.for_workload(w, beta=BETA, smooth=int(args.smooth))
    shape = (w.B, w.H, w.N, w.d)

    # inputs resident in HBM (pinned host copies kept for the end-to-end leg)
    host = {t: synth.tensor_bf16(w, t, out=torch.empty(shape, dtype=torch.bfloat16).pin_memory()) for t in "qkv"}
    qd, kd, vd = (host[t].to(dev) for t in "qkv")
    out = torch.empty_like(qd)
    prep = vc.alloc_prep(shape, params, dev)
    ws = vc.alloc_workspace(shape, params, dev)
    stream = torch.cuda.current_stream(dev)
    # block-sparse: each query tile keeps a seeded random share of the key tiles
    tile_mask, density = None, 1.0
    if args.tile_density < 1.0:
        g = torch.Generator().manual_seed(7)
        tm = torch.rand((w.B, w.H, -(-w.N // 128), -(-w.N // w.block)), generator=g) < args.tile_density
        tile_mask = tm.to(torch.uint8).to(dev)
        density = float(tm.float().mean())

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        vc.smooth_prepare(kd, vd, params, prep=prep, workspace=ws)
        if evs is not None:
            evs[1].record(stream)
        vc.attn_fwd(qd, prep, params, out=out, workspace=ws, tile_mask=tile_mask)
        if evs is not None:
            evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    vc.check(ws)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    vc.check(ws)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    prep_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    attn_ms = max_over_ranks(attn_ms, dev)
    prep_ms = max_over_ranks(prep_ms, dev)
    ms_per_step = total_ms / args.steps
    flops = w.attn_flops * density  # this rank's (the kept key tiles only)
    job_flops = full.attn_flops * density if args.split_heads else world * flops
    # the host-buffer leg runs the dense call (vc_attention_host takes no mask)
    dense_job_flops = full.attn_flops if args.split_heads else world * w.attn_flops
    value = job_flops / (ms_per_step * 1e-3) / 1e12
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12

    # the prep of a later denoising step that keeps this step's regroup
    # (Params.smooth = 2: no k-means, block quantisation only)
    reuse = dataclasses.replace(params, smooth=2)
    vc.smooth_prepare(kd, vd, reuse, prep=prep, workspace=ws)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for _ in range(5):
        vc.smooth_prepare(kd, vd, reuse, prep=prep, workspace=ws)
    r1.record(stream)
    torch.cuda.synchronize(dev)
    vc.check(ws)
    prep_reuse_ms = max_over_ranks(r0.elapsed_time(r1) / 5, dev)

    # end to end through the public API from pinned host buffers
    # Two calls in flight: a step's copies overlap the previous step's
    # computation; each step reads its own result back into its own host
    # buffer.
    e2e = vc.HostAttention(shape, params, dev)
    o_host = [torch.empty(shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for i in range(max(2, args.warmup // 2)):
        e2e(host["q"], host["k"], host["v"], o_host[i % 2])
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(2, min(args.steps, 6))
    e0.record(stream)
    pending = [e2e(host["q"], host["k"], host["v"], o_host[i % 2]) for i in range(e2e_steps)]
    for p in pending:  # the timed region ends when every step's output is back
        p.wait()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    e2e.check()
    # error against exact attention on sampled rows of the first and last head
    acc = accuracy_vs_exact(qd, kd, vd, out, sorted({0, w.H - 1})) if rank == 0 and tile_mask is None else None

    if rank == 0:
        peaks = load_peaks()
        timed_s = total_ms * 1e-3
        bf16, which = tensor_peak(peaks, timed_s)
        fp8_peak = bf16 * FP8_PER_BF16
        four_bit = resid_fmt_of(w) == 1
        if four_bit:
            # QK^T (half the flops) at the FP8 rate, PV (the other half) at the
            # FP4 rate, twice FP8: the time at peak is 3/4 of the all-FP8 time
            peak, kernel = fp8_peak * 4.0 / 3.0, "vc_attn_fwd (vc_attn4_kernel)"
            nominal = 4500.0 * 4.0 / 3.0
            peak_src = (f"{peaks['source']} bf16 {which} {bf16} TFLOP/s x 2 (fp8:bf16) for QK^T, x 4 (fp4:bf16) "
                        f"for PV; harmonic over the two halves")
        else:
            peak, kernel, nominal = fp8_peak, "vc_attn_fwd (vc_attn_kernel)", 4500.0
            peak_src = f"{peaks['source']} bf16 {which} {bf16} TFLOP/s x 2 (fp8:bf16)"
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if args.split_heads else "weak",
            "vs_baseline": None, "dtype": "e4m3+e2m1" if four_bit else "e4m3", "data": "synthetic",
            "config": dict(config_of(full, bool(args.smooth)),
                           **({"heads_per_rank": w.H} if args.split_heads else {}),
                           **({"tile_density": density} if tile_mask is not None else {})),
            "attn_ms": attn_ms, "prep_ms": prep_ms, "prep_reuse_ms": prep_reuse_ms, "attn_tflops": attn_tflops,
            "prep_roofline": prep_roofline(w, prep_ms, peaks, timed_s) if args.smooth else None,
            "frac_of_nominal_fp8_4500": value / 4500.0,
            "roofline": {
                "bound": "tensor", "kernel": kernel,
                "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s", "frac": attn_tflops / peak,
                "peak_source": peak_src, "timed_region_s": timed_s,
                "frac_of_nominal": attn_tflops / nominal, "nominal_peak": nominal,
                "traffic": None if tile_mask is not None else attn_traffic_bytes(
                    w.B * w.H, "vc_attn4_kernel" if four_bit else "vc_attn_kernel", w.N, w.d, w.block),
                "traffic_unit": "DRAM bytes per launch (ncu capture on fewer heads of the same shape, scaled by heads)",
            },
            "accuracy": acc,
            "e2e": {"value": dense_job_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": e2e.h2d_bytes, "d2h_bytes_per_step": e2e.d2h_bytes},
            "gpu_launches": launches_per_step(params) * args.steps,
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            cores = cpu_cores()
            r = oracle_sample(w, args.ref_rows, cores, bool(args.smooth))
            line["cpu_baseline"] = {
                "value": r["value"], "unit": "TFLOPS", "cores": cores,
                "cpu_model": cpu_model(), "kind": "oracle",
                "sample": (f"head 0: full prep ({r['prep_s']:.1f} s) + {args.ref_rows} strided query rows over all "
                           f"keys ({r['rows_s']:.1f} s), extrapolated to the head's {w.N} rows"),
            }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mid_32k_d128", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--ref-rows", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--smooth", choices=["on", "off"], default="on",
                    help="V-Smooth on (k-means regroup, block means) or off (plain per-channel FP8 V)")
    ap.add_argument("--tile-density", type=float, default=1.0,
                    help="block-sparse attention: the share of key tiles each query tile keeps (seeded random mask; "
                         "flops count the kept tiles only)")
    ap.add_argument("--split-heads", action="store_true",
                    help="strong scaling: the ranks split the workload's heads (default: weak scaling, every rank "
                         "runs the whole workload)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only this many heads of the workload (profiling captures on a smaller case)")
    args = ap.parse_args()
    args.smooth = args.smooth == "on"
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, name=f"{w.name}_h{args.heads}", H=args.heads)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
