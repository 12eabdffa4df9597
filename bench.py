"""Benchmark of the FP8 attention path on B200.

One step = the whole FP8 hot path over one batch of synthetic input:
fqa_quantize (K mean, Q/K/V block quantization) + fqa_attention_fp8, on the
context-image editing workload (B=1, H=24, N=8704 = 512 text + 4096 context
image + 4096 output image tokens, d=128).  value = 4*B*H*N^2*d FLOPs per step
/ device time per step, in TFLOP/s, summed over ranks (each rank runs its own
independently seeded batch; no data-path collective: weak scaling).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fqa|reference]
For N > 1 launch with torch.distributed.run (one rank per GPU).
python bench.py --sweep prints one line per workload (quantizer, FP8 and BF16
attention timed separately, at most 200 launches each) instead.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import fqa_synth as synth  # noqa: E402

METRIC = "FP8 attention TFLOP/s and % of B200 FP8 peak at N=8704, H=24, d=128"
WORKLOAD = "kontext_n8704"
NOMINAL_FP8_TFLOPS = 4500.0
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["quantized_fp8_attention_b200/csrc/attention.cuh",
                  "quantized_fp8_attention_b200/csrc/attention_fp8.cuh",
                  "quantized_fp8_attention_b200/csrc/device.cuh"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK), "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_per_launch():
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "attn_fp8_kontext_n8704_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_source_sha") != kernel_source_sha():
        return None
    return d.get("traffic_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        mhz, mx, reasons = [], [], set()
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                mhz.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(mhz)}


def host_inputs(w, rank: int):
    """Seeded BF16 inputs; each rank draws its own batch (seed offset by rank)."""
    import dataclasses
    wr = dataclasses.replace(w, seed=w.seed + 7919 * rank) if rank else w
    return synth.generate(wr), wr


def max_over_ranks(x: float, device, world: int) -> float:
    """The maximum of a per-rank float over all ranks (the job's time is its
    slowest rank's); a plain value when world == 1."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes flops_per_rank per step (weak
    scaling), the step takes the slowest rank's time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def fp8_gemm_probe(dev):
    """A library FP8 GEMM for context (cuBLASLt through torch._scaled_mm,
    8192^3 E4M3 x E4M3 -> BF16, best of 10 after warm-up).  Not the roofline
    denominator: that is the measured BF16 peak x the nominal FP8:BF16 ratio."""
    import torch
    n = 8192
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = float("inf")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(10):
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return {"tflops": 2 * n ** 3 / (best * 1e-3) / 1e12,
                "how": "torch._scaled_mm 8192^3 e4m3 x e4m3 -> bf16, best of 10 (context only)"}
    except Exception as exc:  # an FP8 GEMM the local torch build does not offer
        return {"tflops": None, "how": f"unavailable: {type(exc).__name__}"}


def run_sweep(args):
    """One JSON line per workload: quantizer, FP8 attention and BF16 attention
    each timed alone with CUDA events (the quantizer with an L2 flush before
    every launch), at most 200 launches (about half a second) per kernel."""
    import torch

    import quantized_fp8_attention_b200 as fqa
    from quantized_fp8_attention_b200 import build as fqa_build

    fqa_build.build()
    dev = torch.device("cuda", 0)
    pk, pk_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for w in synth.WORKLOADS:
        g = synth.generate(w)
        q, k, v = (torch.from_numpy(g[t].view(np.int16)).view(torch.bfloat16).to(dev) for t in "qkv")
        qz = fqa.alloc_quantized(w.B, w.H, w.N, dev)
        ws = fqa.alloc_workspace(w.B, w.H, w.N, dev)
        out = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.bfloat16, device=dev)
        scale = fqa.softmax_scale(w.d)

        def timed(fn, reps, pre=None):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
            for i in range(reps):
                if pre:
                    pre()
                e[2 * i].record()
                fn()
                e[2 * i + 1].record()
            torch.cuda.synchronize()
            return sum(e[2 * i].elapsed_time(e[2 * i + 1]) for i in range(reps)) / reps

        fqa.quantize(q, k, v, out=qz, workspace=ws)
        # about 0.5 s of each kernel, between 5 and 200 launches
        reps = lambda tflops: min(200, max(5, int(0.5 / (w.flops / (tflops * 1e12)))))
        ms_a = timed(lambda: fqa.attention_fp8(qz, scale, fqa.FQA_OUT_BF16, out=out), reps(1200))
        ms_b = timed(lambda: fqa.attention_bf16(q, k, v, scale, fqa.FQA_OUT_BF16, out=out), reps(850))
        ms_q = timed(lambda: fqa.quantize(q, k, v, out=qz, workspace=ws), 200, pre=lambda: flush.fill_(1))
        # error-corrected attention (rho = 0.005) on the same codes: selection,
        # masked FP8 attention, exact part and merge
        k_err = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=dev)
        fqa.quantize_keyerr(q, k, v, out=qz, k_err=k_err, workspace=ws)
        cws = fqa.alloc_corrected_workspace(w.B, w.H, w.N, 0.005, dev)
        ms_c = timed(lambda: fqa.attention_fp8_corrected(q, k, v, qz, k_err, scale, 0.005, fqa.FQA_OUT_BF16,
                                                         out=out, workspace=cws), reps(1000))
        # NVFP4 Q.K: the FP4 quantizer and the attention
        fqa.quantize(q, k, v, out=qz, workspace=ws)
        qn = fqa.quantize_nvfp4_qk(q, k, qz.k_mean)
        ms_n = timed(lambda: fqa.attention_nvfp4(qn, qz, scale, fqa.FQA_OUT_BF16, out=out), reps(850))
        ms_nq = timed(lambda: fqa.quantize_nvfp4_qk(q, k, qz.k_mean, out=qn), 100, pre=lambda: flush.fill_(1))
        nv = {"ms": ms_n, "tflops": w.flops / ms_n / 1e9, "time_vs_fp8": ms_n / ms_a,
              "quantize_nvfp4_qk_ms": ms_nq}
        st, flags = fqa.fqa_debug_status()
        if st != fqa.FQA_OK:
            raise RuntimeError(f"device status {flags:#x} on {w.name}")
        fp8_peak = 2 * pk["bf16_tflops"]
        qbytes = 9 * w.B * w.H * w.N * w.d
        print(json.dumps({
            "sweep": True, "workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
            "attention_fp8": {"ms": ms_a, "tflops": w.flops / ms_a / 1e9,
                              "frac_of_fp8_peak": w.flops / ms_a / 1e9 / fp8_peak},
            "attention_fp8_corrected": {"ms": ms_c, "rho": 0.005, "keys_per_head": fqa.fqa_corrected_keys(w.N, 0.005),
                                        "time_vs_fp8": ms_c / ms_a, "time_vs_bf16": ms_c / ms_b},
            "attention_bf16": {"ms": ms_b, "tflops": w.flops / ms_b / 1e9,
                               "frac_of_bf16_peak": w.flops / ms_b / 1e9 / pk["bf16_tflops"]},
            "attention_nvfp4": nv,
            "quantizer": {"ms": ms_q, "gbs": qbytes / ms_q / 1e6, "frac_of_hbm": qbytes / ms_q / 1e6 / pk["hbm_gbs"],
                          "l2": "flushed before every launch"},
            "peaks": pk_kind}), flush=True)
        del q, k, v, qz, ws, out, k_err, cws
        torch.cuda.empty_cache()


def step_line(w, world: int, K: int, warmup: int, ms_per_step: float, attn_ms: float, quant_ms: float,
              bf16_ms: float, e2e_ms: float, h2d: int, d2h: int, clocks: dict, probe, cpu, traffic,
              pk: dict, pk_kind: str, corrected=None, accuracy=None) -> dict:
    """The benchmark's JSON line for workload w from the measured times (ms).
    value and e2e are whole-job throughput (every rank runs its own batch);
    roofline is for the FP8 attention kernel against 2 x the measured BF16
    peak (the nominal FP8:BF16 ratio)."""
    B, H, N, d = w.B, w.H, w.N, w.d
    flops = w.flops
    fp8_peak = 2.0 * pk["bf16_tflops"]            # FP8 dense = 2 x BF16 dense (nominal ratio)
    bf16_peak = pk["bf16_tflops"]
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    quant_bytes = 9 * B * H * N * d
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    bf16_tflops = flops / (bf16_ms * 1e-3) / 1e12
    return {
        "metric": METRIC, "value": job_tflops(flops, world, ms_per_step), "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate)",
        "data": "synthetic (seeded, FLUX-style token mix; see fqa_synth)",
        "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d,
                   "n_text": w.n_text, "n_ctx": w.n_ctx, "n_img": w.n_img,
                   "step": "fqa_quantize + fqa_attention_fp8",
                   "l2": "inputs larger than L2 (BF16 Q,K,V = %.0f MB per step)" % (3 * 2 * B * H * N * d / 1e6),
                   "parallelism": f"dp{world} (independent batches)"},
        "roofline": {"bound": "tensor", "kernel": "attn_fp8_kernel", "achieved": attn_tflops,
                     "peak": fp8_peak, "unit": "TFLOP/s", "frac": attn_tflops / fp8_peak,
                     "peak_source": f"{pk_kind}: 2 x bf16_tflops (burst) of MEASURED_PEAKS.json",
                     "frac_of_nominal_4500": attn_tflops / NOMINAL_FP8_TFLOPS,
                     "target_frac": 0.6,
                     "meets_target": attn_tflops / fp8_peak >= 0.6 and attn_tflops / NOMINAL_FP8_TFLOPS >= 0.6,
                     "ms_per_launch": attn_ms, "traffic": traffic,
                     "traffic_note": "DRAM bytes ncu observed during one launch; most of the BF16 output "
                                     "is still in L2 when it ends, so writes undercount it"},
        "quantizer": {"ms": quant_ms, "gbs": quant_gbs, "algorithmic_bytes": quant_bytes,
                      "frac_of_hbm": quant_gbs / pk["hbm_gbs"], "hbm_peak_gbs": pk["hbm_gbs"],
                      "target_frac": 0.7, "meets_target": quant_gbs / pk["hbm_gbs"] >= 0.7},
        "bf16_path": {"ms": bf16_ms, "tflops": bf16_tflops, "frac_of_bf16_peak": bf16_tflops / bf16_peak,
                      "frac_of_nominal_2250": bf16_tflops / NOMINAL_BF16_TFLOPS},
        "e2e": {"value": job_tflops(flops, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipeline": "two device buffer sets; uploads, kernels and downloads on three streams"},
        # per step: quantize_fused_kernel + attn_fp8_kernel (plus one
        # 16-byte cudaMemsetAsync of the quantizer's counters)
        "gpu_launches": 2 * K,
        "clocks": clocks,
        "fp8_gemm_probe": probe,
        "cpu_baseline": cpu,
        "corrected": corrected,
        "accuracy": accuracy,
    }


# ----------------------------------------------------------------- accuracy

def accuracy_sample(w, g, q, k, v, scale, rho, qz, k_err, out, cws):
    """Cosine against exact FP64 attention (the CPU oracle) on 2 heads x 384
    rows of the workload, for the plain FP8 path and the corrected path, with
    the 0.995 target flagged.  Runs outside the timed region."""
    import torch

    import oracle
    import quantized_fp8_attention_b200 as fqa
    heads = [(0, 0), (0, w.H - 1)]
    rows = list(range(0, 128)) + list(range(w.N // 2, w.N // 2 + 128)) + list(range(w.N - 128, w.N))
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], scale, heads=heads, rows=rows)

    def cos(t):
        a = t.float().cpu().numpy()
        got = np.stack([a[b, h][rows] for (b, h) in heads]).astype(np.float64)
        return float((got * ex).sum() / np.sqrt((got * got).sum() * (ex * ex).sum()))

    fqa.quantize(q, k, v, out=qz)
    plain = cos(fqa.attention_fp8(qz, scale, fqa.FQA_OUT_F32))
    fqa.quantize_keyerr(q, k, v, out=qz, k_err=k_err)
    corr = cos(fqa.attention_fp8_corrected(q, k, v, qz, k_err, scale, rho, fqa.FQA_OUT_F32, workspace=cws))
    fqa.quantize(q, k, v, out=qz)
    nv = cos(fqa.attention_nvfp4(fqa.quantize_nvfp4_qk(q, k, qz.k_mean), qz, scale, fqa.FQA_OUT_F32))
    sample = f"heads {heads}, rows [0,128) u [N/2, N/2+128) u [N-128, N), all keys"
    accuracy = {"cos_vs_exact_fp64": plain, "target": 0.995, "meets_target": plain >= 0.995, "sample": sample}
    corrected = {"rho": rho, "keys_per_head": fqa.fqa_corrected_keys(w.N, rho), "cos_vs_exact_fp64": corr,
                 "meets_target": corr >= 0.995}
    return accuracy, corrected, nv


# ------------------------------------------------------------ CPU baseline

def oracle_sample(w, g, heads, rows):
    """Time the CPU oracle on a bounded sample: the quantizer on the sampled
    heads (full sequence) plus FP8 attention for `rows` query rows of each
    sampled head against all keys.  Returns (seconds, flops, threads)."""
    import oracle
    oracle.build()
    sel = lambda a: np.ascontiguousarray(np.stack([a[b, h] for (b, h) in heads])[None])
    q, k, v = (sel(g[t]) for t in "qkv")
    t0 = time.perf_counter()
    qz = oracle.quantize(q, k, v)
    oracle.attention_fp8(qz, oracle.softmax_scale(), heads=[(0, i) for i in range(len(heads))],
                         rows=rows)
    dt = time.perf_counter() - t0
    flops = 4 * len(heads) * len(rows) * w.N * w.d
    return dt, flops, oracle.num_threads()


def cpu_baseline(w, g):
    rows = list(range(0, w.N, max(1, w.N // 1024)))[:1024]
    heads = [(0, h) for h in range(min(w.H, 4))]
    dt, flops, threads = oracle_sample(w, g, heads, rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(heads)} heads: quantizer over all {w.N} tokens + FP8 attention for "
                      f"{len(rows)} strided query rows x all {w.N} keys ({dt:.1f} s)"}


def run_reference(args, rank: int, world: int):
    """The reference arm: the CPU oracle as it stands, on bounded samples of
    the same workload, in the same metric and unit."""
    if rank != 0:
        return
    w = synth.workload(args.workload)
    g = synth.generate(w, heads=[(0, h) for h in range(2)])
    # per-step sample sized so that the whole run stays within a few minutes:
    # 256 strided query rows up to 50 steps, fewer beyond (at least 64)
    n_rows = max(64, min(256, (256 * 50) // max(1, args.steps + args.warmup)))
    rows = list(range(0, w.N, max(1, w.N // n_rows)))[:n_rows]
    heads = [(0, 0), (0, 1)]
    for _ in range(args.warmup):
        oracle_sample(w, g, heads, rows[:16])
    times, flops, threads = [], 0, 1
    for _ in range(args.steps):
        dt, flops, threads = oracle_sample(w, g, heads, rows)
        times.append(dt)
    t = sum(times) / len(times)
    value = flops / t / 1e12
    sample = (f"per step: quantizer on 2 heads x {w.N} tokens + FP8 attention for {len(rows)} strided "
              f"rows x {w.N} keys on each")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------- GPU arm

def run_fqa(args, rank: int, world: int):
    import torch
    import torch.distributed as dist

    import quantized_fp8_attention_b200 as fqa
    from quantized_fp8_attention_b200 import build as fqa_build

    fqa_build.build()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w0 = synth.workload(args.workload)
    g, w = host_inputs(w0, rank)
    B, H, N, d = w.B, w.H, w.N, w.d
    flops = w.flops
    scale = fqa.softmax_scale(d)

    def dev_tensor(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = (dev_tensor(g[t]) for t in "qkv")
    qz = fqa.alloc_quantized(B, H, N, dev)
    ws = fqa.alloc_workspace(B, H, N, dev)
    out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        fqa.quantize(q, k, v, out=qz, workspace=ws)
        fqa.attention_fp8(qz, scale, fqa.FQA_OUT_BF16, out=out)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st, flags = fqa.fqa_debug_status()
    if st != fqa.FQA_OK:
        raise RuntimeError(f"device status {flags:#x} after warm-up")

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K + 1)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev[0].record(stream)
        for i in range(K):
            fqa.quantize(q, k, v, out=qz, workspace=ws)
            ev[2 * i + 1].record(stream)
            fqa.attention_fp8(qz, scale, fqa.FQA_OUT_BF16, out=out)
            ev[2 * i + 2].record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = ev[0].elapsed_time(ev[2 * K])
    quant_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K)) / K
    attn_ms = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(K)) / K
    st, flags = fqa.fqa_debug_status()
    if st != fqa.FQA_OK:
        raise RuntimeError(f"device status {flags:#x} after the timed steps")

    ms_per_step = max_over_ranks(total_ms, dev, world) / K

    # BF16 comparison path (a9), same inputs
    for _ in range(3):
        fqa.attention_bf16(q, k, v, scale, fqa.FQA_OUT_BF16, out=out)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Kb = max(1, K // 2)
    e0.record(stream)
    for _ in range(Kb):
        fqa.attention_bf16(q, k, v, scale, fqa.FQA_OUT_BF16, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    bf16_ms = e0.elapsed_time(e1) / Kb

    # end to end through the public API with host buffers: every step copies
    # its BF16 Q, K, V in from pinned host memory and its BF16 output back out.
    # Two device buffer sets let step i+1's upload and step i-1's download run
    # beside step i's kernels (uploads, kernels and downloads on three streams).
    hq, hk, hv = (torch.from_numpy(g[t].view(np.int16)).view(torch.bfloat16).pin_memory() for t in "qkv")
    hout = torch.empty(B, H, N, d, dtype=torch.bfloat16).pin_memory()
    h2d = 3 * hq.numel() * hq.element_size()
    d2h = hout.numel() * hout.element_size()
    sets = [(q, k, v, qz, ws, out),
            (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
             fqa.alloc_quantized(B, H, N, dev), fqa.alloc_workspace(B, H, N, dev), torch.empty_like(out))]
    s_up, s_dn = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_dn = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        dq, dk, dv, dqz, dws, dout = sets[b]
        if i >= 2:
            s_up.wait_event(ev_cmp[b])          # step i-2's kernels have read set b
        with torch.cuda.stream(s_up):
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            ev_up[b].record(s_up)
        stream.wait_event(ev_up[b])
        if i >= 2:
            stream.wait_event(ev_dn[b])         # step i-2's output has left dout
        fqa.quantize(dq, dk, dv, out=dqz, workspace=dws)
        fqa.attention_fp8(dqz, scale, fqa.FQA_OUT_BF16, out=dout)
        ev_cmp[b].record(stream)
        s_dn.wait_event(ev_cmp[b])
        with torch.cuda.stream(s_dn):
            hout.copy_(dout, non_blocking=True)
            ev_dn[b].record(s_dn)

    for i in range(4):
        e2e_step(i)
    Ke = max(4, K // 4)
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    s_up.wait_stream(stream)
    for i in range(Ke):
        e2e_step(i + 4)
    stream.wait_stream(s_dn)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, dev, world)

    # error-corrected FP8 attention at the pages' rho, same inputs: the quantizer
    # with the key error, selection, masked FP8 attention, exact part + merge
    rho = 0.005
    k_err = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    cws = fqa.alloc_corrected_workspace(B, H, N, rho, dev)

    def corrected_step():
        fqa.quantize_keyerr(q, k, v, out=qz, k_err=k_err, workspace=ws)
        fqa.attention_fp8_corrected(q, k, v, qz, k_err, scale, rho, fqa.FQA_OUT_BF16, out=out, workspace=cws)

    for _ in range(3):
        corrected_step()
    Kc = max(1, K // 2)
    e0.record(stream)
    for _ in range(Kc):
        corrected_step()
    e1.record(stream)
    torch.cuda.synchronize()
    corr_ms = e0.elapsed_time(e1) / Kc
    st, flags = fqa.fqa_debug_status()
    if st != fqa.FQA_OK:
        raise RuntimeError(f"device status {flags:#x} after the corrected steps")

    # NVFP4 Q.K with FP8 P.V, same inputs: the FP8 quantizer (V codes and the K
    # mean), the NVFP4 quantizer of Q and smoothed K, the attention
    qn = fqa.alloc_quantized_nvfp4(B, H, N, dev)

    def nvfp4_step():
        fqa.quantize(q, k, v, out=qz, workspace=ws)
        fqa.quantize_nvfp4_qk(q, k, qz.k_mean, out=qn)
        fqa.attention_nvfp4(qn, qz, scale, fqa.FQA_OUT_BF16, out=out)

    for _ in range(3):
        nvfp4_step()
    Kn = max(1, K // 4)
    e0.record(stream)
    for _ in range(Kn):
        nvfp4_step()
    e1.record(stream)
    torch.cuda.synchronize()
    nv_ms = e0.elapsed_time(e1) / Kn
    st, flags = fqa.fqa_debug_status()
    if st != fqa.FQA_OK:
        raise RuntimeError(f"device status {flags:#x} after the NVFP4 steps")

    ulysses = run_ulysses(w0, scale, dev, rank, world, K, ms_per_step) if world > 1 else None

    if rank != 0:
        return
    pk, pk_kind = peaks()
    probe = fp8_gemm_probe(dev)
    accuracy, corrected, nv_cos = accuracy_sample(w, g, q, k, v, scale, rho, qz, k_err, out, cws)
    corrected.update({"ms_per_step": corr_ms, "step": "fqa_quantize_keyerr + fqa_attention_fp8_corrected",
                      "tflops": flops / (corr_ms * 1e-3) / 1e12,
                      "time_vs_fp8_step": corr_ms / ms_per_step, "time_vs_bf16_attention": corr_ms / bf16_ms})
    cpu = None if args.no_cpu_baseline else cpu_baseline(w, g)
    line = step_line(w, world, K, args.warmup, ms_per_step, attn_ms, quant_ms, bf16_ms, e2e_ms, h2d, d2h,
                     clk.summary(), probe, cpu, traffic_per_launch(), pk, pk_kind, corrected, accuracy)
    if ulysses is not None:
        line["ulysses"] = ulysses
    line["nvfp4"] = {"ms_per_step": nv_ms, "tflops": flops / (nv_ms * 1e-3) / 1e12,
                     "step": "fqa_quantize + fqa_quantize_nvfp4_qk + fqa_attention_nvfp4",
                     "time_vs_fp8_step": nv_ms / ms_per_step, "cos_vs_exact_fp64": nv_cos}
    print(json.dumps(line), flush=True)


def run_ulysses(w0, scale, dev, rank: int, world: int, K: int, dp_ms: float):
    """The pages' multi-GPU form ("FLUX 3 Image Klein Base", sections "결과" and
    "고를 때 기준": Ulysses sequence parallel): one workload's sequence split
    over the world, all-to-all to head shards, FP8 attention per rank,
    all-to-all back.  Every rank holds a shard of the same inputs (rank 0's
    seed); timed like the step (events, barriers, max over ranks)."""
    import torch
    import torch.distributed as dist

    from quantized_fp8_attention_b200 import ulysses as uly

    B, H, N, d = w0.B, w0.H, w0.N, w0.d
    if H % world or N % world or (N // world) % 64:
        return {"skipped": f"{H} heads / {N} tokens do not split over {world} ranks"}
    try:
        g, _ = host_inputs(w0, 0)
        Nl = N // world

        def shard(bits):
            x = np.ascontiguousarray(bits[:, :, rank * Nl:(rank + 1) * Nl])
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)

        qs, ks, vs = (shard(g[t]) for t in "qkv")
        for _ in range(3):
            uly.ulysses_fp8_attention(qs, ks, vs, scale)
        torch.cuda.synchronize()
        Ku = max(4, K // 8)
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(Ku):
            uly.ulysses_fp8_attention(qs, ks, vs, scale)
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        ms = max_over_ranks(e0.elapsed_time(e1) / Ku, dev, world)
        return {"degree": world, "workload": w0.name, "steps": Ku, "ms_per_step": ms,
                "tflops": w0.flops / (ms * 1e-3) / 1e12, "scaling": "strong",
                "step": "all-to-all (q, k, v) + fqa_quantize_a2a + fqa_attention_fp8_a2a + all-to-all (out)",
                "speedup_vs_one_gpu_step": dp_ms / ms}
    except Exception as e:  # noqa: BLE001 -- reported in the line, the step's numbers stand
        return {"error": f"{type(e).__name__}: {e}"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="fqa", choices=["fqa", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="one line per workload instead of the step")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_fqa(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
