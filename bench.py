"""Per-layer GPTQ throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload q_proj_4096]
                    [--impl ours|reference] [--no-cpu-baseline]

--workload decoder_layer times the layer-sequential calibration of a whole
decoder layer; --workload w4a16 times the product of bf16 activations with the
packed 4-bit output (the inference-side consumer of the format).

One step = the whole per-layer path on one synthetic layer: Hessian over all
calibration tokens (H = 2 X^T X), damping + Cholesky factor of the inverse,
the blocked GPTQ column loop with lazy-batch updates, unpermute and int4
packing.  Inputs (X 2.15 GB bf16 for q_proj_4096, larger than the 126 MB L2)
are resident in HBM before the timed region.  With N > 1 (torchrun), every
rank quantizes its own independent layer (layers are independent, GPTQ
overview page "Równoległość"): weak scaling, no collective in the data path.

With --split tokens_rows (torchrun, N ranks) the ranks instead share ONE
layer: each accumulates the Hessian over its own slice of the tokens, one NCCL
all-reduce sums H, every rank factorises the same H, and each quantizes its
own block of rows (GPTQ overview page, "Równoległość"; strong scaling).

The default run also times the other single-GPU workloads of the layer recipe
once each (down_proj 11008, 70B up_proj, a full Llama-2-7B decoder layer, the
fp32-activation Hessian) under "by_config" of the same line.

Prints one JSON line (rank 0).  value = quantized weights/s over all ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ quantized weights/s per layer; Hessian+update TFLOP/s vs B200 peak"
UNIT = "weights/s"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "hessian_tc_kernel_q_proj_4096.md")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="q_proj_4096")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="decoder_layer: bits {2,3,4} x group_size {64,128,per-channel}")
    ap.add_argument("--split", default="layers", choices=["layers", "tokens_rows"],
                    help="N > 1: an independent layer per rank, or one layer split over the ranks")
    ap.add_argument("--no-by-config", action="store_true",
                    help="skip the other workloads in the default run")
    ap.add_argument("--validate-cost-laws", action="store_true",
                    help="reference arm: also run the checker's factorisation at full d_in and "
                         "256 full rows of the column loop, against the sample's extrapolation")
    return ap.parse_args()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples every 100 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.5)   # let the sampler start before the timed region
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ------------------------------------------------------------------ helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return json.load(open(p)), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


PROFILE_TF32 = os.path.join(ROOT, "profiles", "tf32_peak_cublas.md")


def tf32_peaks():
    """Measured dense tf32 throughput of the vendor GEMM, burst and
    sustained, from the committed measurement; None where missing."""
    out = {"burst": None, "sustained": None}
    try:
        for line in open(PROFILE_TF32):
            if line.startswith("tf32_tflops:"):
                out["burst"] = float(line.split(":", 1)[1].split()[0])
            if line.startswith("tf32_tflops_sustained:"):
                out["sustained"] = float(line.split(":", 1)[1].split()[0])
    except OSError:
        pass
    return out


def regime(clocks) -> str:
    """Which measured peak applies to this run: "burst" when the clock record
    of the timed region never showed the power cap and the median SM clock sat
    at its maximum, else "sustained" (the figure taken under the power cap)."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if mhz is None or mx is None:
        return "sustained"
    if "sw_power_cap" in clocks.get("reasons", []) or mhz < 0.97 * mx:
        return "sustained"
    return "burst"


def bf16_peaks(peaks):
    return {"burst": float(peaks.get("bf16_tflops")),
            "sustained": float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))}


def lazy_flops(spec) -> float:
    """fp32 flops of all lazy-batch products of one layer: every (j, k) column
    pair in different blocks, per row: d_out (d_in^2 - sum of block widths^2)."""
    bw = [min(spec.block_size, spec.d_in - j) for j in range(0, spec.d_in, spec.block_size)]
    return float(spec.d_out) * (spec.d_in ** 2 - sum(b * b for b in bw))


def lazy_batch_line(spec, stage):
    """All lazy-batch products of the column loop against the measured tf32
    peak: `ms` is the sum of the products' own spans in the production launch
    sequence (gptq_quantize_timed: device clock from each product's first CTA
    past its dependency wait to its last CTA's end); `frac` against the burst
    figure (the products run as short bursts inside the column loop),
    `frac_sustained` against the power-capped one."""
    if not stage or not stage.get("lazy_batch_ms"):
        return None
    fl = lazy_flops(spec)
    rate = fl / (stage["lazy_batch_ms"] / 1e3) / 1e12
    pk = tf32_peaks()
    return {"flops_fp32": fl, "ms": stage["lazy_batch_ms"], "achieved_fp32_tflops": rate,
            "tf32_rate_tflops": 3 * rate, "peak": pk["burst"], "peak_sustained": pk["sustained"],
            "unit": "TFLOP/s", "frac": (3 * rate / pk["burst"]) if pk["burst"] else None,
            "frac_sustained": (3 * rate / pk["sustained"]) if pk["sustained"] else None,
            "note": "3xTF32: three tf32 MMAs per fp32-accurate product; ms = summed in-schedule "
                    "kernel spans (globaltimer); peaks = measured cuBLAS tf32 (profiles/tf32_peak_cublas.md)"}


def layer_roofline(spec, ms, reg, peaks):
    """Ideal time of the layer's tensor work at the measured peaks of this
    run's clock regime (Hessian on bf16, factorisation and lazy batch as
    3xTF32) against the measured step; the column loop's chain of dependent
    column steps has no flop roofline and is not in the ideal."""
    tf = tf32_peaks()[reg]
    if not tf:
        return None
    d = spec.d_in
    t_h = spec.n_tokens * d * (d + 1) / (bf16_peaks(peaks)[reg] * 1e12) * 1e3
    t_f = 3 * (2.0 / 3.0) * d ** 3 / (tf * 1e12) * 1e3
    t_l = 3 * lazy_flops(spec) / (tf * 1e12) * 1e3
    ideal = t_h + t_f + t_l
    return {"ideal_ms": ideal, "measured_ms": ms, "frac": ideal / ms, "peaks": reg,
            "terms_ms": {"hessian": t_h, "factorisation": t_f, "lazy_batch": t_l}}


def hessian_split(spec, sms: int = 148) -> int:
    """Token spans per tile of one Hessian launch (the launcher's rule): the
    longest power-of-two span in 4096 .. 32768 that still gives every pair of
    SMs about eight work units; a single unit when H is one 256-column tile."""
    n_t = (spec.d_in + 255) // 256
    if n_t == 1:
        return 1
    tiles = n_t * (n_t + 1) // 2
    span = 32768
    while span > 4096 and tiles * -(-spec.n_tokens // span) < 8 * (sms // 2):
        span //= 2
    return -(-spec.n_tokens // span)


def hessian_alg_bytes(spec) -> float:
    """Algorithmic DRAM bytes of one Hessian launch: X read once, and every
    token span's partial sum added into the upper triangle of H (one read and
    one write of each element per span)."""
    d = spec.d_in
    return 2.0 * spec.n_tokens * d + hessian_split(spec) * (d * (d + 1) / 2) * 8.0


def hessian_roofline(spec, h_ms, clocks, peaks, peak_kind):
    """Roofline object of the Hessian kernel (the dominant kernel): achieved =
    N d (d + 1) flops (upper triangle incl. the diagonal) / launch time, peak
    = the measured bf16 figure of the run's clock regime; both fractions."""
    reg = regime(clocks)
    pk = bf16_peaks(peaks)
    alg_flops = spec.n_tokens * spec.d_in * (spec.d_in + 1)
    achieved = alg_flops / (h_ms / 1e3) / 1e12
    traffic = profiled_traffic(os.path.join(ROOT, "post_weight_quantization_accumulate_b200",
                                            "csrc", "hessian.cu"))
    if traffic is not None and spec.name != "q_proj_4096":
        traffic = None
    alg_bytes = hessian_alg_bytes(spec)
    return {"kernel": "hessian_tc_kernel (+ mirror copy)", "bound": "tensor",
            "achieved": achieved, "peak": pk[reg], "unit": "TFLOP/s", "frac": achieved / pk[reg],
            "traffic": traffic, "peak_source": f"{peak_kind} bf16_tflops ({reg}; clocks of this run)",
            "frac_burst": achieved / pk["burst"], "frac_sustained": achieved / pk["sustained"],
            "flops_per_launch": alg_flops, "launch_ms": h_ms, "alg_bytes": alg_bytes,
            "traffic_over_alg_bytes": (traffic / alg_bytes) if traffic else None}


def profiled_traffic(kernel_src: str):
    """dram read+write bytes per launch of the Hessian kernel from the committed
    ncu summary, or None when the kernel source changed since the capture."""
    import hashlib
    try:
        text = open(PROFILE_TRAFFIC).read()
    except OSError:
        return None
    h = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    val, src_hash = None, None
    for line in text.splitlines():
        if line.startswith("traffic_bytes_per_launch:"):
            val = float(line.split(":", 1)[1].split()[0])
        if line.startswith("kernel_source_sha256_16:"):
            src_hash = line.split(":", 1)[1].strip()
    return val if (val is not None and src_hash == h) else None


def cpu_baseline(spec, threads: int):
    """The float64 checker on a bounded sample of the same workload, each stage
    extrapolated to the full layer by its own cost law:
      Hessian      2048 of n_tokens tokens, full d_in     (x n_tokens/2048, O(N d^2))
      factor       leading 1024 x 1024 block of that H    (x (d_in/1024)^3, O(d^3))
      column loop  32 rows at d_in = 1024                 (x d_out/32 x (d_in/1024)^2)
    `measured_s` is the time the sample took; `extrapolated_layer_s` the full
    layer's time by those laws (an extrapolation, not a measurement)."""
    import numpy as np
    import oracle
    from post_weight_quantization_accumulate_b200 import synth
    n_s, d_s, r_s = 2048, min(1024, spec.d_in), 32
    xb = synth.x_bf16(spec, tokens=slice(0, n_s))
    t0 = time.perf_counter()
    H = oracle.hessian(xb)
    t_h = time.perf_counter() - t0
    Hs = np.ascontiguousarray(H[:d_s, :d_s])
    t0 = time.perf_counter()
    perm, U, _, _ = oracle.prepare(Hs, spec.damp, spec.act_order)
    t_p = time.perf_counter() - t0
    W = synth.weight_f32(spec, rows=slice(0, r_s))[:, :d_s].astype(np.float64)
    t0 = time.perf_counter()
    oracle.quantize(W, U, perm, spec.bits, spec.group_size if spec.group_size <= d_s else -1,
                    spec.block_size)
    t_q = time.perf_counter() - t0
    laws = {"hessian": spec.n_tokens / n_s, "factor": (spec.d_in / d_s) ** 3,
            "column_loop": (spec.d_out / r_s) * (spec.d_in / d_s) ** 2}
    stages = {"hessian": t_h, "factor": t_p, "column_loop": t_q}
    full = sum(stages[k] * laws[k] for k in stages)
    sample = (f"Hessian on {n_s}/{spec.n_tokens} tokens (x{laws['hessian']:g}); factor at d={d_s} "
              f"(x{laws['factor']:g}); column loop {r_s} rows at d_in={d_s} "
              f"(x{laws['column_loop']:g}); float64, OpenMP; value extrapolated by these cost laws")
    return {"value": spec.d_out * spec.d_in / full, "unit": UNIT, "cores": threads,
            "kind": "oracle", "sample": sample, "measured_s": t_h + t_p + t_q,
            "stages_measured_s": stages, "extrapolated_layer_s": full,
            "value_basis": "extrapolated: full-layer time from the measured sample by the cost laws"}


def validate_cost_laws(spec, threads: int):
    """Checks the extrapolation once against full-size runs of the checker:
    the factorisation at the workload's own d_in (from the Hessian of 2048
    tokens), and 256 full rows of the column loop (with that factor); each
    against the sample's time scaled by its cost law."""
    import numpy as np
    import oracle
    from post_weight_quantization_accumulate_b200 import synth
    d_s, r_s, rows = min(1024, spec.d_in), 32, 256
    xb = synth.x_bf16(spec, tokens=slice(0, 2048))
    H = oracle.hessian(xb)
    t0 = time.perf_counter()
    oracle.prepare(np.ascontiguousarray(H[:d_s, :d_s]), spec.damp, spec.act_order)
    t_small = time.perf_counter() - t0
    t0 = time.perf_counter()
    perm, U, _, _ = oracle.prepare(H, spec.damp, spec.act_order)
    t_full = time.perf_counter() - t0
    gs = spec.group_size
    Ws = synth.weight_f32(spec, rows=slice(0, r_s))[:, :d_s].astype(np.float64)
    perm_s, U_s, _, _ = oracle.prepare(np.ascontiguousarray(H[:d_s, :d_s]), spec.damp, spec.act_order)
    t0 = time.perf_counter()
    oracle.quantize(Ws, U_s, perm_s, spec.bits, gs if gs <= d_s else -1, spec.block_size)
    q_small = time.perf_counter() - t0
    Wf = synth.weight_f32(spec, rows=slice(0, rows)).astype(np.float64)
    t0 = time.perf_counter()
    oracle.quantize(Wf, U, perm, spec.bits, gs, spec.block_size)
    q_full = time.perf_counter() - t0
    f_pred = t_small * (spec.d_in / d_s) ** 3
    q_pred = q_small * (rows / r_s) * (spec.d_in / d_s) ** 2
    return {"factor": {"d": spec.d_in, "measured_s": t_full, "extrapolated_s": f_pred,
                       "extrapolated_over_measured": f_pred / t_full},
            "column_loop": {"rows": rows, "d_in": spec.d_in, "measured_s": q_full,
                            "extrapolated_s": q_pred, "extrapolated_over_measured": q_pred / q_full},
            "cores": threads}


# ------------------------------------------------------------------ reference arm

def run_reference(args, rank, world):
    """The float64 checker (the reference of this path) on the host cores.
    One step = one bounded sample of the workload (see cpu_baseline); the
    line's ms_per_step is the time a sample took, and `value` the full
    layer's rate extrapolated from it by the stages' cost laws."""
    if rank != 0:
        return 0
    threads = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(threads))
    from post_weight_quantization_accumulate_b200 import synth
    spec = synth.WORKLOADS[args.workload if args.workload in synth.WORKLOADS else "q_proj_4096"]
    vals = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(spec, threads)
        if i >= args.warmup:
            vals.append(cb)
    value = statistics.median(v["value"] for v in vals)
    step_ms = statistics.median(v["measured_s"] for v in vals) * 1e3
    layer_s = spec.d_out * spec.d_in / value
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_of(spec, args.gpus),
            "step": "one bounded sample of the layer (ms_per_step is its measured time)",
            "extrapolated_layer_ms": layer_s * 1e3,
            "value_basis": vals[0]["value_basis"],
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if args.validate_cost_laws:
        line["cost_law_check"] = validate_cost_laws(spec, threads)
    print(json.dumps(line), flush=True)
    return 0


def config_of(spec, n):
    return {"workload": spec.name, "d_out": spec.d_out, "d_in": spec.d_in, "n_tokens": spec.n_tokens,
            "bits": spec.bits, "group_size": spec.group_size, "block_size": spec.block_size,
            "damp": spec.damp, "act_order": spec.act_order, "x_dtype": "bf16",
            "w_dtype": "bf16" if spec.w_bf16 else "f32",
            "l2": "inputs larger than L2 (X is %.2f GB)" % (spec.n_tokens * spec.d_in * 2 / 1e9),
            "parallelism": f"independent layer per rank x{n}"}


# ------------------------------------------------------------------ our arm

def run_decoder_layer(args, rank) -> int:
    """Layer-sequential calibration of a Llama-2-7B-shaped decoder layer (all
    seven linears, one Hessian per input group, each group's input produced by
    the quantized earlier groups) on one GPU; one JSON line, rank 0 only."""
    if rank != 0:
        return 0
    import torch
    from post_weight_quantization_accumulate_b200 import build as build_mod
    from post_weight_quantization_accumulate_b200 import decoder as D

    build_mod.build()
    torch.cuda.set_device(0)
    shape = D.LLAMA2_7B
    W, X = D.synthetic_layer(shape)
    combos = [(b, g) for b in (2, 3, 4) for g in (64, 128, -1)] if args.sweep else [(4, 128)]
    cache = {}
    for _ in range(max(1, min(args.warmup, 1))):
        D.calibrate(X, W, shape, bits=4, group_size=128, cache=cache)
    torch.cuda.synchronize()
    rows = []
    for bits, gs in combos:
        ms = []
        for _ in range(max(1, min(args.steps, 3))):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            r = D.calibrate(X, W, shape, bits=bits, group_size=gs, cache=cache)
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        rows.append({"bits": bits, "group_size": gs, "ms": min(ms), "groups_ms": r.ms})
        del r
    n_w = D.quantized_weights(shape)
    best = rows[-1] if not args.sweep else next(r for r in rows if r["bits"] == 4 and r["group_size"] == 128)
    print(json.dumps({
        "metric": "GPTQ quantized weights/s, full decoder layer (7 linears, layer-sequential)",
        "value": n_w / (best["ms"] / 1e3), "unit": "weights/s", "n_gpus": 1,
        "ms_per_layer": best["ms"], "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "llama2_7b_decoder_layer", "d_model": shape.d_model, "d_ff": shape.d_ff,
                   "n_tokens": shape.n_tokens, "weights": n_w,
                   "glue": "vendor bf16 GEMM between groups (not a GPTQ step)"},
        "sweep": rows}), flush=True)
    return 0


W4A16_SHAPES = (("qkv", 12288, 4096), ("o", 4096, 4096), ("gate_up", 22016, 4096), ("down", 4096, 11008))


def run_w4a16(args, rank) -> int:
    """The inference-side consumer of the packed output: one decode step of a
    Llama-2-7B-shaped model's linears (per layer q/k/v fused, o, gate/up
    fused, down; 4-bit codes, group 128) through gptq_w4a16_gemm, over L
    distinct layers whose weights (about 0.46 GB) do not fit in L2.  The
    4 L launches of a step are replayed from a CUDA graph.  value = weight
    bytes streamed per second (codes + scales + zeros); the roofline is HBM."""
    if rank != 0:
        return 0
    import numpy as np
    import torch
    from post_weight_quantization_accumulate_b200 import binding as B
    from post_weight_quantization_accumulate_b200 import build as build_mod
    from post_weight_quantization_accumulate_b200 import synth

    build_mod.build()
    torch.cuda.set_device(0)
    L, gs = 4, 128
    peaks, src = measured_peaks()
    out = {"metric": "W4A16 decode: packed-weight bytes streamed per second (Llama-2-7B linears)",
           "unit": "GB/s", "n_gpus": 1, "higher_is_better": True, "dtype": "bf16 x int4 -> f32",
           "data": "synthetic", "steps": max(args.steps, 400), "warmup": max(3, args.warmup),
           "config": {"workload": "w4a16_llama2_7b_decode", "layers": L, "group_size": gs,
                      "shapes": [list(x) for x in W4A16_SHAPES], "l2": "weights > L2 (0.46 GB)"}}
    lines = {}
    paths = {1: ((B.W4A16_AUTO, "auto"), (B.W4A16_TENSOR_CORE, "tensor_core"), (B.W4A16_GENERAL, "general")),
             16: ((B.W4A16_AUTO, "auto"), (B.W4A16_GENERAL, "general"))}
    for M in (1, 16):
        for path, pname in paths[M]:
            ops, wbytes = [], 0
            for name, N, K in W4A16_SHAPES:
                x, p, sc, z, _ = synth.w4a16_operands(11, M, N, K, gs)
                X = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
                P0, S0, Z0 = (torch.from_numpy(a).cuda() for a in (p, sc, z))
                for _ in range(L):
                    Y = torch.empty(M, N, device="cuda")
                    ops.append((Y, X, P0.clone(), S0.clone(), Z0.clone()))
                    wbytes += P0.numel() + 4 * (S0.numel() + Z0.numel())
                del P0, S0, Z0
            for o in ops[:4]:
                B.gptq_w4a16_gemm(*o, None, gs, path)
            torch.cuda.synchronize()
            n0 = B.gptq_launch_count()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for o in ops:
                    B.gptq_w4a16_gemm(*o, None, gs, path)
            launches = B.gptq_launch_count() - n0
            for _ in range(max(3, args.warmup)):
                g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = max(args.steps, 400)    # long enough for the 100 ms clock samples
            with ClockSampler(0) as clk:
                e0.record()
                for _ in range(reps):
                    g.replay()
                e1.record()
                torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            assert B.gptq_device_status() == 0
            gbs = wbytes / (ms / 1e3) / 1e9
            lines[f"M{M}_{pname}"] = {"ms_per_step": ms, "gbs": gbs, "tokens_per_s": M / (ms / 1e3),
                                      "weight_bytes": wbytes, "launches_per_step": launches,
                                      "frac_of_hbm": gbs / peaks["hbm_gbs"], "clocks": clk.summary()}
            del g, ops
            torch.cuda.empty_cache()
    head = lines["M1_auto"]   # M = 1 takes the decode path, M = 16 the tensor-core path
    out.update({"value": head["gbs"], "ms_per_step": head["ms_per_step"], "gpu_launches": head["launches_per_step"] * max(args.steps, 400),
                "roofline": {"bound": "hbm", "achieved": head["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": head["frac_of_hbm"], "peak_source": src, "traffic": None},
                "clocks": head["clocks"], "vs_baseline": None, "by_case": lines})
    print(json.dumps(out), flush=True)
    return 0


def _timed_layer(q, X, Wd, stream, steps, warmup, barrier, clock_gpu):
    """`steps` timed per-layer steps (H zeroed, Hessian over X, factorisation,
    column loop) after `warmup` untimed ones; returns (ms per step, mean
    Hessian-call ms, launches, clocks)."""
    import torch
    from post_weight_quantization_accumulate_b200 import binding as B
    ev_h = []

    def step(record=False):
        q.reset()
        if record:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        q.add_batch(X)
        if record:
            e1.record(stream)
            ev_h.append((e0, e1))
        q.run(Wd)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    launches0 = B.gptq_launch_count()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(clock_gpu) as clk:
        t_start.record(stream)
        for _ in range(steps):
            step(record=True)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    launches = B.gptq_launch_count() - launches0
    ms = t_start.elapsed_time(t_end) / steps
    h_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_h)
    return ms, h_ms, launches, clk.summary()


def _stages(q, X, Wd, stream):
    """One step broken down by stage (after the timed region), and the column
    loop split into its kernel classes (in-schedule kernel spans)."""
    import torch
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    evs[0].record(stream)
    q.reset()
    q.add_batch(X)
    evs[1].record(stream)
    q.prepare()
    evs[2].record(stream)
    q.quantize(Wd)
    evs[3].record(stream)
    torch.cuda.synchronize()
    stage = {"hessian_ms": evs[0].elapsed_time(evs[1]), "prepare_ms": evs[1].elapsed_time(evs[2]),
             "quantize_ms": evs[2].elapsed_time(evs[3])}
    qt = q.quantize_timed(Wd)
    stage.update({"column_loop_ms": qt[0], "lazy_batch_ms": qt[1], "quantize_other_ms": qt[2]})
    return stage


def _host_inputs(spec):
    """Seeded synthetic X (bf16) and W of the workload in pinned host memory."""
    import numpy as np
    import torch
    from post_weight_quantization_accumulate_b200 import synth
    X_host = torch.empty(spec.n_tokens, spec.d_in, dtype=torch.int16).pin_memory()
    synth.x_bf16(spec, out=X_host.numpy().view(np.uint16))
    X_host = X_host.view(torch.bfloat16)
    wbits = synth.weight_bf16_bits(spec) if spec.w_bf16 else None
    W_host = (torch.from_numpy(wbits.view(np.int16)).view(torch.bfloat16) if spec.w_bf16
              else torch.from_numpy(synth.weight_f32(spec))).pin_memory()
    return X_host, W_host


def by_config_line(name, dev, peaks, peak_kind, steps=2, warmup=1):
    """One other single-GPU workload of the recipe: its step time, stages and
    rooflines (no e2e, no CPU baseline)."""
    import torch
    from post_weight_quantization_accumulate_b200 import binding as B
    from post_weight_quantization_accumulate_b200 import synth
    from post_weight_quantization_accumulate_b200.layer import LayerQuantizer
    spec = synth.WORKLOADS[name]
    X_host, W_host = _host_inputs(spec)
    X, Wd = X_host.to(dev), W_host.to(dev)
    del X_host, W_host
    q = LayerQuantizer(spec.d_out, spec.d_in, spec.bits, spec.group_size, spec.block_size,
                       spec.damp, spec.act_order, device=dev, keep_codes=False)
    stream = torch.cuda.current_stream(dev)
    ms, h_ms, launches, clocks = _timed_layer(q, X, Wd, stream, steps, warmup, lambda: None, dev.index)
    stage = _stages(q, X, Wd, stream)
    status = B.gptq_device_status()
    reg = regime(clocks)
    out = {"workload": name, "config": config_of(spec, 1), "value": spec.d_out * spec.d_in / (ms / 1e3),
           "unit": UNIT, "ms_per_step": ms, "steps": steps, "warmup": warmup,
           "roofline": hessian_roofline(spec, h_ms, clocks, peaks, peak_kind),
           "lazy_batch": lazy_batch_line(spec, stage),
           "layer_roofline": layer_roofline(spec, ms, reg, peaks), "stages_ms": stage,
           "clocks": clocks, "gpu_launches": int(launches), "device_status": status}
    del q, X, Wd
    torch.cuda.empty_cache()
    return out


def decoder_layer_result(bits=4, group_size=128, steps=1, warmup=1):
    """One Llama-2-7B-shaped decoder layer, layer-sequential, on cuda:0."""
    import torch
    from post_weight_quantization_accumulate_b200 import decoder as D
    shape = D.LLAMA2_7B
    W, X = D.synthetic_layer(shape)
    cache = {}   # the layer quantizers of one decoder layer, reused as a model's layers would
    for _ in range(warmup):
        D.calibrate(X, W, shape, bits=bits, group_size=group_size, cache=cache)
    torch.cuda.synchronize()
    ms, r = [], None
    for _ in range(max(1, steps)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        r = D.calibrate(X, W, shape, bits=bits, group_size=group_size, cache=cache)
        b.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    n_w = D.quantized_weights(shape)
    out = {"bits": bits, "group_size": group_size, "ms": min(ms), "groups_ms": r.ms,
           "weights": n_w, "value": n_w / (min(ms) / 1e3), "unit": UNIT}
    del r, W, X, cache
    torch.cuda.empty_cache()
    return out


def hessian_f32_line(dev, peaks, reps=3):
    """gptq_hessian_accumulate_f32 at the q_proj size (262144 x 4096 fp32
    activations, N(0, 1) drawn on the device by a seeded generator) in
    16384-token chunks; its tensor work is four bf16 Hessians of the
    [hi | lo] split, so the roofline counts 4 N d (d + 1) flops."""
    import torch
    from post_weight_quantization_accumulate_b200 import binding as B
    n, d, chunk = 262144, 4096, 16384
    g = torch.Generator(device=dev)
    g.manual_seed(4096)
    X = torch.randn(n, d, generator=g, device=dev, dtype=torch.float32)
    H = torch.zeros(d, d, dtype=torch.float32, device=dev)
    ws = torch.empty(B.gptq_hessian_f32_workspace_bytes(d, chunk), dtype=torch.uint8, device=dev)
    B.gptq_hessian_accumulate_f32(H, X, ws, chunk)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        H.zero_()
        B.gptq_hessian_accumulate_f32(H, X, ws, chunk)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    status = B.gptq_device_status()
    tensor_flops = float(n) * (2 * d) * (2 * d + 1)   # upper triangle of the 2d x 2d block Hessian
    pk = bf16_peaks(peaks)
    del X, H, ws
    torch.cuda.empty_cache()
    return {"workload": "hessian_f32_262144x4096", "ms": ms, "tokens": n, "d_in": d,
            "chunk_tokens": chunk, "tensor_tflops": tensor_flops / (ms / 1e3) / 1e12,
            "frac_of_bf16_burst": tensor_flops / (ms / 1e3) / 1e12 / pk["burst"],
            "note": "tensor work = upper triangle of 2 Z^T Z for Z = [hi | lo] (n x 2d), plus "
                    "the split and fold passes", "device_status": status}


def run_split(args, rank, world, local):
    """One layer over all ranks (--split tokens_rows): token-sharded Hessian,
    one NCCL all-reduce of H, the factorisation on every rank, each rank's
    block of rows.  value = one layer's weights per step time (strong
    scaling); at N = 1 this is the default line's work."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from post_weight_quantization_accumulate_b200 import binding as B
    from post_weight_quantization_accumulate_b200 import build as build_mod
    from post_weight_quantization_accumulate_b200 import ranks, synth
    from post_weight_quantization_accumulate_b200.sharded import ShardedLayer, token_range

    if rank == 0:
        build_mod.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=600))
        dist.barrier()
        if rank != 0:
            build_mod.build()
    B.lib()
    spec = synth.WORKLOADS[args.workload]
    t0, t1 = token_range(spec.n_tokens, rank, world)
    xb = synth.x_bf16(spec, tokens=slice(t0, t1))
    X = torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
    del xb
    W = torch.from_numpy(synth.weight_f32(spec)).to(dev)
    sl = ShardedLayer(spec.d_out, spec.d_in, spec.bits, spec.group_size, spec.block_size, spec.damp,
                      spec.act_order, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        sl.reset()
        sl.add_batch(X)
        sl.prepare()
        sl.quantize(W)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    launches0 = B.gptq_launch_count()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
    barrier()
    launches = B.gptq_launch_count() - launches0
    ms = ranks.max_over_ranks([a.elapsed_time(b) / args.steps], device=dev)[0]
    status = B.gptq_device_status()
    if rank == 0:
        cfg = config_of(spec, world)
        cfg["parallelism"] = f"one layer over {world} ranks: tokens sharded, H all-reduced, rows sharded"
        print(json.dumps({
            "metric": METRIC, "value": spec.d_out * spec.d_in / (ms / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": cfg, "clocks": clk.summary(), "gpu_launches": int(launches),
            "device_status": status, "split": "tokens_rows"}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.workload == "decoder_layer":
        return run_decoder_layer(args, rank)
    if args.workload == "w4a16":
        return run_w4a16(args, rank)
    if args.split == "tokens_rows":
        return run_split(args, rank, world, local)

    import torch
    import torch.distributed as dist
    from post_weight_quantization_accumulate_b200 import binding as B
    from post_weight_quantization_accumulate_b200 import build as build_mod
    from post_weight_quantization_accumulate_b200 import ranks, synth
    from post_weight_quantization_accumulate_b200.layer import LayerQuantizer

    if rank == 0:
        build_mod.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=600))
        dist.barrier()
        if rank != 0:
            build_mod.build()
    B.lib()

    base = synth.WORKLOADS[args.workload]
    spec = ranks.rank_workload(base, rank)          # an independent layer per rank
    threads = len(os.sched_getaffinity(0))

    # inputs: generated on the host, pinned, copied to HBM once
    X_host, W_host = _host_inputs(spec)
    X = X_host.to(dev, non_blocking=False)
    Wd = W_host.to(dev)
    q = LayerQuantizer(spec.d_out, spec.d_in, spec.bits, spec.group_size, spec.block_size,
                       spec.damp, spec.act_order, device=dev, keep_codes=False)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    ms, h_ms, launches, clocks = _timed_layer(q, X, Wd, stream, args.steps, args.warmup, barrier, local)
    status = B.gptq_device_status()
    ms, h_ms = ranks.max_over_ranks([ms, h_ms], device=dev)
    stage = _stages(q, X, Wd, stream) if rank == 0 else {}

    # end to end through the public API with host buffers: X and W copied in
    # (overlapped chunked copy of X), packed codes + scales + zeros + g_idx out
    e2e = None
    if not args.no_e2e:
        packed_h = torch.empty_like(q.packed, device="cpu").pin_memory()
        scales_h = torch.empty_like(q.scales, device="cpu").pin_memory()
        zeros_h = torch.empty_like(q.zeros, device="cpu").pin_memory()
        gidx_h = torch.empty_like(q.g_idx, device="cpu").pin_memory()
        Wd2 = torch.empty_like(Wd)
        w_stream = torch.cuda.Stream(dev)
        ev_w, ev_w_free = torch.cuda.Event(), torch.cuda.Event()

        def e2e_step():
            # X's chunks go up on the library's copy stream as soon as the
            # previous step's accumulations have freed the staging buffers, and
            # W on a stream of its own once the previous step has consumed it:
            # both uploads overlap the previous step's factorisation and
            # column loop.  The factorisation's status is checked by the next
            # prepare (and after the loop).
            q.reset()
            q.add_batch_host(X_host, chunk_tokens=16384)
            w_stream.wait_event(ev_w_free)
            with torch.cuda.stream(w_stream):
                Wd2.copy_(W_host, non_blocking=True)
                ev_w.record(w_stream)
            stream.wait_event(ev_w)
            q.prepare(wait=False)
            res = q.quantize(Wd2)
            ev_w_free.record(stream)
            packed_h.copy_(res.packed, non_blocking=True)
            scales_h.copy_(res.scales, non_blocking=True)
            zeros_h.copy_(res.zeros, non_blocking=True)
            gidx_h.copy_(res.g_idx, non_blocking=True)

        for _ in range(min(args.warmup, 2)):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        q.check()
        e2e_ms = a.elapsed_time(b) / args.steps
        e2e_ms = ranks.max_over_ranks([e2e_ms], device=dev)[0]
        h2d = X_host.numel() * 2 + W_host.numel() * W_host.element_size()
        d2h = (packed_h.numel() + scales_h.numel() * 4 + zeros_h.numel() * 4 + gidx_h.numel() * 4)
        e2e = {"value": ranks.job_rate(world, spec.d_out, spec.d_in, e2e_ms), "unit": UNIT,
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
        del Wd2

    peaks, peak_kind = measured_peaks()
    by_config = None
    if rank == 0 and world == 1 and not args.no_by_config and args.workload == "q_proj_4096":
        del q, X, Wd
        torch.cuda.empty_cache()
        by_config = {}
        for name in ("down_proj_11008", "up_proj_70b"):
            by_config[name] = by_config_line(name, dev, peaks, peak_kind)
        by_config["llama2_7b_decoder_layer_4bit_g128"] = decoder_layer_result()
        by_config["hessian_f32_262144x4096"] = hessian_f32_line(dev, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        os.environ.setdefault("OMP_NUM_THREADS", str(threads))
        cpu = cpu_baseline(spec, threads)

    if rank == 0:
        reg = regime(clocks)
        line = {
            "metric": METRIC, "value": ranks.job_rate(world, spec.d_out, spec.d_in, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config_of(spec, world),
            "roofline": hessian_roofline(spec, h_ms, clocks, peaks, peak_kind),
            "hessian_tflops_dense_equiv": 2 * spec.n_tokens * spec.d_in ** 2 / (h_ms / 1e3) / 1e12,
            "lazy_batch": lazy_batch_line(spec, stage),
            "layer_roofline": layer_roofline(spec, ms, reg, peaks),
            "stages_ms": stage,
            "clocks": clocks, "gpu_launches": int(launches), "device_status": status,
            "e2e": e2e, "cpu_baseline": cpu, "by_config": by_config,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
