"""Runs one library call on a synthetic layer, a few times, for profiling.

    python kernel_case.py \
        --call hessian|prepare|quantize|layer --workload q_proj_4096 [--tokens N] [--reps R]
    python kernel_case.py \
        --call w4a16 [--m M] [--n N] [--k K] [--group-size G] [--path 0|1|2] [--reps R]
    python kernel_case.py \
        --call hessian_f32 --workload q_proj_4096 --tokens N [--reps R]

The inputs follow the workload's recipe (see synth.py) with `--tokens`
overriding the calibration size, so a profiler can capture a launch on a case
that is larger than L2 but small in device memory.  Prints the mean CUDA-event
time of the call and the host time spent enqueueing it.
"""
from __future__ import annotations

import argparse
import os
import sys
import time

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from post_weight_quantization_accumulate_b200 import binding as B  # noqa: E402
from post_weight_quantization_accumulate_b200 import synth  # noqa: E402
from post_weight_quantization_accumulate_b200.layer import LayerQuantizer  # noqa: E402


def tf32_peak(n: int = 8192, seconds: float = 3.0):
    """Dense tf32 tensor-core throughput of the vendor GEMM (cuBLAS through
    torch.matmul on float32 with tf32 allowed): a burst (3 products after
    warm-up) and a sustained figure (back-to-back products for `seconds`), the
    denominators of the lazy-batch products' roofline."""
    torch.backends.cuda.matmul.allow_tf32 = True
    dev = torch.device("cuda", 0)
    a = torch.randn(n, n, device=dev)
    b = torch.randn(n, n, device=dev)
    c = torch.empty(n, n, device=dev)
    flop = 2.0 * n ** 3
    for _ in range(3):
        torch.matmul(a, b, out=c)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        torch.matmul(a, b, out=c)
    e1.record()
    torch.cuda.synchronize()
    burst = 3 * flop / (e0.elapsed_time(e1) / 1e3) / 1e12
    reps = max(3, int(seconds / (e0.elapsed_time(e1) / 3e3)))
    e0.record()
    for _ in range(reps):
        torch.matmul(a, b, out=c)
    e1.record()
    torch.cuda.synchronize()
    sustained = reps * flop / (e0.elapsed_time(e1) / 1e3) / 1e12
    print(f"tf32_tflops: {burst:.1f}")
    print(f"tf32_tflops_sustained: {sustained:.1f}")
    print(f"(n = {n}, {reps} products in the sustained loop)")


def w4a16_case(a):
    """gptq_w4a16_gemm on seeded operands; a 256 MB buffer is rewritten before
    every call so that the weights come from HBM, not L2."""
    dev = torch.device("cuda", 0)
    x, p, sc, z, _ = synth.w4a16_operands(7, a.m, a.n, a.k, a.group_size)
    X = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    P, S, Z = (torch.from_numpy(t).to(dev) for t in (p, sc, z))
    Y = torch.empty(a.m, a.n, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ms = []
    for _ in range(a.reps + 1):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        B.gptq_w4a16_gemm(Y, X, P, S, Z, None, a.group_size, a.path)
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    print(f"w4a16 M={a.m} N={a.n} K={a.k} g={a.group_size} path={a.path}: "
          f"{min(ms[1:]) * 1e3:.1f} us/call (cold L2, single launch), status {B.gptq_device_status()}")


def hessian_f32_case(a):
    """gptq_hessian_accumulate_f32 on the workload's fp32 activation draw
    (`--tokens` of them), 8192-token chunks."""
    spec = synth.WORKLOADS[a.workload]
    if a.tokens:
        spec = synth.scaled(spec, n_tokens=a.tokens)
    dev = torch.device("cuda", 0)
    X = torch.from_numpy(synth.x_f32_unrounded(spec)).to(dev)
    H = torch.zeros(spec.d_in, spec.d_in, dtype=torch.float32, device=dev)
    chunk = 8192
    ws = torch.empty(B.gptq_hessian_f32_workspace_bytes(spec.d_in, chunk), dtype=torch.uint8, device=dev)
    B.gptq_hessian_accumulate_f32(H, X, ws, chunk)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        H.zero_()
        B.gptq_hessian_accumulate_f32(H, X, ws, chunk)
    e1.record()
    torch.cuda.synchronize()
    print(f"hessian_f32 {spec.name} tokens={spec.n_tokens}: {e0.elapsed_time(e1) / a.reps:.3f} ms/call "
          f"on the device, status {B.gptq_device_status()}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--call", default="hessian",
                    choices=["hessian", "hessian_f32", "prepare", "quantize", "quantize_q4k", "layer",
                             "tf32_peak", "w4a16"])
    ap.add_argument("--workload", default="q_proj_4096")
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--group-size", type=int, default=128)
    ap.add_argument("--path", type=int, default=0)
    a = ap.parse_args()
    if a.call == "tf32_peak":
        tf32_peak()
        return
    if a.call == "w4a16":
        w4a16_case(a)
        return
    if a.call == "hessian_f32":
        hessian_f32_case(a)
        return
    spec = synth.WORKLOADS[a.workload]
    if a.tokens:
        spec = synth.scaled(spec, n_tokens=a.tokens)
    dev = torch.device("cuda", 0)
    X = torch.from_numpy(synth.x_bf16(spec).view(np.int16)).to(dev).view(torch.bfloat16)
    W = torch.from_numpy(synth.weight_f32(spec)).to(dev)
    q = LayerQuantizer(spec.d_out, spec.d_in, spec.bits, spec.group_size, spec.block_size,
                       spec.damp, spec.act_order, device=dev)
    q.reset()
    q.add_batch(X)
    q.prepare()
    Wq = torch.empty_like(W)
    nb, ns = spec.d_in // 32, max(1, spec.d_in // 256)
    q4k_out = {"sc6": torch.empty(spec.d_out, nb, dtype=torch.uint8, device=dev),
               "m6": torch.empty(spec.d_out, nb, dtype=torch.uint8, device=dev),
               "dsup": torch.empty(spec.d_out, ns, dtype=torch.float32, device=dev),
               "dmin": torch.empty(spec.d_out, ns, dtype=torch.float32, device=dev),
               "scales": torch.empty(spec.d_out, nb, dtype=torch.float32, device=dev),
               "offsets": torch.empty(spec.d_out, nb, dtype=torch.float32, device=dev)}

    def once():
        if a.call == "hessian":
            q.reset()
            q.add_batch(X)
        elif a.call == "prepare":
            q.prepare()
        elif a.call == "quantize":
            q.quantize(W)
        elif a.call == "quantize_q4k":
            Wq.copy_(W)
            B.gptq_quantize_q4k(Wq, q.U, None, q4k_out, q.ws, codes=q.codes)
        else:
            q.reset()
            q.add_batch(X)
            q.run(W)

    once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    t0 = time.perf_counter()
    for _ in range(a.reps):
        once()
    t_host = (time.perf_counter() - t0) / a.reps
    e1.record()
    torch.cuda.synchronize()
    print(f"{a.call} {spec.name} tokens={spec.n_tokens}: {e0.elapsed_time(e1) / a.reps:.3f} ms/call on "
          f"the device, {t_host * 1e3:.3f} ms/call to enqueue on the host, status {B.gptq_device_status()}")


if __name__ == "__main__":
    main()
