"""H = 2 X^T X for float32 activations (the tiny workload's fp32 draw and
ragged shapes) on the device against the float64 checker.  Tolerance: the
Hessian bound of the bf16 path, 1e-5 relative in the Frobenius norm (the split
leaves at most 2^-17 relative per product, the sums are fp32)."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import synth

import parity as P

pytestmark = pytest.mark.gpu


def _gpu_h(x: np.ndarray, chunk: int, H: torch.Tensor | None = None) -> torch.Tensor:
    n, d = x.shape
    X = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    if H is None:
        H = torch.zeros(d, d, dtype=torch.float32, device="cuda")
    ws = torch.empty(B.gptq_hessian_f32_workspace_bytes(d, chunk), dtype=torch.uint8, device="cuda")
    B.gptq_hessian_accumulate_f32(H, X, ws, chunk)
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
    return H


def _x(seed, n, d):
    g = np.random.default_rng(seed)
    x = g.standard_normal((n, d)).astype(np.float32)
    x[:, g.choice(d, size=max(1, d // 64), replace=False)] *= 20.0   # outlier channels
    return x


@pytest.mark.parametrize("n,d,chunk", [(2048, 256, 8192), (5000, 200, 2048), (3000, 1024, 1000)])
def test_hessian_f32_matches_checker(n, d, chunk):
    x = _x(n + d, n, d)
    Hg = _gpu_h(x, chunk).cpu().numpy()
    ref = oracle.hessian_f32(x)
    err = P.rel_fro(Hg, ref)
    assert err <= P.H_RTOL, err
    np.testing.assert_array_equal(Hg, Hg.T)               # bitwise symmetric
    # the low parts are used: rounding X to bf16 first is far less accurate
    assert P.rel_fro(oracle.hessian(synth.f32_to_bf16_bits(x)), ref) > 30 * err


def test_hessian_f32_tiny_workload():
    """The tiny configuration's fp32 activations (2048 tokens x 256)."""
    x = synth.x_f32_unrounded(synth.WORKLOADS["tiny"])
    Hg = _gpu_h(x, 8192).cpu().numpy()
    assert P.rel_fro(Hg, oracle.hessian_f32(x)) <= P.H_RTOL


def test_hessian_f32_accumulates_across_calls():
    x = _x(3, 4096, 256)
    H = _gpu_h(x[:1500], 512)
    H = _gpu_h(x[1500:], 512, H).cpu().numpy()
    assert P.rel_fro(H, oracle.hessian_f32(x)) <= P.H_RTOL


def test_hessian_f32_through_the_layer_wrapper():
    from post_weight_quantization_accumulate_b200.layer import LayerQuantizer
    x = _x(9, 3000, 256)
    q = LayerQuantizer(64, 256)
    q.reset()
    q.add_batch_f32(torch.from_numpy(x).cuda(), chunk_tokens=1024)
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
    assert q.n_tokens == 3000
    assert P.rel_fro(q.H.cpu().numpy(), oracle.hessian_f32(x)) <= P.H_RTOL
