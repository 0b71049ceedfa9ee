"""The 4-bit linear (Y = X W^T from the packed codes, scales, zeros and group
map) on the device against the float64 checker, element by element.

Tolerance, from the arithmetic: every path forms sums of K products of bf16
activations with W^ = s (q - z) (exact in fp32 on the general path; exact bf16
products scaled once per group on the tensor-core path) in fp32, so an output
differs from the exact sum by at most about 2 K u sum_k |x_k W^_k| with
u = 2^-24 (the factor 2 leaves room for an accumulator that truncates).  Wrong
nibbles, groups, scales or a column permutation that does not match give
errors of the order of the sum itself."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import synth
from post_weight_quantization_accumulate_b200.layer import LayerQuantizer

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.view(dtype) if dtype is not None else t


def _run(xb, packed, scales, zeros, g_idx, gs, path):
    M, K = xb.shape
    N = packed.shape[0]
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    B.gptq_w4a16_gemm(Y, _dev(xb.view(np.int16), torch.bfloat16), _dev(packed), _dev(scales),
                      _dev(zeros), None if g_idx is None else _dev(g_idx), gs, path)
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
    return Y.cpu().numpy().astype(np.float64)


def _check(Y, xb, packed, scales, zeros, g_idx, gs, where):
    K = xb.shape[1]
    ref = oracle.w4a16(xb, packed, scales, zeros, g_idx, gs)
    mag = np.abs(synth.bf16_bits_to_f32(xb).astype(np.float64)) @ np.abs(
        oracle.dequant_int4(packed, scales, zeros, g_idx, gs)).T
    err = np.abs(Y - ref)
    bound = 2 * K * U * mag + 1e-30
    assert np.isfinite(Y).all(), where
    worst = float((err / bound).max())
    assert worst <= 1.0, (where, worst)
    return worst


# (M, N, K, group_size): several 128-row tiles and a ragged last tile, stages
# of 128 columns with a ragged last stage, every accumulator width (M padded
# to 16, 32, 64 and a second pass of rows), groups smaller than, equal to and
# larger than a stage, and one group per row
TC_CASES = [
    (1, 384, 1024, 128),
    (5, 200, 1056, 32),
    (16, 256, 768, -1),
    (17, 130, 512, 64),
    (40, 128, 384, 16),
    (70, 260, 640, 128),
    (3, 256, 2048, 256),
    (2, 128, 160, -1),
    (8, 1000, 4096, 128),
]


@pytest.mark.parametrize("M,N,K,gs", TC_CASES)
def test_w4a16_tensor_core_path(M, N, K, gs):
    ops = synth.w4a16_operands(1, M, N, K, gs)
    Y = _run(*ops, gs, B.W4A16_TENSOR_CORE)
    _check(Y, *ops, gs, f"tc {M}x{N}x{K} g{gs}")


# decode path (M <= 4): ragged row counts, groups of 32 .. 256 columns and one
# group per row, a chunk count that is not a multiple of the 32 lanes
# (K = 11008: 344 chunks), every M from 1 to 4
GEMV_CASES = [
    (1, 384, 1024, 128),
    (2, 77, 512, 32),
    (3, 130, 11008, 128),
    (4, 64, 2048, 256),
    (1, 1000, 4096, -1),
    (1, 33, 96, 32),
]


@pytest.mark.parametrize("M,N,K,gs", GEMV_CASES)
def test_w4a16_decode_path(M, N, K, gs):
    ops = synth.w4a16_operands(4, M, N, K, gs)
    Y = _run(*ops, gs, B.W4A16_DECODE)
    _check(Y, *ops, gs, f"decode {M}x{N}x{K} g{gs}")
    # the automatic choice takes the same path for these shapes
    np.testing.assert_array_equal(_run(*ops, gs, B.W4A16_AUTO), Y)


def test_w4a16_decode_path_refuses_what_it_cannot_do():
    ops = synth.w4a16_operands(5, 5, 64, 512, 128)   # M > 4
    with pytest.raises(B.GptqError):
        _run(*ops, 128, B.W4A16_DECODE)
    ops = synth.w4a16_operands(5, 2, 64, 512, 16)    # groups of 16 columns
    with pytest.raises(B.GptqError):
        _run(*ops, 16, B.W4A16_DECODE)


@pytest.mark.parametrize("M,N,K,gs", [(1, 384, 1024, 128), (9, 77, 520, 8), (3, 64, 96, -1)])
def test_w4a16_general_path(M, N, K, gs):
    ops = synth.w4a16_operands(2, M, N, K, gs)
    Y = _run(*ops, gs, B.W4A16_GENERAL)
    _check(Y, *ops, gs, f"general {M}x{N}x{K} g{gs}")


@pytest.mark.parametrize("gs", [128, 32])
def test_w4a16_group_map(gs):
    """act_order layout: groups scattered over the columns through g_idx."""
    ops = synth.w4a16_operands(3, 4, 256, 1024, gs, act_order=True)
    Y = _run(*ops, gs, B.W4A16_AUTO)
    _check(Y, *ops, gs, f"g_idx g{gs}")


def test_w4a16_paths_agree_and_are_deterministic():
    ops = synth.w4a16_operands(4, 16, 512, 2048, 128)
    a = _run(*ops, 128, B.W4A16_TENSOR_CORE)
    b = _run(*ops, 128, B.W4A16_TENSOR_CORE)
    np.testing.assert_array_equal(a, b)          # fixed split-K summation order
    c = _run(*ops, 128, B.W4A16_GENERAL)
    _check(c, *ops, 128, "general")
    _check(a, *ops, 128, "tc")


@pytest.mark.parametrize("M", [1, 16])
def test_w4a16_full_size_q_proj(M):
    """The 4096 x 4096 group-128 layer at the decode batch sizes the bench
    times, every output checked."""
    ops = synth.w4a16_operands(5, M, 4096, 4096, 128)
    Y = _run(*ops, 128, B.W4A16_AUTO)
    _check(Y, *ops, 128, f"q_proj M={M}")


@pytest.mark.parametrize("act_order", [False, True])
def test_w4a16_consumes_the_quantizers_output(act_order):
    """End to end on the device: quantize a layer, then multiply with its
    packed output; the checker dequantizes the same packed bytes."""
    d_out, d_in, gs = 256, 512, 64
    W, xb = synth.random_layer(21, d_out, d_in, 1024, correlated=True)
    q = LayerQuantizer(d_out, d_in, 4, gs, 128, 0.01, act_order)
    q.add_batch(_dev(xb.view(np.int16), torch.bfloat16))
    q.prepare()
    ql = q.quantize(torch.from_numpy(W.astype(np.float32)).cuda())
    packed = ql.packed.cpu().numpy()
    scales = ql.scales.cpu().numpy()
    zeros = ql.zeros.cpu().numpy()
    g_idx = ql.g_idx.cpu().numpy() if act_order else None
    # the packed bytes dequantize to the W^ the quantizer wrote back
    np.testing.assert_array_equal(
        oracle.dequant_int4(packed, scales, zeros, g_idx, gs).astype(np.float32), ql.W_hat.cpu().numpy())
    xq = synth.w4a16_operands(22, 12, 8, d_in, gs)[0]
    Y = _run(xq, packed, scales, zeros, g_idx, gs, B.W4A16_AUTO)
    _check(Y, xq, packed, scales, zeros, g_idx, gs, f"quantizer output act_order={act_order}")
