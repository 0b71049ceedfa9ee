"""The Python binding refuses wrong dtypes and shapes before it calls into
the library (no device needed)."""
import pytest
import torch

from post_weight_quantization_accumulate_b200 import binding as B


def test_w4a16_binding_checks():
    Y = torch.empty(2, 8)
    X = torch.empty(2, 16, dtype=torch.bfloat16)
    packed = torch.empty(8, 8, dtype=torch.uint8)
    s = torch.empty(8, 1)
    with pytest.raises(TypeError):
        B.gptq_w4a16_gemm(Y.double(), X, packed, s, s, None, -1)
    with pytest.raises(TypeError):
        B.gptq_w4a16_gemm(Y, X.float(), packed, s, s, None, -1)
    with pytest.raises(TypeError):
        B.gptq_w4a16_gemm(Y, X, packed.to(torch.int8), s, s, None, -1)
    with pytest.raises(ValueError):
        B.gptq_w4a16_gemm(torch.empty(2, 9), X, packed, s, s, None, -1)     # Y is not [M, N]
    with pytest.raises(ValueError):
        B.gptq_w4a16_gemm(Y, X, torch.empty(8, 4, dtype=torch.uint8), s, s, None, -1)   # K / 2


def test_hessian_and_quantize_binding_checks():
    H = torch.empty(16, 16)
    with pytest.raises(TypeError):
        B.gptq_hessian_accumulate_f32(H, torch.empty(4, 16, dtype=torch.bfloat16), torch.empty(1))
    with pytest.raises(TypeError):
        B.gptq_hessian_accumulate_f32(H.double(), torch.empty(4, 16), torch.empty(1))
    with pytest.raises(TypeError):
        B.gptq_quantize_q4k(torch.empty(4, 256, dtype=torch.float64), H, None, {}, torch.empty(1))
    with pytest.raises(TypeError):
        B.gptq_bf16_to_f32(torch.empty(4), torch.empty(4))                  # src not bf16
    with pytest.raises(ValueError):
        B.gptq_bf16_to_f32(torch.empty(4), torch.empty(5, dtype=torch.bfloat16))


def test_non_contiguous_tensors_are_refused():
    with pytest.raises(ValueError):
        B._ptr(torch.empty(8, 8).t())
