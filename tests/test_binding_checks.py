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


def test_q4k_binding_checks_output_dtypes():
    W = torch.empty(4, 256)
    good = {"sc6": torch.empty(4, 8, dtype=torch.uint8), "m6": torch.empty(4, 8, dtype=torch.uint8),
            "dsup": torch.empty(4, 1), "dmin": torch.empty(4, 1),
            "scales": torch.empty(4, 8), "offsets": torch.empty(4, 8)}
    for k in good:
        bad = dict(good)
        bad[k] = good[k].double() if good[k].dtype == torch.float32 else good[k].to(torch.int8)
        with pytest.raises(TypeError):
            B.gptq_quantize_q4k(W, torch.empty(256, 256), None, bad, torch.empty(1))


def test_layer_wrappers_reach_the_library_boundary(monkeypatch):
    """On a machine without a GPU the high-level wrappers get as far as the
    library, which refuses the call (no device); no Python-side error first.
    (The stream lookup, which needs a driver, is replaced by the null stream.)"""
    import ctypes
    from post_weight_quantization_accumulate_b200.layer import LayerQuantizer
    if torch.cuda.is_available():
        pytest.skip("checks the device-less refusal")
    monkeypatch.setattr(B, "_stream", lambda t, stream=None: ctypes.c_void_p(None))
    q = LayerQuantizer(32, 256, device="cpu")
    with pytest.raises(B.GptqError):
        q.quantize_q4k(torch.zeros(32, 256))
    with pytest.raises(B.GptqError):
        q.add_batch_f32(torch.zeros(16, 256))
    with pytest.raises(ValueError):
        LayerQuantizer(32, 264, device="cpu").quantize_q4k(torch.zeros(32, 264))
