"""Layer-sequential calibration of a decoder layer (TINY shape: d_model 256,
d_ff 512, 2048 tokens), checked stage by stage against the float64 checker:
for every input group, the Hessian of the GPU's input, the factor computed
from the GPU's Hessian, and the codes of each linear computed with the GPU's
factor and order; and the next group's input against a float64 evaluation of
the same glue from the GPU's quantized weights (bf16 roundings at the same
places, so results agree to a bf16 rounding)."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import decoder as D
from post_weight_quantization_accumulate_b200 import synth

import parity as P

pytestmark = pytest.mark.gpu


def _bf16(x: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (nearest even) and back to float64."""
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x.astype(np.float32))).astype(np.float64)


def _np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _rms(x):
    return _bf16(x / np.sqrt((x.astype(np.float32).astype(np.float64) ** 2).mean(axis=1, keepdims=True) + 1e-6))


def _glue_ref(group, X, W_hat):
    """The glue of decoder.next_inputs in float64 with the same bf16 roundings."""
    if group == "qkv":
        return _rms(_bf16(X @ W_hat["v"].T))
    if group == "o":
        return _rms(_bf16(X["qkv"] + _bf16(X["o"] @ W_hat["o"].T)))
    g = _bf16(X @ W_hat["gate"].T)
    u = _bf16(X @ W_hat["up"].T)
    return _bf16(g / (1.0 + np.exp(-g)) * u)


@pytest.mark.parametrize("bits,gs,act_order", [(4, 128, False), (3, 64, True), (2, -1, False)])
def test_decoder_layer_staged_parity(bits, gs, act_order):
    shape = D.TINY
    W, X = D.synthetic_layer(shape)
    r = D.calibrate(X, W, shape, bits=bits, group_size=gs, act_order=act_order, keep_state=True)
    assert B.gptq_device_status() == 0
    nxt = {"qkv": "o", "o": "gate_up", "gate_up": "down"}
    for group, names in D.GROUPS:
        Xg = _np(r.inputs[group])
        # Hessian of the GPU's input
        Hg = r.H[group].cpu().numpy()
        Hr = oracle.hessian(synth.f32_to_bf16_bits(Xg.astype(np.float32)))
        assert P.rel_fro(Hg, Hr) <= P.H_RTOL, group
        # factor from the GPU's Hessian
        perm_r, Ur, Hp, _ = oracle.prepare(Hg.astype(np.float64), 0.01, act_order)
        perm_g = r.perm[group].cpu().numpy()
        np.testing.assert_array_equal(perm_g, perm_r)
        Ug = r.U[group].cpu().numpy()
        assert P.rel_fro(Ug, Ur) <= P.U_RTOL, group
        # codes with the GPU's factor and order
        for name in names:
            ql = r.layers[name]
            Wf = _np(W[name])
            ref = oracle.quantize(Wf, Ug.astype(np.float64), perm_g, bits, gs, 128)
            codes = ql.codes.cpu().numpy()
            scales = ql.scales.cpu().numpy()
            zeros = ql.zeros.cpu().numpy()
            P.check_quantized(codes, scales, zeros, ref, bits, gs, perm_g, f"{group}/{name}")
        # the next group's input from the GPU's quantized weights
        if group in nxt:
            W_hat = {n: _bf16(r.layers[n].W_hat.cpu().numpy().astype(np.float64))
                     for g2, ns in D.GROUPS for n in ns if n in r.layers}
            src = {"qkv": _np(r.inputs["qkv"]), "o": Xg} if group == "o" else Xg
            ref_next = _glue_ref(group, src, W_hat)
            got = _np(r.inputs[nxt[group]])
            scale = np.sqrt((ref_next ** 2).mean())
            # two bf16 ulps of the value, or of the row scale for small entries
            ok = np.abs(got - ref_next) <= 2 ** -7 * np.maximum(np.abs(ref_next), 1e-2 * scale)
            assert ok.mean() >= 0.999, (group, ok.mean())


def test_decoder_weight_count():
    assert D.quantized_weights(D.LLAMA2_7B) == 4 * 4096 * 4096 + 3 * 4096 * 11008
