"""Layer-sequential GPTQ calibration of one decoder layer.

The flow of the torchao issue "GPTQ implementation with tensor subclasses"
("Background"): the activations that reach each linear are collected, the
linear is quantized with GPTQ, and the layer goes on with the quantized weight,
so that the next linear sees the inputs the quantized model will produce.  The
layer has the Llama shape of the pages' complexity discussion (GPTQ overview,
"Złożoność obliczeniowa"): q/k/v/o d_model -> d_model, gate/up d_model -> d_ff,
down d_ff -> d_model.

Linears that read the same input share one Hessian and one factorisation
(input groups qkv, o, gate/up, down).  There are no trained weights here, so
the mixing between the groups is a stand-in for attention and the MLP:

    X_o    = rms(X_attn V^T),  V = W^_v           (each token attends to itself)
    X_mlp  = rms(X_attn + X_o W^_o^T)             (residual stream, normalised)
    X_down = silu(X_mlp W^_gate^T) * (X_mlp W^_up^T)

with rms(x) = x / sqrt(mean_c x_c^2 + 1e-6) per token.  The products use the
quantized weights rounded to bf16, fp32 accumulation and a bf16 result (the
vendor bf16 GEMM through torch: glue between the calls, not a step of the
GPTQ path); every GPTQ step runs in libgptq.so through `LayerQuantizer`.
"""
from __future__ import annotations

import time
from dataclasses import dataclass, field

import numpy as np
import torch

from . import synth
from .layer import LayerQuantizer, QuantizedLayer

GROUPS = (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gate_up", ("gate", "up")), ("down", ("down",)))


@dataclass(frozen=True)
class DecoderShape:
    d_model: int = 4096
    d_ff: int = 11008
    n_tokens: int = 262144
    w_std: float = 0.02
    seed: int = 0

    def linear_shape(self, name: str) -> tuple[int, int]:
        """(d_out, d_in) of a linear."""
        if name in ("q", "k", "v", "o"):
            return self.d_model, self.d_model
        if name in ("gate", "up"):
            return self.d_ff, self.d_model
        return self.d_model, self.d_ff


LLAMA2_7B = DecoderShape()
TINY = DecoderShape(d_model=256, d_ff=512, n_tokens=2048)

_TENSOR_ID = {"x": 100, "q": 101, "k": 102, "v": 103, "o": 104, "gate": 105, "up": 106, "down": 107}


def synthetic_layer(shape: DecoderShape, device="cuda"):
    """Seeded bf16 weights of the seven linears and the layer input X_attn
    (the q_proj recipe: N(0,1) with 1% lognormal-scaled channels)."""
    W = {}
    for name in _TENSOR_ID:
        if name == "x":
            continue
        d_out, d_in = shape.linear_shape(name)
        spec = synth.LayerSpec(name, d_out, d_in, shape.n_tokens, shape.w_std, True,
                               synth.XRecipe("normal"), 4, 128, seed=shape.seed,
                               tensor_id=_TENSOR_ID[name])
        W[name] = torch.from_numpy(synth.weight_bf16_bits(spec).view(np.int16)).to(device).view(
            torch.bfloat16)
    xspec = synth.scaled(synth.WORKLOADS["q_proj_4096"], d_in=shape.d_model, d_out=shape.d_model,
                         n_tokens=shape.n_tokens, seed=shape.seed, tensor_id=_TENSOR_ID["x"])
    X = torch.from_numpy(synth.x_bf16(xspec).view(np.int16)).to(device).view(torch.bfloat16)
    return W, X


def _rms(x: torch.Tensor) -> torch.Tensor:
    xf = x.float()
    return (xf * torch.rsqrt(xf.pow(2).mean(dim=1, keepdim=True) + 1e-6)).to(torch.bfloat16)


def next_inputs(group: str, inputs: dict, W_hat: dict) -> None:
    """The input of the group after `group`, from the quantized weights
    (W_hat: bf16 [d_out, d_in] per linear); stored into `inputs`."""
    if group == "qkv":
        inputs["o"] = _rms(inputs["qkv"] @ W_hat["v"].t())
    elif group == "o":
        inputs["gate_up"] = _rms((inputs["qkv"].float() + (inputs["o"] @ W_hat["o"].t()).float())
                                 .to(torch.bfloat16))
    elif group == "gate_up":
        x = inputs["gate_up"]
        g = (x @ W_hat["gate"].t()).float()
        u = (x @ W_hat["up"].t()).float()
        inputs["down"] = (torch.nn.functional.silu(g) * u).to(torch.bfloat16)


@dataclass
class DecoderResult:
    layers: dict = field(default_factory=dict)      # linear -> QuantizedLayer (own copies)
    inputs: dict = field(default_factory=dict)      # group -> bf16 input X
    H: dict = field(default_factory=dict)           # group -> float32 Hessian (keep_state)
    U: dict = field(default_factory=dict)           # group -> float32 U (keep_state)
    perm: dict = field(default_factory=dict)        # group -> int32 perm (keep_state)
    ms: dict = field(default_factory=dict)          # group -> device ms of its GPTQ calls


def _copy(ql: QuantizedLayer) -> QuantizedLayer:
    c = lambda t: None if t is None else t.clone()
    return QuantizedLayer(c(ql.packed), c(ql.codes), c(ql.scales), c(ql.zeros), c(ql.g_idx),
                          c(ql.perm), c(ql.W_hat), c(ql.err_sq))


def calibrate(X_attn: torch.Tensor, W: dict, shape: DecoderShape, bits: int = 4, group_size: int = 128,
              block_size: int = 128, damp: float = 0.01, act_order: bool = False,
              keep_state: bool = False, cache: dict | None = None) -> DecoderResult:
    """Quantizes the seven linears group by group; each group's Hessian comes
    from the input the earlier (already quantized) groups produce.

    `cache` (a dict the caller keeps between calls) holds the per-shape
    LayerQuantizer buffers, so that repeated calibrations of layers of the
    same shape reuse them -- and the library's CUDA graphs, which are keyed
    by the buffers' addresses -- instead of allocating and capturing anew."""
    res = DecoderResult()
    inputs = {"qkv": X_attn}
    for group, names in GROUPS:
        X = inputs[group]
        d_out, d_in = shape.linear_shape(names[0])
        key = (d_out, d_in, bits, group_size, block_size, damp, act_order, str(X.device))
        q = cache.get(key) if cache is not None else None
        if q is None:
            q = LayerQuantizer(d_out, d_in, bits, group_size, block_size, damp, act_order,
                               device=X.device)
            if cache is not None:
                cache[key] = q
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        q.reset()
        q.add_batch(X)
        q.prepare(wait=False)
        for name in names:
            res.layers[name] = _copy(q.quantize(W[name]))
        q.check()
        ev[1].record()
        if keep_state:
            res.H[group], res.U[group], res.perm[group] = q.H.clone(), q.U.clone(), q.perm.clone()
        W_hat = {n: res.layers[n].W_hat.to(torch.bfloat16) for n in names}
        next_inputs(group, inputs, W_hat)
        torch.cuda.synchronize()
        res.ms[group] = ev[0].elapsed_time(ev[1])
        del q
    res.inputs = inputs
    return res


def quantized_weights(shape: DecoderShape) -> int:
    return sum(int(np.prod(shape.linear_shape(n))) for _, names in GROUPS for n in names)


def run_sweep(shape: DecoderShape, bits_list=(2, 3, 4), group_sizes=(64, 128, -1), device="cuda"):
    """The decoder-layer sweep: one calibration per (bits, group_size); returns
    rows of (bits, group_size, wall ms, per-group device ms)."""
    W, X = synthetic_layer(shape, device)
    rows = []
    for bits in bits_list:
        for gs in group_sizes:
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            r = calibrate(X, W, shape, bits=bits, group_size=gs)
            torch.cuda.synchronize()
            rows.append((bits, gs, (time.perf_counter() - t0) * 1e3, r.ms))
            del r
    return rows
