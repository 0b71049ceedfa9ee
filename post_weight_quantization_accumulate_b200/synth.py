"""Seeded synthetic inputs for the per-layer GPTQ path.

This module only draws random numbers and rounds them to the storage type the
layer uses; it holds none of the quantization arithmetic, so both the CUDA path
and the float64 checker can consume the exact same bytes.

Workload shapes follow the Llama-shaped layers the GPTQ overview page sizes its
complexity claims on ("Złożoność obliczeniowa": O(N_calib * d^2) for the
Hessian, O(d^3) for the inverse).  The pages name no calibration dataset for
this path, so these seeded distributions stand in for calibration activations:

* ``normal``      -- iid N(0,1) per token and channel;
* ``outliers``    -- iid N(0,1) with a fixed set of channels multiplied by a
                     constant factor (activation outlier channels);
* ``lognormal``   -- iid N(0,1) with a fixed 1% of channels multiplied by a
                     per-channel lognormal(0, sigma) factor;
* ``silu_gated``  -- a * SiLU(b) with a, b iid N(0,1) (the input of a gated
                     MLP's down projection).

Streams are generated per 8192-token chunk from
``SeedSequence([seed, tensor_id, chunk])`` so that any chunk (or any sampled
token range) can be regenerated on its own, and chunks can be produced in
parallel threads.  Outlier channel indices and factors come from the separate
child ``SeedSequence([seed, tensor_id, CHANNEL_STREAM])``.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
import os

import numpy as np

CHUNK_TOKENS = 8192
CHANNEL_STREAM = 1 << 30   # child-seed index reserved for per-channel factors
WEIGHT_STREAM = 1 << 29    # child-seed index reserved for weight matrices


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even); return the
    16-bit patterns as uint16.  Inputs here are finite."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class XRecipe:
    kind: str                      # normal | outliers | lognormal | silu_gated
    n_outlier: int = 0             # outliers / lognormal: number of scaled channels
    factor: float = 1.0            # outliers: constant factor
    sigma: float = 0.0             # lognormal: sigma of log(factor)


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer of a workload: W [d_out, d_in], X [n_tokens, d_in]."""
    name: str
    d_out: int
    d_in: int
    n_tokens: int
    w_std: float
    w_bf16: bool                   # W stored as bf16 (else fp32 as-is)
    x: XRecipe
    bits: int
    group_size: int                # -1 = one group per row
    block_size: int = 128
    damp: float = 0.01
    act_order: bool = False
    seed: int = 0
    tensor_id: int = 0
    extra: dict = field(default_factory=dict, compare=False, hash=False)


def _n_channels(d: int, frac: float) -> int:
    return max(1, int(round(d * frac)))


# Workloads.  "tiny" is the small case the checker finishes in seconds.
WORKLOADS = {
    "tiny": LayerSpec("tiny", 256, 256, 2048, 0.02, False,
                      XRecipe("outliers", n_outlier=4, factor=20.0), 4, 128),
    "q_proj_4096": LayerSpec("q_proj_4096", 4096, 4096, 262144, 0.02, True,
                             XRecipe("lognormal", n_outlier=_n_channels(4096, 0.01), sigma=1.5),
                             4, 128),
    "down_proj_11008": LayerSpec("down_proj_11008", 4096, 11008, 131072, 0.02, True,
                                 XRecipe("silu_gated"), 3, 128, act_order=True),
    "up_proj_70b": LayerSpec("up_proj_70b", 28672, 8192, 131072, 0.015, True,
                             XRecipe("outliers", n_outlier=_n_channels(8192, 0.005), factor=30.0),
                             4, 128, act_order=True),
}


def scaled(spec: LayerSpec, **kw) -> LayerSpec:
    """Same recipe at other sizes / quantizer settings (parity-test cases)."""
    d = dict(spec.__dict__)
    d.update(kw)
    if "d_in" in kw and spec.x.n_outlier and "x" not in kw:
        frac = spec.x.n_outlier / spec.d_in
        d["x"] = XRecipe(spec.x.kind, n_outlier=min(kw["d_in"], _n_channels(kw["d_in"], frac)),
                         factor=spec.x.factor, sigma=spec.x.sigma)
    return LayerSpec(**d)


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def channel_factors(spec: LayerSpec) -> np.ndarray:
    """Per-channel multiplicative factors (float32 [d_in]); 1 for ordinary channels."""
    f = np.ones(spec.d_in, dtype=np.float32)
    r = spec.x
    if r.kind in ("outliers", "lognormal") and r.n_outlier > 0:
        g = _rng(spec.seed, spec.tensor_id, CHANNEL_STREAM)
        idx = g.choice(spec.d_in, size=min(r.n_outlier, spec.d_in), replace=False)
        if r.kind == "outliers":
            f[idx] = np.float32(r.factor)
        else:
            f[idx] = g.lognormal(0.0, r.sigma, size=idx.size).astype(np.float32)
    return f


def _x_chunk_f32(spec: LayerSpec, chunk: int, factors: np.ndarray) -> np.ndarray:
    t0 = chunk * CHUNK_TOKENS
    n = min(CHUNK_TOKENS, spec.n_tokens - t0)
    g = _rng(spec.seed, spec.tensor_id, chunk)
    if spec.x.kind == "silu_gated":
        a = g.standard_normal((n, spec.d_in), dtype=np.float32)
        b = g.standard_normal((n, spec.d_in), dtype=np.float32)
        return a * (b / (np.float32(1.0) + np.exp(-b)))
    z = g.standard_normal((n, spec.d_in), dtype=np.float32)
    if spec.x.kind != "normal":
        z *= factors[None, :]
    return z


def x_bf16(spec: LayerSpec, tokens: slice | None = None, threads: int | None = None,
           out: np.ndarray | None = None) -> np.ndarray:
    """Calibration activations as bf16 bit patterns, uint16 [n, d_in] row-major.

    ``tokens`` selects a chunk-aligned or arbitrary token range; the values are
    identical to the same rows of the full tensor.  ``out`` (uint16, right
    shape) is filled in place when given, e.g. a pinned host buffer.
    """
    t_start, t_stop = 0, spec.n_tokens
    if tokens is not None:
        t_start, t_stop, _ = tokens.indices(spec.n_tokens)
    n = t_stop - t_start
    if out is None:
        out = np.empty((n, spec.d_in), dtype=np.uint16)
    assert out.shape == (n, spec.d_in) and out.dtype == np.uint16
    factors = channel_factors(spec)
    c_lo, c_hi = t_start // CHUNK_TOKENS, (t_stop - 1) // CHUNK_TOKENS if n else -1

    def work(c):
        blk = f32_to_bf16_bits(_x_chunk_f32(spec, c, factors))
        g0 = c * CHUNK_TOKENS
        a, b = max(g0, t_start), min(g0 + blk.shape[0], t_stop)
        out[a - t_start:b - t_start] = blk[a - g0:b - g0]

    chunks = range(c_lo, c_hi + 1)
    threads = threads or min(32, len(os.sched_getaffinity(0)))
    if threads > 1 and len(chunks) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, chunks))
    else:
        for c in chunks:
            work(c)
    return out


def x_f32_unrounded(spec: LayerSpec) -> np.ndarray:
    """The float32 draw before bf16 rounding (small workloads only)."""
    factors = channel_factors(spec)
    n_chunks = (spec.n_tokens + CHUNK_TOKENS - 1) // CHUNK_TOKENS
    return np.concatenate([_x_chunk_f32(spec, c, factors) for c in range(n_chunks)], axis=0)


def weight_f32(spec: LayerSpec, rows: slice | None = None) -> np.ndarray:
    """Layer weight W [d_out, d_in] as float32 values (bf16-representable when
    the layer stores bf16 weights).  ``rows`` selects a row range."""
    g = _rng(spec.seed, spec.tensor_id, WEIGHT_STREAM)
    w = g.standard_normal((spec.d_out, spec.d_in), dtype=np.float32) * np.float32(spec.w_std)
    if rows is not None:
        w = w[rows]
    if spec.w_bf16:
        w = bf16_bits_to_f32(f32_to_bf16_bits(w))
    return np.ascontiguousarray(w)


def weight_bf16_bits(spec: LayerSpec) -> np.ndarray:
    assert spec.w_bf16
    return f32_to_bf16_bits(weight_f32(spec))


def random_layer(seed: int, d_out: int, d_in: int, n_tokens: int, *, correlated: bool = True,
                 w_std: float = 0.02):
    """Small random layer for property tests: W float64 and X bf16 bits.

    With ``correlated`` the activations are mixed by a random matrix so that
    the Hessian has off-diagonal mass (the case where compensation matters).
    """
    g = _rng(seed, 7919, d_out, d_in, n_tokens)
    w = (g.standard_normal((d_out, d_in)) * w_std).astype(np.float64)
    z = g.standard_normal((n_tokens, d_in)).astype(np.float32)
    if correlated:
        m = (g.standard_normal((d_in, d_in)) / np.sqrt(d_in)).astype(np.float32)
        m += np.eye(d_in, dtype=np.float32)
        z = z @ m
    return w, f32_to_bf16_bits(z)


def w4a16_operands(seed: int, M: int, N: int, K: int, group_size: int, *, act_order: bool = False):
    """Seeded operands of the 4-bit linear: X bf16 bits [M, K] (the q_proj
    activation recipe: N(0, 1) with 1% of the channels scaled lognormally),
    packed codes uint8 [N, K/2] (uniform random bytes = uniform 4-bit codes),
    float32 scales [N, n_groups] around the size a 0.02-std weight row gives
    at 4 bits (lognormal, median 0.008), integer zeros uniform in 0..15, and
    with act_order a group map g_idx [K] that assigns each group's columns
    to random positions (as the act_order permutation does)."""
    g = _rng(seed, 4016, M, N, K, max(group_size, 0))
    ng = K // group_size if group_size > 0 else 1
    x = g.standard_normal((M, K)).astype(np.float32)
    ch = g.choice(K, size=max(1, K // 100), replace=False)
    x[:, ch] *= np.exp(g.normal(1.5, 0.5, size=ch.size)).astype(np.float32)
    packed = g.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = (0.008 * np.exp(g.normal(0.0, 0.3, size=(N, ng)))).astype(np.float32)
    zeros = g.integers(0, 16, size=(N, ng)).astype(np.float32)
    g_idx = None
    if act_order:
        gs = group_size if group_size > 0 else K
        g_idx = g.permutation(np.arange(K) // gs).astype(np.int32)
    return f32_to_bf16_bits(x), packed, scales, zeros, g_idx
