"""Float64 CPU checker for GPTQ on one linear layer (TEST INFRASTRUCTURE ONLY).

The heavy loops live in gptq_oracle.c (plain C, OpenMP, binary64); this file
loads it with ctypes and composes the steps in the order the GPTQ overview page
(robocikowo.com/technologie-ai/gptq, "Jak działa", "Komponenty",
"Hiperparametry") gives them:

  1. H = 2 X X^T from the layer inputs                     ("Jak działa")
  2. a value added to the Hessian diagonal for stability   ("Hiperparametry")
  3. optional order of columns by activation importance    ("Hiperparametry")
  4. the Cholesky form of the inverse Hessian              ("Komponenty")
  5. column-by-column quantization with OBS compensation,
     one scale per group, block updates                    ("Jak działa")
  6. packed 4-bit storage of the codes (AutoGPTQ page, "Mixed Precision Scheme")

Readings where the pages are silent (each also listed in the design notes):
  * damping amount: lambda * mean(diag H), lambda = 0.01, mean taken before
    any permutation;
  * activation order key: diag(H) of the undamped Hessian, descending, ties by
    lower original index first;
  * groups are consecutive group_size columns in processing order, and a
    group's scale/zero come from the row's current (fully compensated) values;
  * the min/max range always includes 0; an all-zero range is [-1, 1];
    rounding is round-half-to-even; the grid choice and the code decision are
    taken in binary32;
  * group_size = -1 means one (scale, zero) per row from the original row;
  * packed storage: two codes per byte, even column in the low nibble.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gptq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

ORC_OK, ORC_ERR_ARG, ORC_ERR_NOT_PD = 0, 1, 2


class NotPositiveDefinite(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile gptq_oracle.c into liboracle.so (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def configure(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Argument and result types of the checker's C entry points on `lib`."""
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.orc_hessian_accumulate.argtypes = [P, P, I64, I64]
    lib.orc_hessian_block.argtypes = [P, P, I64, I64, P, I64, P, I64]
    lib.orc_inverse_gauss_jordan.argtypes = [P, I64]
    lib.orc_obs_upper.argtypes = [P, I64, P]
    lib.orc_gptq_rows.argtypes = [P, P, I64, I64, ctypes.c_int, I64, I64, P, P, P, P, P, P]
    lib.orc_gptq_rows_q4k.argtypes = [P, P, I64, I64, I64, P, P, P, P, P, P, P, P, P]
    for f in (lib.orc_hessian_accumulate, lib.orc_hessian_block, lib.orc_inverse_gauss_jordan,
              lib.orc_obs_upper, lib.orc_gptq_rows, lib.orc_gptq_rows_q4k):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = configure(ctypes.CDLL(_LIB))
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _check(status: int, what: str):
    if status == ORC_ERR_NOT_PD:
        raise NotPositiveDefinite(what)
    if status != ORC_OK:
        raise ValueError(f"{what}: invalid argument")


# --- 1. Hessian --------------------------------------------------------------

def hessian(x_bits: np.ndarray, H: np.ndarray | None = None) -> np.ndarray:
    """H (+)= 2 * sum_t x_t x_t^T over the rows of X, in float64.

    ``x_bits`` are bf16 bit patterns (uint16 [n, d]); the values are widened
    exactly, so the checker consumes the bytes the kernel consumes."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n, d = x_bits.shape
    if H is None:
        H = np.zeros((d, d), dtype=np.float64)
    assert H.shape == (d, d) and H.dtype == np.float64 and H.flags.c_contiguous
    _check(_load().orc_hessian_accumulate(_ptr(H), _ptr(x_bits), n, d), "hessian")
    return H


def hessian_f32(x: np.ndarray, H: np.ndarray | None = None, chunk: int = 4096) -> np.ndarray:
    """H (+)= 2 * sum_t x_t x_t^T for float32 activations X [n, d] (GPTQ
    overview, "Złożoność obliczeniowa": H = 2 X X^T), in float64.  The binary32
    values are widened exactly; the token sum is a float64 matrix product over
    chunks of rows."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x.shape
    if H is None:
        H = np.zeros((d, d), dtype=np.float64)
    for t0 in range(0, n, chunk):
        xc = x[t0:t0 + chunk].astype(np.float64)
        H += 2.0 * (xc.T @ xc)
    return H


def hessian_block(x_bits: np.ndarray, rows, cols) -> np.ndarray:
    """Entries H[rows][:, cols] of 2 X^T X, each summed directly over tokens."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n, d = x_bits.shape
    I = np.ascontiguousarray(rows, dtype=np.int64)
    J = np.ascontiguousarray(cols, dtype=np.int64)
    out = np.empty((I.size, J.size), dtype=np.float64)
    _check(_load().orc_hessian_block(_ptr(out), _ptr(x_bits), n, d, _ptr(I), I.size,
                                     _ptr(J), J.size), "hessian_block")
    return out


# --- 2./3. damping and activation order --------------------------------------

def damp(H: np.ndarray, lam: float) -> tuple[np.ndarray, float]:
    """H_d = H + lam * mean(diag H) * I.  Raises if mean(diag H) <= 0."""
    mu = float(np.mean(np.diag(H)))
    if not (mu > 0.0) or not np.isfinite(mu):
        raise NotPositiveDefinite("mean(diag H) is not positive")
    Hd = np.array(H, dtype=np.float64, copy=True)
    Hd[np.diag_indices_from(Hd)] += lam * mu
    return Hd, mu


def act_order_perm(H: np.ndarray) -> np.ndarray:
    """Processing order by activation importance: descending diag(H); equal
    keys keep their original order.  perm[k] = original column processed k-th."""
    key = np.diag(H)
    return np.argsort(-key, kind="stable").astype(np.int32)


# --- 4. Cholesky form of the inverse Hessian ---------------------------------

def inverse_gauss_jordan(A: np.ndarray) -> np.ndarray:
    M = np.array(A, dtype=np.float64, copy=True, order="C")
    _check(_load().orc_inverse_gauss_jordan(_ptr(M), M.shape[0]), "inverse")
    return M


def obs_upper(Hinv: np.ndarray) -> np.ndarray:
    Hinv = np.ascontiguousarray(Hinv, dtype=np.float64)
    U = np.empty_like(Hinv)
    _check(_load().orc_obs_upper(_ptr(Hinv), Hinv.shape[0], _ptr(U)), "obs_upper")
    return U


def prepare(H: np.ndarray, lam: float = 0.01, act_order: bool = False):
    """Damp, order, and factor: returns (perm, U, H_d_permuted, mu).

    U is upper triangular with U^T U = (P^T H_d P)^{-1} in processing order."""
    d = H.shape[0]
    Hd, mu = damp(H, lam)
    perm = act_order_perm(H) if act_order else np.arange(d, dtype=np.int32)
    Hp = np.ascontiguousarray(Hd[np.ix_(perm, perm)])
    U = obs_upper(inverse_gauss_jordan(Hp))
    return perm, U, Hp, mu


# --- 5. the column loop ------------------------------------------------------

def gptq_rows(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int, block: int = 0,
              raw: dict | None = None):
    """Column loop on W already in processing order.  Returns
    (W_hat, codes, scales, zeros, E) all in processing order.  With `raw` (a
    dict), also fills raw["qraw"] = w / s and raw["zraw"] = -min / s before
    rounding (how close each integer decision was to a tie)."""
    W = np.array(Wp, dtype=np.float64, copy=True, order="C")
    d_out, d_in = W.shape
    U = np.ascontiguousarray(U, dtype=np.float64)
    assert U.shape == (d_in, d_in)
    ng = (d_in + group_size - 1) // group_size if group_size > 0 else 1
    codes = np.empty((d_out, d_in), dtype=np.uint8)
    scales = np.empty((d_out, ng), dtype=np.float32)
    zeros = np.empty((d_out, ng), dtype=np.float32)
    E = np.empty((d_out, d_in), dtype=np.float64)
    qraw = zraw = None
    if raw is not None:
        qraw = np.empty((d_out, d_in), dtype=np.float32)
        zraw = np.empty((d_out, ng), dtype=np.float32)
        raw["qraw"], raw["zraw"] = qraw, zraw
    _check(_load().orc_gptq_rows(_ptr(W), _ptr(U), d_out, d_in, bits, group_size, block,
                                 _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(E),
                                 _ptr(qraw) if qraw is not None else None,
                                 _ptr(zraw) if zraw is not None else None), "gptq_rows")
    return W, codes, scales, zeros, E


def g_idx(perm: np.ndarray, group_size: int) -> np.ndarray:
    """Group of each original column: g_idx[perm[k]] = k // group_size."""
    d = perm.size
    g = np.empty(d, dtype=np.int32)
    k = np.arange(d)
    g[perm] = (k // group_size) if group_size > 0 else 0
    return g


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_int4: codes [..., 2 * bytes], low nibble first."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def dequant_int4(packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                 g_idx: np.ndarray | None, group_size: int) -> np.ndarray:
    """W^[n][k] = scales[n][g] * (q[n][k] - zeros[n][g]) from the packed 4-bit
    storage (AutoGPTQ page, "Mixed Precision Scheme": int4 weights dequantized
    with their group's scale at inference), g = g_idx[k] when given, else
    k // group_size (group_size -1: one group per row).  The exact product of
    the binary32 scale and the integer q - z, in float64 (as the column loop
    here forms W^)."""
    q = unpack_int4(packed).astype(np.float32)
    K = q.shape[1]
    if g_idx is not None:
        g = np.asarray(g_idx, dtype=np.int64)
    else:
        g = (np.arange(K) // group_size) if group_size > 0 else np.zeros(K, dtype=np.int64)
    s = np.asarray(scales, dtype=np.float32)[:, g].astype(np.float64)
    z = np.asarray(zeros, dtype=np.float32)[:, g].astype(np.float64)
    return s * (q.astype(np.float64) - z)


def w4a16(x_bits: np.ndarray, packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
          g_idx: np.ndarray | None, group_size: int) -> np.ndarray:
    """Y = X W^T in float64 for bf16 activations X [M, K] (bits) and the packed
    4-bit weights [N, K/2] (the inference-side use of the quantized layer)."""
    x = bf16_bits_to_f64(x_bits)
    return x @ dequant_int4(packed, scales, zeros, g_idx, group_size).T


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: column 2i in the low nibble, 2i+1 in the high one."""
    c = np.asarray(codes, dtype=np.uint8)
    assert c.shape[-1] % 2 == 0 and c.max(initial=0) < 16
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def quantize(W: np.ndarray, U: np.ndarray, perm: np.ndarray | None, bits: int,
             group_size: int, block: int = 0) -> dict:
    """GPTQ for one layer, W in original column order.

    Returns original-order codes, dequantized W^ and E (scaled errors), and
    per-group scales/zeros indexed by processing-order group, plus g_idx and
    packed nibbles (bits <= 4, even d_in)."""
    W = np.asarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    if perm is None:
        perm = np.arange(d_in, dtype=np.int32)
    perm = np.asarray(perm, dtype=np.int64)
    raw = {}
    What_p, codes_p, scales, zeros, E_p = gptq_rows(W[:, perm], U, bits, group_size, block, raw)
    codes = np.empty_like(codes_p)
    codes[:, perm] = codes_p
    What = np.empty_like(What_p)
    What[:, perm] = What_p
    out = dict(codes=codes, scales=scales, zeros=zeros, W_hat=What, E_perm=E_p,
               codes_perm=codes_p, g_idx=g_idx(perm, group_size), perm=perm.astype(np.int32),
               qraw_perm=raw["qraw"], zraw=raw["zraw"])
    if bits <= 4 and d_in % 2 == 0:
        out["packed"] = pack_int4(codes)
    return out


def rtn(W: np.ndarray, bits: int, group_size: int) -> dict:
    """Round-to-nearest with the same grid, no compensation, groups over the
    original columns (the baseline GPTQ improves on, page "Rozwiązany problem").
    Written separately from the C column loop, vectorised over rows."""
    W = np.asarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    maxq = np.float32((1 << bits) - 1)
    gs = group_size if group_size > 0 else d_in
    ng = (d_in + gs - 1) // gs
    codes = np.empty((d_out, d_in), dtype=np.uint8)
    scales = np.empty((d_out, ng), dtype=np.float32)
    zeros = np.empty((d_out, ng), dtype=np.float32)
    What = np.empty_like(W)
    for g in range(ng):
        sl = slice(g * gs, min(d_in, (g + 1) * gs))
        v = W[:, sl].astype(np.float32)
        xmin = np.minimum(v.min(axis=1), np.float32(0))
        xmax = np.maximum(v.max(axis=1), np.float32(0))
        flat = xmin == xmax
        xmin = np.where(flat, np.float32(-1), xmin)
        xmax = np.where(flat, np.float32(1), xmax)
        s = ((xmax - xmin) / maxq).astype(np.float32)
        z = np.rint(-xmin / s).astype(np.float32)
        q = np.clip(np.rint(v / s[:, None]) + z[:, None], 0, maxq)
        codes[:, sl] = q.astype(np.uint8)
        scales[:, g] = s
        zeros[:, g] = z
        What[:, sl] = s[:, None].astype(np.float64) * (q.astype(np.float64) - z[:, None])
    return dict(codes=codes, scales=scales, zeros=zeros, W_hat=What)


# --- GPTQ onto the two-level Q4_K grid -----------------------------------------

Q4K_BLOCK, Q4K_SUPER = 32, 256


def gptq_rows_q4k(Wp: np.ndarray, U: np.ndarray, block: int = 0) -> dict:
    """Column loop onto the Q4_K grid (torchao pull request "Add gguf q4_k
    quantization": w = q * block_scale + block_min, 6-bit block scales and
    mins, a super-block scale above them) for W in processing order; see
    orc_gptq_rows_q4k for the parameter choice.  Returns W^ (float64), codes,
    sc6 and m6 [d_out, d_in/32], d and dmin [d_out, d_in/256], E, and the
    decision values before rounding (qraw = (w + o) / s per column, scraw =
    scale / d and mraw = offset / dmin per block), all in processing order."""
    W = np.array(Wp, dtype=np.float64, copy=True, order="C")
    d_out, d_in = W.shape
    U = np.ascontiguousarray(U, dtype=np.float64)
    assert U.shape == (d_in, d_in) and d_in % Q4K_SUPER == 0
    codes = np.empty((d_out, d_in), dtype=np.uint8)
    sc6 = np.empty((d_out, d_in // Q4K_BLOCK), dtype=np.uint8)
    m6 = np.empty((d_out, d_in // Q4K_BLOCK), dtype=np.uint8)
    d = np.empty((d_out, d_in // Q4K_SUPER), dtype=np.float32)
    dmin = np.empty((d_out, d_in // Q4K_SUPER), dtype=np.float32)
    E = np.empty((d_out, d_in), dtype=np.float64)
    qraw = np.empty((d_out, d_in), dtype=np.float32)
    scraw = np.empty((d_out, d_in // Q4K_BLOCK), dtype=np.float32)
    mraw = np.empty((d_out, d_in // Q4K_BLOCK), dtype=np.float32)
    _check(_load().orc_gptq_rows_q4k(_ptr(W), _ptr(U), d_out, d_in, block, _ptr(codes),
                                     _ptr(sc6), _ptr(m6), _ptr(d), _ptr(dmin), _ptr(E),
                                     _ptr(qraw), _ptr(scraw), _ptr(mraw)),
           "gptq_rows_q4k")
    return dict(W_hat=W, codes=codes, sc6=sc6, m6=m6, d=d, dmin=dmin, E=E, qraw=qraw,
                scraw=scraw, mraw=mraw)


def dequant_q4k(codes: np.ndarray, sc6: np.ndarray, m6: np.ndarray, d: np.ndarray,
                dmin: np.ndarray) -> np.ndarray:
    """w^ = d sc q - dmin m for every column (processing order), float64, with
    the products of the binary32 levels formed in binary32 as the grid does."""
    blk = np.arange(codes.shape[1]) // Q4K_BLOCK
    sup = np.arange(codes.shape[1]) // Q4K_SUPER
    s = (d[:, sup] * sc6[:, blk].astype(np.float32)).astype(np.float32)
    o = (dmin[:, sup] * m6[:, blk].astype(np.float32)).astype(np.float32)
    return s.astype(np.float64) * codes.astype(np.float64) - o.astype(np.float64)


def quantize_q4k(W: np.ndarray, U: np.ndarray, perm: np.ndarray | None, block: int = 0) -> dict:
    """GPTQ onto the Q4_K grid for one layer, W in original column order (the
    blocks and super-blocks run over processing order, as groups do)."""
    W = np.asarray(W, dtype=np.float64)
    d_in = W.shape[1]
    perm = np.arange(d_in, dtype=np.int64) if perm is None else np.asarray(perm, dtype=np.int64)
    r = gptq_rows_q4k(W[:, perm], U, block)
    codes = np.empty_like(r["codes"])
    codes[:, perm] = r["codes"]
    What = np.empty_like(r["W_hat"])
    What[:, perm] = r["W_hat"]
    r.update(codes_perm=r["codes"], codes=codes, W_hat_perm=r["W_hat"], W_hat=What,
             perm=perm.astype(np.int32), block_of=g_idx(perm, Q4K_BLOCK))
    return r


# --- metrics -----------------------------------------------------------------

def output_mse(W: np.ndarray, What: np.ndarray, H: np.ndarray, n_tokens: int) -> float:
    """Layer output MSE on the calibration set, ||(W - W^) X^T||^2 / (N d_out),
    through the identity sum_rows dW H dW^T = 2 ||dW X^T||^2 (undamped H)."""
    dW = np.asarray(W, np.float64) - np.asarray(What, np.float64)
    return float(np.einsum("ij,jk,ik->", dW, H, dW) / (2.0 * n_tokens * dW.shape[0]))


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def layer(W: np.ndarray, x_bits: np.ndarray, bits: int, group_size: int, lam: float = 0.01,
          act_order: bool = False, block: int = 0) -> dict:
    """The whole per-layer path from scratch: H, prepare, quantize."""
    H = hessian(x_bits)
    perm, U, Hp, mu = prepare(H, lam, act_order)
    out = quantize(W, U, perm, bits, group_size, block)
    out.update(H=H, U=U, mu=mu,
               mse=output_mse(W, out["W_hat"], H, x_bits.shape[0]))
    return out
