"""Thin helpers the GPU tests share: run one step of the path through the C
ABI on torch tensors and bring the results back as numpy arrays, and the
staged comparison of the column loop with the float64 checker given the
device's own Hessian, factor and order.  No arithmetic of the method lives
here."""
import numpy as np
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import synth

import parity as P

DEV = "cuda"


def x_dev(xb: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16)


def gpu_hessian(xb: np.ndarray) -> np.ndarray:
    d = xb.shape[1]
    H = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    B.gptq_hessian_accumulate(H, x_dev(xb))
    torch.cuda.synchronize()
    return H.cpu().numpy()


def rand_x(seed, n, d, outliers=0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((n, d)).astype(np.float32)
    if outliers:
        idx = g.choice(d, outliers, replace=False)
        x[:, idx] *= 20
    return synth.f32_to_bf16_bits(x)


def gpu_prepare(Hg: np.ndarray, act_order: bool, damp=0.01):
    d = Hg.shape[0]
    H = torch.from_numpy(np.ascontiguousarray(Hg, dtype=np.float32)).to(DEV)
    U = torch.empty(d, d, dtype=torch.float32, device=DEV)
    perm = torch.empty(d, dtype=torch.int32, device=DEV)
    ws = B.workspace(1, d, 128)
    B.gptq_prepare(H, damp, act_order, perm, U, ws)
    torch.cuda.synchronize()
    return perm.cpu().numpy(), U.cpu().numpy()


def gpu_quantize(W: np.ndarray, Ug: np.ndarray, perm, bits, gs, block):
    d_out, d_in = W.shape
    Wt = torch.from_numpy(np.ascontiguousarray(W, dtype=np.float32)).to(DEV)
    U = torch.from_numpy(np.ascontiguousarray(Ug, dtype=np.float32)).to(DEV)
    pm = torch.from_numpy(perm.astype(np.int32)).to(DEV) if perm is not None else None
    ng = d_in // gs if gs > 0 else 1
    scales = torch.empty(d_out, ng, dtype=torch.float32, device=DEV)
    zeros = torch.empty_like(scales)
    codes = torch.empty(d_out, d_in, dtype=torch.uint8, device=DEV)
    packed = torch.empty(d_out, d_in // 2, dtype=torch.uint8, device=DEV) if bits <= 4 else None
    g_idx = torch.empty(d_in, dtype=torch.int32, device=DEV)
    err = torch.empty(d_out, dtype=torch.float32, device=DEV)
    ws = B.workspace(d_out, d_in, block)
    B.gptq_quantize(Wt, U, pm, bits, gs, block, scales, zeros, ws, codes=codes,
                    packed_int4=packed, g_idx=g_idx, err_sq=err)
    torch.cuda.synchronize()
    return dict(W_hat=Wt.cpu().numpy(), scales=scales.cpu().numpy(), zeros=zeros.cpu().numpy(),
                codes=codes.cpu().numpy(), packed=None if packed is None else packed.cpu().numpy(),
                g_idx=g_idx.cpu().numpy(), err_sq=err.cpu().numpy())


def staged_from_h(W, Hg, n_tokens, bits, gs, block, act_order, where, damp=0.01):
    """GPU column loop vs checker given the GPU's own factor and order of the
    Hessian Hg (float32, as the device holds it)."""
    perm, Ug = gpu_prepare(Hg, act_order, damp)
    g = gpu_quantize(W, Ug, perm if act_order else None, bits, gs, block)
    r = oracle.quantize(W.astype(np.float64), Ug.astype(np.float64), perm, bits, gs, block)
    P.check_quantized(g["codes"], g["scales"], g["zeros"], r, bits, gs, perm, where)
    H64 = Hg.astype(np.float64)
    mse_g = oracle.output_mse(W, g["W_hat"], H64, n_tokens)
    mse_r = oracle.output_mse(W, r["W_hat"], H64, n_tokens)
    P.check_mse(mse_g, mse_r, where)
    # W^ is exactly s (q - z) of the GPU's own codes and grid
    gi = g["g_idx"]
    np.testing.assert_array_equal(gi, oracle.g_idx(perm, gs))
    s = g["scales"][:, gi] if gs > 0 else np.repeat(g["scales"], W.shape[1], axis=1)
    z = g["zeros"][:, gi] if gs > 0 else np.repeat(g["zeros"], W.shape[1], axis=1)
    deq = s * (g["codes"].astype(np.float32) - z)
    np.testing.assert_array_equal(g["W_hat"], deq)
    if g["packed"] is not None:
        np.testing.assert_array_equal(g["packed"], oracle.pack_int4(g["codes"]))
    # |e|^2 per row equals (w - w^) H_d (w - w^)^T in processing order
    Hd, _ = oracle.damp(H64, damp)
    Hp = Hd[np.ix_(perm, perm)]
    dW = (W - g["W_hat"].astype(np.float64))[:, perm]
    lhs = np.einsum("ij,jk,ik->i", dW, Hp, dW)
    np.testing.assert_allclose(g["err_sq"], lhs, rtol=2e-3, atol=1e-12 * lhs.max())
    return g, r, perm, Ug


def staged_check(W, xb, bits, gs, block, act_order, where):
    """GPU column loop vs checker given the GPU's own H, U and order."""
    return staged_from_h(W, gpu_hessian(xb), xb.shape[0], bits, gs, block, act_order, where)[:2]
