"""Full-size workloads, in the launch configuration the benchmark uses,
checked on sampled outputs the float64 checker computes one by one and on
properties that hold at any size:

  * H: a 24 x 24 block of entries (rows/cols include outlier channels and the
    diagonal) recomputed as 2 sum_t x_ti x_tj over every token; bitwise
    symmetry of the whole matrix;
  * U: sampled columns of U^T U H_d - I (each costs two triangular products);
  * the column loop: sampled rows rerun by the checker with the GPU's U and
    order (codes, grid, W^, output error), and for every row the identity
    sum_c e_c^2 = (w - w^) H_d (w - w^)^T, evaluated on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import synth
from post_weight_quantization_accumulate_b200.layer import LayerQuantizer

import parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"


def _sample_channels(spec, k, seed):
    g = np.random.default_rng(seed)
    f = synth.channel_factors(spec)
    big = np.nonzero(f != 1.0)[0][: k // 3]
    rest = g.choice(spec.d_in, k - big.size, replace=False)
    return np.unique(np.concatenate([big, rest]))[:k]


@pytest.mark.parametrize("name", ["q_proj_4096", "down_proj_11008", "up_proj_70b"])
def test_full_size_layer_sampled(name):
    spec = synth.WORKLOADS[name]
    xb = synth.x_bf16(spec)
    W = synth.weight_f32(spec)
    q = LayerQuantizer(spec.d_out, spec.d_in, spec.bits, spec.group_size, spec.block_size,
                       spec.damp, spec.act_order, keep_err=True)
    q.reset()
    q.add_batch(torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16))
    res = q.run(torch.from_numpy(W).to(DEV))
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0

    # --- H, sampled entries (every token) and symmetry
    Hg = q.H.cpu().numpy()
    assert np.array_equal(Hg, Hg.T)
    idx = _sample_channels(spec, 24, 1)
    blk = oracle.hessian_block(xb, idx, idx)
    scale = np.sqrt(np.outer(np.diag(blk), np.diag(blk)))
    err = np.abs(Hg[np.ix_(idx, idx)] - blk) / scale
    assert err.max() < 1e-5, err.max()
    rel = np.linalg.norm(Hg[np.ix_(idx, idx)] - blk) / np.linalg.norm(blk)
    assert rel <= P.H_RTOL

    # --- U: U^T U H_d e_j = e_j for sampled j (processing order)
    perm = q.perm.cpu().numpy()
    U = q.U.cpu().numpy().astype(np.float64)
    H64 = Hg.astype(np.float64)
    Hd, _ = oracle.damp(H64, spec.damp)
    Hp_cols = Hd[np.ix_(perm, perm[np.asarray([0, 1, spec.d_in // 2, spec.d_in - 2, spec.d_in - 1])])]
    for col_i, j in enumerate([0, 1, spec.d_in // 2, spec.d_in - 2, spec.d_in - 1]):
        v = U.T @ (U @ Hp_cols[:, col_i])
        e = np.zeros(spec.d_in)
        e[j] = 1.0
        assert np.abs(v - e).max() < 2e-3, (j, np.abs(v - e).max())
    if spec.act_order:
        dg = np.diag(Hg)[perm]
        assert np.all(np.diff(dg) <= 0)          # descending order of the GPU's own diag

    # --- sampled rows rerun by the checker with the GPU's U and order
    rows = np.random.default_rng(2).choice(spec.d_out, 24, replace=False)
    rows.sort()
    ref = oracle.quantize(W[rows].astype(np.float64), U, perm, spec.bits, spec.group_size,
                          spec.block_size)
    codes = res.codes.cpu().numpy()[rows]
    scales = res.scales.cpu().numpy()[rows]
    zeros = res.zeros.cpu().numpy()[rows]
    P.check_quantized(codes, scales, zeros, ref, spec.bits, spec.group_size, perm, name)
    What = res.W_hat.cpu().numpy()[rows].astype(np.float64)
    mse_g = oracle.output_mse(W[rows], What, H64, spec.n_tokens)
    mse_r = oracle.output_mse(W[rows], ref["W_hat"], H64, spec.n_tokens)
    P.check_mse(mse_g, mse_r, name)
    # sum e^2 = dW H_d dW^T per sampled row
    dW = (W[rows].astype(np.float64) - What)[:, perm]
    Hp = Hd[np.ix_(perm, perm)]
    lhs = np.einsum("ij,jk,ik->i", dW, Hp, dW)
    np.testing.assert_allclose(res.err_sq.cpu().numpy()[rows], lhs, rtol=5e-3)
    # packed layout and g_idx on the full matrix
    packed = res.packed.cpu().numpy()
    np.testing.assert_array_equal(packed[rows], oracle.pack_int4(codes))
    np.testing.assert_array_equal(res.g_idx.cpu().numpy(), oracle.g_idx(perm, spec.group_size))
