"""Comparison helpers shared by the GPU parity tests (no arithmetic of the
method lives here: only element-wise comparisons and the tolerances).

Tolerances (spec bar for this path):
  H          relative Frobenius error <= 1e-5 (fp32 accumulation of exact bf16 products)
  codes      identical on >= 99.9% of entries; every mismatch exactly one level
  scales/zeros  within 1e-5 relative, except in a row after an earlier code
                mismatch (processing order), which the mismatch explains
  output MSE relative difference <= 0.5%
"""
import numpy as np

H_RTOL = 1e-5
U_RTOL = 1e-4
CODE_MATCH = 0.999
SZ_RTOL = 1e-5
MSE_RTOL = 5e-3


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def check_codes(codes_gpu, codes_ref, where=""):
    codes_gpu = np.asarray(codes_gpu).astype(np.int32)
    codes_ref = np.asarray(codes_ref).astype(np.int32)
    diff = codes_gpu - codes_ref
    mism = diff != 0
    rate = 1.0 - mism.mean()
    assert rate >= CODE_MATCH, f"{where}: code match {rate:.6f} < {CODE_MATCH}"
    if mism.any():
        assert np.abs(diff[mism]).max() == 1, f"{where}: a code differs by more than one level"
    return rate, int(mism.sum())


def check_scales_zeros(s_gpu, z_gpu, s_ref, z_ref, codes_perm_gpu, codes_perm_ref, gs, where=""):
    """s/z are [d_out, n_groups] in processing order; codes_perm in processing order."""
    s_gpu, s_ref = np.asarray(s_gpu, np.float64), np.asarray(s_ref, np.float64)
    z_gpu, z_ref = np.asarray(z_gpu, np.float64), np.asarray(z_ref, np.float64)
    bad = (np.abs(s_gpu - s_ref) > SZ_RTOL * np.abs(s_ref)) | (np.abs(z_gpu - z_ref) > SZ_RTOL * np.maximum(np.abs(z_ref), 1.0))
    if not bad.any():
        return 0
    mism = np.asarray(codes_perm_gpu) != np.asarray(codes_perm_ref)
    d_in = mism.shape[1]
    first = np.where(mism.any(axis=1), mism.argmax(axis=1), d_in)
    rows, groups = np.nonzero(bad)
    g_start = groups * (gs if gs > 0 else d_in)
    # a code mismatch strictly before the group's first column explains it
    unexplained = first[rows] >= g_start
    assert not unexplained.any(), (
        f"{where}: {int(unexplained.sum())} scale/zero differences with no earlier code mismatch; "
        f"first at row {rows[unexplained][0]} group {groups[unexplained][0]}: "
        f"s {s_gpu[rows[unexplained][0], groups[unexplained][0]]} vs {s_ref[rows[unexplained][0], groups[unexplained][0]]}")
    return int(bad.sum())


def check_mse(mse_gpu, mse_ref, where=""):
    rel = abs(mse_gpu - mse_ref) / mse_ref
    assert rel <= MSE_RTOL, f"{where}: output MSE {mse_gpu} vs {mse_ref} (rel {rel:.2e})"
    return rel
