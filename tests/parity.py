"""Comparison helpers shared by the GPU parity tests (no arithmetic of the
method lives here: only element-wise comparisons and the tolerances).

Tolerances (spec bar for this path):
  H          relative Frobenius error <= 1e-5 (fp32 accumulation of exact bf16 products)
  codes      identical on >= 99.9% of entries (2-4 bits; the stated widths);
             every mismatch exactly one level.  For wider codes the bar scales
             with the number of grid levels, 1 - 1e-3 * 2^(bits - 4): with the
             same float32 rounding noise in the compensated weights, the chance
             that a value sits within that noise of a rounding boundary grows
             with 1/scale, i.e. with 2^bits.
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


def code_match_min(bits: int) -> float:
    return CODE_MATCH if bits <= 4 else 1.0 - (1.0 - CODE_MATCH) * 2 ** (bits - 4)


def check_codes(codes_gpu, codes_ref, where="", bits=4, perm=None):
    """codes in original column order; `perm` gives the processing order.

    The first mismatch of a row (processing order) must be exactly one level:
    it is a rounding decision at a grid boundary.  Later ones in the same row
    may be cascades (a different error carried forward); for the stated 2-4
    bit widths every mismatch must still be one level."""
    codes_gpu = np.asarray(codes_gpu).astype(np.int32)
    codes_ref = np.asarray(codes_ref).astype(np.int32)
    if perm is not None:
        codes_gpu, codes_ref = codes_gpu[:, perm], codes_ref[:, perm]
    diff = codes_gpu - codes_ref
    mism = diff != 0
    rate = 1.0 - mism.mean()
    bar = code_match_min(bits)
    print(f"[parity] {where}: code match {rate:.6f} (bar {bar}), mismatches {int(mism.sum())}")
    assert rate >= bar, f"{where}: code match {rate:.6f} < {bar}"
    if mism.any():
        rows = np.nonzero(mism.any(axis=1))[0]
        first = mism[rows].argmax(axis=1)
        assert np.all(np.abs(diff[rows, first]) == 1), f"{where}: a first mismatch is not one level"
        if bits <= 4:
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
