"""Comparison helpers shared by the GPU parity tests (no arithmetic of the
method lives here: only element-wise comparisons and the tolerances).

Tolerances of this path (the stated parity bar):
  H          relative Frobenius error <= 1e-5 (fp32 accumulation of exact bf16 products)
  codes      identical on >= 99.9% of entries (2-4 bits; the stated widths);
             every mismatch exactly one level.  Wider codes (up to 8 bits, not
             among the stated widths) are bounded by rows instead: a code that
             sits at a rounding tie (with 2^bits levels, 16 times likelier at 8
             bits than at 4) changes the error carried along the rest of its
             row, so one tie costs up to a row of codes and the share of equal
             entries says little; at most 3% of the rows may diverge, each from
             a tie (checked below for every width).  Measured on the 256 x 512
             8-bit sweep: at most 1.6% of the rows.
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


ROWS_DIVERGING_WIDE = 0.03


def code_match_min(bits: int) -> float:
    """Entry agreement bar of a code width (none beyond the stated widths)."""
    return CODE_MATCH if bits <= 4 else 0.0


TIE_TOL = 1e-3   # a decision value this close to a .5 boundary is a rounding tie


def _near_tie(v):
    v = np.asarray(v, np.float64)
    return np.abs(v - np.floor(v) - 0.5) <= TIE_TOL


def check_quantized(codes_gpu, s_gpu, z_gpu, ref, bits, gs, perm, where=""):
    """GPU codes (original column order) and grid (processing-order groups)
    against the checker's result `ref` (oracle.quantize output).

    Every divergence must be explained.  Walking a row in processing order,
    its first divergence is either a code or a group's zero point whose
    decision value in the checker (w / s, or -min / s) lies within TIE_TOL of
    a rounding tie, off by exactly one level; everything after it in the same
    row may differ (the error carried forward differs).  A scale may differ by
    more than 1e-5 only after such a divergence.  For the stated 2-4 bit
    widths every code mismatch must be one level."""
    d_in = codes_gpu.shape[1]
    cg = np.asarray(codes_gpu).astype(np.int32)[:, perm]
    cr = np.asarray(ref["codes_perm"]).astype(np.int32)
    qraw = ref["qraw_perm"]
    zraw = ref["zraw"]
    sg, sr = np.asarray(s_gpu, np.float64), np.asarray(ref["scales"], np.float64)
    zg, zr = np.asarray(z_gpu, np.float64), np.asarray(ref["zeros"], np.float64)
    diff = cg - cr
    mism = diff != 0
    rate = 1.0 - mism.mean()
    bar = code_match_min(bits)
    gsz = gs if gs > 0 else d_in
    s_bad = np.abs(sg - sr) > SZ_RTOL * np.abs(sr)
    z_bad = zg != zr
    n_rows_div = 0
    ties = 0
    for r in np.nonzero(mism.any(axis=1) | s_bad.any(axis=1) | z_bad.any(axis=1))[0]:
        n_rows_div += 1
        c1 = int(np.argmax(mism[r])) if mism[r].any() else d_in
        g_ev = np.nonzero(s_bad[r] | z_bad[r])[0]
        g1 = int(g_ev[0]) * gsz if g_ev.size else d_in
        if g1 <= c1:                      # first divergence: a group's grid
            g = g1 // gsz
            assert not s_bad[r, g], f"{where}: row {r} group {g}: scale {sg[r, g]} vs {sr[r, g]} with no earlier divergence"
            assert abs(zg[r, g] - zr[r, g]) == 1 and _near_tie(zraw[r, g]), (
                f"{where}: row {r} group {g}: zero {zg[r, g]} vs {zr[r, g]} (checker -min/s = {zraw[r, g]})")
        else:                             # first divergence: a code
            assert abs(diff[r, c1]) == 1 and _near_tie(qraw[r, c1]), (
                f"{where}: row {r} col {c1} (processing order): code {cg[r, c1]} vs {cr[r, c1]} "
                f"(checker w/s = {qraw[r, c1]})")
        ties += 1
    print(f"[parity] {where}: code match {rate:.6f} (bar {bar}), mismatches {int(mism.sum())}, "
          f"rows diverging {n_rows_div} (each from a rounding tie)")
    assert rate >= bar, f"{where}: code match {rate:.6f} < {bar}"
    if bits > 4:
        share = n_rows_div / codes_gpu.shape[0]
        assert share <= ROWS_DIVERGING_WIDE, f"{where}: {share:.4f} of the rows diverge"
    if bits <= 4 and mism.any():
        assert np.abs(diff[mism]).max() == 1, f"{where}: a code differs by more than one level"
    return rate, int(mism.sum())


def check_mse(mse_gpu, mse_ref, where=""):
    rel = abs(mse_gpu - mse_ref) / mse_ref
    assert rel <= MSE_RTOL, f"{where}: output MSE {mse_gpu} vs {mse_ref} (rel {rel:.2e})"
    return rel


def check_q4k(g, ref, perm, where=""):
    """Device outputs of GPTQ onto the two-level Q4_K grid (`g`: codes in
    original column order; sc6, m6, dsup, dmin in processing order) against
    the checker's result `ref` (oracle.quantize_q4k, with its decision values
    qraw, scraw, mraw).

    The same bar as the one-level grid.  Walking a row in processing order,
    its first divergence must be a 6-bit block level (sc6 or m6) or a code
    that differs by exactly one and whose decision value in the checker lies
    within TIE_TOL of a rounding tie; a super-block scale (d or dmin) may
    differ by more than 1e-5 only after such a divergence.  The 4-bit codes
    agree on >= 99.9% of entries and every code mismatch is one level.  The
    6-bit levels, with 64 steps, sit at ties 4 times as often as the codes and
    a divergence carries through the rest of the row's blocks, so they are
    bounded by rows as the wide codes are: at most 3% of the rows diverge,
    each from a tie."""
    d_in = g["codes"].shape[1]
    cg = np.asarray(g["codes"]).astype(np.int32)[:, perm]
    cr = np.asarray(ref["codes_perm"]).astype(np.int32)
    scg, scr = g["sc6"].astype(np.int32), ref["sc6"].astype(np.int32)
    mg, mr = g["m6"].astype(np.int32), ref["m6"].astype(np.int32)
    dg, dr = np.asarray(g["dsup"], np.float64), np.asarray(ref["d"], np.float64)
    dmg, dmr = np.asarray(g["dmin"], np.float64), np.asarray(ref["dmin"], np.float64)
    c_mis = cg != cr
    b_mis = (scg != scr) | (mg != mr)
    s_bad = (np.abs(dg - dr) > SZ_RTOL * np.abs(dr)) | (np.abs(dmg - dmr) > SZ_RTOL * np.abs(dmr))
    rows = np.nonzero(c_mis.any(axis=1) | b_mis.any(axis=1) | s_bad.any(axis=1))[0]
    for r in rows:
        c1 = int(np.argmax(c_mis[r])) if c_mis[r].any() else d_in
        b1 = 32 * int(np.argmax(b_mis[r])) if b_mis[r].any() else d_in
        s1 = 256 * int(np.argmax(s_bad[r])) if s_bad[r].any() else d_in
        assert s1 > min(b1, c1) or s1 == d_in, (
            f"{where}: row {r} super-block {s1 // 256}: d {dg[r, s1 // 256]} / {dr[r, s1 // 256]}, "
            f"dmin {dmg[r, s1 // 256]} / {dmr[r, s1 // 256]} with no earlier divergence")
        if b1 <= c1:                      # first divergence: a block's 6-bit levels
            b = b1 // 32
            for lv_g, lv_r, raw, name in ((scg, scr, ref["scraw"], "sc6"), (mg, mr, ref["mraw"], "m6")):
                if lv_g[r, b] != lv_r[r, b]:
                    assert abs(lv_g[r, b] - lv_r[r, b]) == 1 and _near_tie(raw[r, b]), (
                        f"{where}: row {r} block {b}: {name} {lv_g[r, b]} vs {lv_r[r, b]} "
                        f"(checker raw {raw[r, b]})")
        else:                             # first divergence: a code
            assert abs(cg[r, c1] - cr[r, c1]) == 1 and _near_tie(ref["qraw"][r, c1]), (
                f"{where}: row {r} col {c1} (processing order): code {cg[r, c1]} vs {cr[r, c1]} "
                f"(checker (w + o) / s = {ref['qraw'][r, c1]})")
    rates = {k: 1.0 - float(m.mean()) for k, m in (("codes", c_mis), ("sc6", scg != scr), ("m6", mg != mr))}
    print(f"[parity] {where}: Q4_K match {rates}, rows diverging {rows.size} (each from a rounding tie)")
    assert rates["codes"] >= CODE_MATCH, f"{where}: code match {rates['codes']:.6f} < {CODE_MATCH}"
    share = rows.size / cg.shape[0]
    assert share <= ROWS_DIVERGING_WIDE, f"{where}: {share:.4f} of the rows diverge"
    if c_mis.any():
        assert np.abs(cg - cr)[c_mis].max() == 1, f"{where}: a Q4_K code differs by more than one level"
    return rates
