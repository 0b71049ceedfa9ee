"""The method's degenerate cases on the device, element by element against the
float64 checker (or an exact invariant), under the same bar as the other
parity tests:

  * dead input channels (diag H = 0): no special case; damping keeps H_d
    positive definite and such a column is rounded with no compensation;
  * all-zero rows and all-zero groups: the grid of an all-zero range is
    [-1, 1];
  * act_order with exactly tied diagonal values: the order is descending
    diag(H) with ties in increasing column index, identical to the checker's;
  * power-of-two invariances of the whole path on the device: H * 2^k (k even)
    leaves every output bitwise unchanged, W * 2^k scales the scales and W^
    exactly and keeps the codes and zeros;
  * groups whose range is so small that 1 / s overflows binary32 (subnormal
    scales): the codes are still decided as IEEE division decides them;
  * bitwise reproducibility of a whole layer (Hessian with several token
    spans per tile, factorisation, column loop) from run to run;
  * two factorisations issued concurrently from two host threads on two
    streams give the results of two serial calls.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import synth
from post_weight_quantization_accumulate_b200.layer import LayerQuantizer

import parity as P
from gpu_steps import DEV, gpu_hessian, gpu_prepare, gpu_quantize, staged_from_h, x_dev

pytestmark = pytest.mark.gpu


def _inverse(perm):
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=perm.dtype)
    return inv


# ------------------------------------------------------------- dead channels

@pytest.mark.parametrize("act_order", [False, True])
def test_dead_input_channels(act_order):
    d_out, d_in, n = 128, 512, 2048
    W, xb = synth.random_layer(91, d_out, d_in, n, correlated=True)
    dead = np.array([3, 200, 511])
    xb = xb.copy()
    xb[:, dead] = 0                                   # +0.0 in bf16
    Hg = gpu_hessian(xb)
    assert (Hg[dead] == 0).all() and (Hg[:, dead] == 0).all()
    g, r, perm, Ug = staged_from_h(W, Hg, n, 4, 128, 128, act_order, f"dead channels ao{act_order}")
    # a dead column's factor row and column hold only the diagonal 1 / sqrt(damp mean diag H)
    pos = _inverse(perm)[dead]
    if act_order:   # diag 0 sorts last, ties by column index
        np.testing.assert_array_equal(pos, np.arange(d_in - 3, d_in))
    delta = np.float32(0.01) * np.float32(np.mean(np.diag(Hg).astype(np.float64)))
    for k in pos:
        off = np.delete(Ug[k], k)
        assert (off == 0).all() and (np.delete(Ug[:, k], k) == 0).all()
        assert abs(Ug[k, k] - 1.0 / np.sqrt(np.float64(delta))) <= 1e-5 * Ug[k, k]


# ------------------------------------------------------ zero rows and groups

@pytest.mark.parametrize("bits,gs,act_order", [(4, 128, False), (3, 32, True), (2, -1, False), (4, 64, True)])
def test_zero_rows_and_zero_groups(bits, gs, act_order):
    d_out, d_in, n = 96, 512, 2048
    W, xb = synth.random_layer(92 + bits, d_out, d_in, n, correlated=True)
    zero_rows = [0, 17, 95]
    W[zero_rows] = 0.0
    g0 = gs if gs > 0 else 64
    W[5, :g0] = 0.0                 # the first group of a row (no compensation reaches it yet)
    W[6, 128:128 + g0] = 0.0        # a later group (compensated before its start)
    W[7, -g0:] = 0.0
    Hg = gpu_hessian(xb)
    g, r, perm, _ = staged_from_h(W, Hg, n, bits, gs, 128, act_order, f"zero rows/groups b{bits} g{gs}")
    maxq = np.float32((1 << bits) - 1)
    s_flat = np.float32(2.0) / maxq                   # the range [-1, 1]
    z_flat = np.rint(np.float32(1.0) / s_flat)
    assert (g["scales"][zero_rows] == s_flat).all() and (g["zeros"][zero_rows] == z_flat).all()
    assert (g["W_hat"][zero_rows] == 0).all()
    assert (g["codes"][zero_rows] == z_flat).all()
    if not act_order and gs > 0:
        assert g["scales"][5, 0] == s_flat and g["zeros"][5, 0] == z_flat


# ------------------------------------------------------------ act_order ties

def test_act_order_exact_ties_follow_the_stable_order():
    d, d_out = 384, 64
    rng = np.random.default_rng(93)
    A = rng.standard_normal((d, 2 * d))
    H = (A @ A.T) / (2 * d)
    H = ((H + H.T) / 2).astype(np.float32)
    # sets of channels with bitwise-equal diagonals (raising a diagonal entry
    # keeps H positive definite), including a tie at the top of the order
    top = int(np.argmax(np.diag(H)))
    sets = [rng.choice(d, 5, replace=False), rng.choice(d, 3, replace=False),
            np.array([top, (top + 7) % d, (top + 100) % d])]
    for st in sets:
        v = np.diag(H)[st].max()
        H[st, st] = v
    perm_g, _ = gpu_prepare(H, True)
    perm_r = oracle.act_order_perm(H.astype(np.float64))
    np.testing.assert_array_equal(perm_g, perm_r)
    for st in sets:   # tied channels are processed in increasing column index
        pos = _inverse(perm_g)[np.sort(st)]
        assert (np.diff(pos) > 0).all()
    W = rng.standard_normal((d_out, d)) * 0.02
    staged_from_h(W, H, 1, 4, 128, 128, True, "act_order ties")


# --------------------------------------------------- power-of-two invariance

def test_power_of_two_invariance_on_device():
    """P-g on the device.  Scaling H by 2^k (k even) scales U by 2^(-k/2)
    exactly and leaves codes, grid and W^ bitwise unchanged; scaling W by 2^k
    scales the scales and W^ by 2^k exactly and leaves codes and zeros
    unchanged -- down to group ranges far below 2^-60, where the quotient's
    operands are lifted before the division-free rounding."""
    d_out, d_in, n = 128, 512, 2048
    W, xb = synth.random_layer(94, d_out, d_in, n, correlated=True)
    W = W.astype(np.float32)
    Hg = gpu_hessian(xb)
    p0, U0 = gpu_prepare(Hg, True)
    g0 = gpu_quantize(W, U0, p0, 4, 128, 128)
    for k in (-60, -2, 2, 60):
        f = np.float32(2.0 ** k)
        pk, Uk = gpu_prepare(Hg * f, True)
        np.testing.assert_array_equal(pk, p0)
        np.testing.assert_array_equal(Uk, U0 * np.float32(2.0 ** (-k // 2)), err_msg=f"U, H * 2^{k}")
        gk = gpu_quantize(W, Uk, pk, 4, 128, 128)
        for key in ("codes", "scales", "zeros", "W_hat", "packed"):
            np.testing.assert_array_equal(gk[key], g0[key], err_msg=f"{key}, H * 2^{k}")
        np.testing.assert_array_equal(gk["err_sq"], g0["err_sq"] * f, err_msg=f"err_sq, H * 2^{k}")
    for k in (-80, -62, -20, 20, 60, 100):
        f = np.float32(2.0 ** k)
        gk = gpu_quantize(W * f, U0, p0, 4, 128, 128)
        for key in ("codes", "zeros", "packed"):
            np.testing.assert_array_equal(gk[key], g0[key], err_msg=f"{key}, W * 2^{k}")
        np.testing.assert_array_equal(gk["scales"], g0["scales"] * f, err_msg=f"scales, W * 2^{k}")
        np.testing.assert_array_equal(gk["W_hat"], g0["W_hat"] * f, err_msg=f"W_hat, W * 2^{k}")
        if abs(k) <= 40:
            np.testing.assert_array_equal(gk["err_sq"], g0["err_sq"] * f * f, err_msg=f"err_sq, W * 2^{k}")


# ------------------------------------------------------- tiny-range groups

def _tiny_range_layer(seed, d_out=64, d_in=512):
    """Weights whose groups span every magnitude: ordinary values, values near
    2^-100 (scales below 2^-60), and normal values in [2^-126, 1.7 * 2^-126]
    with mixed signs, whose range / 15 is a subnormal scale whose reciprocal
    overflows binary32.  Rows 0..15 are tiny as a whole (per-row grids);
    later rows mix tiny and ordinary 128-column blocks and 8-column chunks."""
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((d_out, d_in)) * 0.02

    def tiny(shape):
        return rng.choice([-1.0, 1.0], shape) * rng.uniform(1.0, 1.7, shape) * 2.0 ** -126

    for r in range(16):
        W[r] = tiny(d_in) if r % 2 == 0 else W[r] * 2.0 ** -100
    for r in range(16, 40):
        for b in range(0, d_in, 128):
            m = rng.integers(3)
            if m == 1:
                W[r, b:b + 128] = tiny(128)
            elif m == 2:
                W[r, b:b + 128] *= 2.0 ** -100
    for r in range(40, d_out):
        for b in range(0, d_in, 8):
            if rng.integers(2):
                W[r, b:b + 8] = tiny(8)
    return W.astype(np.float32)


@pytest.mark.parametrize("gs", [128, 8, -1])
def test_tiny_range_groups_are_decided_like_ieee_division(gs):
    """With a diagonal H nothing is compensated, so the codes and grid must be
    exactly those of round-to-nearest decided with IEEE binary32 division,
    also where the scale is subnormal (1 / s = inf in binary32)."""
    W = _tiny_range_layer(95)
    d_in = W.shape[1]
    H = np.diag(np.random.default_rng(96).uniform(0.5, 5.0, d_in)).astype(np.float32)
    perm, Ug = gpu_prepare(H, False)
    g = gpu_quantize(W, Ug, None, 4, gs, 128)
    rt = oracle.rtn(W.astype(np.float64), 4, gs)
    s = rt["scales"]
    with np.errstate(over="ignore", divide="ignore"):
        assert (s < 2.0 ** -126).any() and (np.float32(1.0) / s == np.inf).any()   # reached
    np.testing.assert_array_equal(g["codes"], rt["codes"])
    np.testing.assert_array_equal(g["scales"], rt["scales"])
    np.testing.assert_array_equal(g["zeros"], rt["zeros"])


def test_tiny_range_blocks_on_the_q4k_grid():
    """The Q4_K grid's quotient (w + o) / (d sc) under the same tiny ranges,
    with no compensation: codes and every level exactly as the checker."""
    W = _tiny_range_layer(97, d_out=48, d_in=512)
    d_out, d_in = W.shape
    H = np.diag(np.random.default_rng(98).uniform(0.5, 5.0, d_in)).astype(np.float32)
    _, Ug = gpu_prepare(H, False)
    Wt = torch.from_numpy(W).to(DEV)
    nb, ns = d_in // 32, d_in // 256
    out = {"sc6": torch.empty(d_out, nb, dtype=torch.uint8, device=DEV),
           "m6": torch.empty(d_out, nb, dtype=torch.uint8, device=DEV),
           "dsup": torch.empty(d_out, ns, dtype=torch.float32, device=DEV),
           "dmin": torch.empty(d_out, ns, dtype=torch.float32, device=DEV),
           "scales": torch.empty(d_out, nb, dtype=torch.float32, device=DEV),
           "offsets": torch.empty(d_out, nb, dtype=torch.float32, device=DEV)}
    codes = torch.empty(d_out, d_in, dtype=torch.uint8, device=DEV)
    B.gptq_quantize_q4k(Wt, torch.from_numpy(Ug).to(DEV), None, out, B.workspace(d_out, d_in, 128),
                        codes=codes)
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
    ref = oracle.quantize_q4k(W.astype(np.float64), Ug.astype(np.float64), None)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref["codes"])
    for k, rk in (("sc6", "sc6"), ("m6", "m6"), ("dsup", "d"), ("dmin", "dmin")):
        np.testing.assert_array_equal(out[k].cpu().numpy(), ref[rk], err_msg=k)


# ------------------------------------------------------- reproducibility

def test_full_layer_runs_are_bitwise_reproducible():
    """Two runs of a whole layer from the same inputs give the same bits:
    the Hessian (5 token spans per tile here, flushed in a fixed order), the
    order and factor, and every output of the column loop."""
    d_out, d_in, n = 256, 768, 20000
    W, xb = synth.random_layer(99, d_out, d_in, n, correlated=True)
    X = x_dev(xb)
    runs = []
    for _ in range(2):
        q = LayerQuantizer(d_out, d_in, 4, 128, 128, 0.01, True, keep_err=True)
        q.reset()
        q.add_batch(X)
        res = q.run(torch.from_numpy(W.astype(np.float32)).to(DEV))
        torch.cuda.synchronize()
        assert B.gptq_device_status() == 0
        runs.append({"H": q.H.cpu().numpy(), "U": q.U.cpu().numpy(), "perm": q.perm.cpu().numpy(),
                     "codes": res.codes.cpu().numpy(), "scales": res.scales.cpu().numpy(),
                     "zeros": res.zeros.cpu().numpy(), "W_hat": res.W_hat.cpu().numpy(),
                     "err_sq": res.err_sq.cpu().numpy()})
    for k in runs[0]:
        np.testing.assert_array_equal(runs[0][k], runs[1][k], err_msg=k)
    Hg = runs[0]["H"]
    assert np.array_equal(Hg, Hg.T)
    assert P.rel_fro(Hg, oracle.hessian(xb)) <= P.H_RTOL


# ------------------------------------------------------ concurrent prepares

def test_concurrent_prepares_match_serial_runs():
    """Two host threads, each on its own stream, factorise different
    Hessians at the same time; the results equal those of serial calls."""
    Hs = [gpu_hessian(synth.random_layer(100 + i, 8, d, 2 * d, correlated=True)[1])
          for i, d in enumerate((512, 1024))]
    serial = [gpu_prepare(H, True) for H in Hs]
    results = [[None] * 3 for _ in Hs]
    errors = []

    def worker(i):
        try:
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                d = Hs[i].shape[0]
                H = torch.from_numpy(Hs[i]).to(DEV)
                ws = B.workspace(1, d, 128)
                stream.synchronize()
                for rep in range(3):
                    U = torch.empty(d, d, dtype=torch.float32, device=DEV)
                    perm = torch.empty(d, dtype=torch.int32, device=DEV)
                    B.gptq_prepare(H, 0.01, True, perm, U, ws)
                    stream.synchronize()
                    results[i][rep] = (perm.cpu().numpy(), U.cpu().numpy())
        except Exception as e:  # reported in the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert B.gptq_device_status() == 0
    for i, (perm_s, U_s) in enumerate(serial):
        for perm_c, U_c in results[i]:
            np.testing.assert_array_equal(perm_c, perm_s)
            np.testing.assert_array_equal(U_c, U_s)
