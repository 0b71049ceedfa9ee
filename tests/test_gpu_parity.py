"""GPU path vs the float64 checker, element by element, on seeded inputs.

Staged as in the design notes: the Hessian against the checker's H from the
same bf16 bytes; the factor U against the checker's OBS elimination of the
GPU's own H; the column loop against the checker given the GPU's U and order;
and the whole path from scratch against the checker's own H, U and order.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import synth
from post_weight_quantization_accumulate_b200.layer import LayerQuantizer

import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"

from gpu_steps import gpu_hessian as _gpu_hessian  # noqa: E402
from gpu_steps import gpu_prepare as _gpu_prepare  # noqa: E402
from gpu_steps import gpu_quantize as _gpu_quantize  # noqa: E402
from gpu_steps import rand_x as _rand_x  # noqa: E402
from gpu_steps import staged_check as _staged_check  # noqa: E402
from gpu_steps import x_dev as _x_dev  # noqa: E402


# --------------------------------------------------------------------- Hessian

@pytest.mark.parametrize("n,d", [(2048, 256), (1000, 200), (4097, 392), (63, 8), (64, 64),
                                 (8192 + 77, 520), (20000, 1024)])
def test_hessian_matches_checker(n, d):
    xb = _rand_x(n * 7 + d, n, d, outliers=min(4, d // 8))
    Hg = _gpu_hessian(xb)
    Hr = oracle.hessian(xb)
    assert np.array_equal(Hg, Hg.T), "H must be bitwise symmetric"
    assert P.rel_fro(Hg, Hr) <= P.H_RTOL
    # every entry, relative to the scale of its row/column
    scale = np.sqrt(np.outer(np.diag(Hr), np.diag(Hr))) + 1e-30
    assert np.max(np.abs(Hg - Hr) / scale) < 1e-5


def test_hessian_tiny_workload_and_chunked_accumulation():
    spec = synth.WORKLOADS["tiny"]
    xb = synth.x_bf16(spec)
    Hr = oracle.hessian(xb)
    H = torch.zeros(256, 256, dtype=torch.float32, device=DEV)
    for a, b in [(0, 700), (700, 701), (701, 2048)]:
        B.gptq_hessian_accumulate(H, _x_dev(xb[a:b]))
    torch.cuda.synchronize()
    Hg = H.cpu().numpy()
    assert np.array_equal(Hg, Hg.T)
    assert P.rel_fro(Hg, Hr) <= P.H_RTOL


def test_hessian_host_streaming_matches_device():
    xb = _rand_x(5, 5000, 256, 4)
    Hd = _gpu_hessian(xb)
    H = torch.zeros(256, 256, dtype=torch.float32, device=DEV)
    Xh = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    staging = torch.empty(2 * 1024 * 256, dtype=torch.bfloat16, device=DEV)
    B.gptq_hessian_accumulate_host(H, Xh, staging, 1024)
    torch.cuda.synchronize()
    Hh = H.cpu().numpy()
    assert np.array_equal(Hh, Hh.T)
    assert P.rel_fro(Hh, Hd) <= 1e-6
    assert P.rel_fro(Hh, oracle.hessian(xb)) <= P.H_RTOL


def test_hessian_host_streaming_back_to_back_calls():
    """Calls that share the staging buffers, enqueued without a synchronise in
    between (the second call's uploads wait only for the first call's
    accumulations): each H equals the device-resident result bit for bit, and
    a kernel queued on the stream between the calls does not hold them up."""
    xa, xc = _rand_x(6, 3000, 256, 2), _rand_x(7, 4100, 256, 3)
    staging = torch.empty(2 * 512 * 256, dtype=torch.bfloat16, device=DEV)
    Ha = torch.zeros(256, 256, dtype=torch.float32, device=DEV)
    Hc = torch.zeros(256, 256, dtype=torch.float32, device=DEV)
    Xa = torch.from_numpy(xa.view(np.int16)).view(torch.bfloat16).pin_memory()
    Xc = torch.from_numpy(xc.view(np.int16)).view(torch.bfloat16).pin_memory()
    # references: one call at a time, the same chunks
    B.gptq_hessian_accumulate_host(Ha, Xa, staging, 512)
    torch.cuda.synchronize()
    B.gptq_hessian_accumulate_host(Hc, Xc, staging, 512)
    torch.cuda.synchronize()
    Ha_ref, Hc_ref = Ha.cpu().numpy(), Hc.cpu().numpy()
    assert P.rel_fro(Ha_ref, _gpu_hessian(xa)) <= 1e-6 and P.rel_fro(Hc_ref, _gpu_hessian(xc)) <= 1e-6
    for _ in range(2):
        Ha.zero_()
        Hc.zero_()
        B.gptq_hessian_accumulate_host(Ha, Xa, staging, 512)
        torch.cuda._sleep(1000000)            # ~1 ms of other work on the stream
        B.gptq_hessian_accumulate_host(Hc, Xc, staging, 512)
        torch.cuda.synchronize()
        assert np.array_equal(Ha.cpu().numpy(), Ha_ref)
        assert np.array_equal(Hc.cpu().numpy(), Hc_ref)


def test_hessian_zero_tokens_is_noop():
    H = torch.ones(64, 64, dtype=torch.float32, device=DEV)
    X = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    B.gptq_hessian_accumulate(H, X)
    torch.cuda.synchronize()
    assert torch.all(H == 1)


# ---------------------------------------------------------------- factorisation

@pytest.mark.parametrize("d", [8, 64, 200, 256, 392, 1000, 1024])
@pytest.mark.parametrize("act_order", [False, True])
def test_prepare_matches_checker(d, act_order):
    xb = _rand_x(d + 3, max(4 * d, 512), d, outliers=max(1, d // 64))
    Hg = _gpu_hessian(xb)
    perm_g, Ug = _gpu_prepare(Hg, act_order)
    H64 = Hg.astype(np.float64)
    perm_r, Ur, Hp, _ = oracle.prepare(H64, 0.01, act_order)
    np.testing.assert_array_equal(perm_g, perm_r)
    assert np.all(np.tril(Ug, -1) == 0)
    assert P.rel_fro(Ug, Ur) <= P.U_RTOL
    # U^T U H_d = I (property at any size)
    I = Ug.astype(np.float64).T @ Ug.astype(np.float64) @ Hp
    assert np.abs(I - np.eye(d)).max() < 1e-3


@pytest.mark.parametrize("act_order", [False, True])
def test_prepare_batched_trailing_updates_match_checker(act_order):
    """From d_in = 7168 on, the factorisation applies most trailing
    corrections in batches of 512 columns (band and far products on streams
    of their own).  d = 7232: 113 panels of 64, a ragged last batch; against
    the float64 checker, and bitwise equal on a second run."""
    d = 7232
    xb = _rand_x(d + 5, 2 * d, d, outliers=d // 64)
    Hg = _gpu_hessian(xb)
    perm_g, Ug = _gpu_prepare(Hg, act_order)
    perm_r, Ur, Hp, _ = oracle.prepare(Hg.astype(np.float64), 0.01, act_order)
    np.testing.assert_array_equal(perm_g, perm_r)
    assert np.all(np.tril(Ug, -1) == 0)
    assert P.rel_fro(Ug, Ur) <= P.U_RTOL, P.rel_fro(Ug, Ur)
    perm_2, U2 = _gpu_prepare(Hg, act_order)
    assert np.array_equal(perm_2, perm_g) and np.array_equal(U2, Ug)


def test_prepare_rejects_singular_and_nonfinite():
    d = 64
    with pytest.raises(B.GptqError) as e:
        _gpu_prepare(np.zeros((d, d), np.float32), False)
    assert e.value.status == 2
    H = np.eye(d, dtype=np.float32)
    H[3, 3] = np.nan
    with pytest.raises(B.GptqError) as e:
        _gpu_prepare(H, False)
    assert e.value.status == 3
    # indefinite even after damping
    H = np.eye(d, dtype=np.float32)
    H[0, 1] = H[1, 0] = 5.0
    with pytest.raises(B.GptqError) as e:
        _gpu_prepare(H, False, damp=0.0)
    assert e.value.status == 2


def test_prepare_async_matches_prepare_and_reports_status():
    """gptq_prepare_async: the same U and perm bits as gptq_prepare, the
    status in a device word or a pinned host word once the stream passes the
    call, and LayerQuantizer.run raising on a failed factorisation."""
    d = 392
    xb = _rand_x(17, 4 * d, d, outliers=3)
    Hg = _gpu_hessian(xb)
    perm_s, U_s = _gpu_prepare(Hg, True)
    H = torch.from_numpy(Hg).to(DEV)
    U = torch.empty(d, d, device=DEV)
    perm = torch.empty(d, dtype=torch.int32, device=DEV)
    ws = B.workspace(1, d, 128)
    st = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    B.gptq_prepare_async(H, 0.01, True, perm, U, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(U.cpu().numpy(), U_s) and np.array_equal(perm.cpu().numpy(), perm_s)
    sp = torch.full((1,), -7, dtype=torch.int32).pin_memory()
    B.gptq_prepare_async(torch.zeros(d, d, device=DEV), 0.01, False, perm, U, ws, sp)
    torch.cuda.synchronize()
    assert int(sp[0]) == 2                      # GPTQ_ERR_NOT_PD
    Hn = torch.eye(d, device=DEV)
    Hn[3, 3] = float("nan")
    B.gptq_prepare_async(Hn, 0.01, False, perm, U, ws, sp)
    torch.cuda.synchronize()
    assert int(sp[0]) == 3                      # GPTQ_ERR_NONFINITE
    q = LayerQuantizer(64, 384, 4, 128, 128, 0.01, False)
    q.reset()                                   # H = 0: not positive definite
    with pytest.raises(B.GptqError) as e:
        q.run(torch.zeros(64, 384, device=DEV))
    assert e.value.status == 2


# ------------------------------------------------------------------ column loop

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("gs", [-1, 32, 64, 128, 256])
@pytest.mark.parametrize("act_order", [False, True])
def test_quantize_matches_checker(bits, gs, act_order):
    d_out, d_in, n = 256, 512, 2048
    W, xb = synth.random_layer(bits * 31 + gs, d_out, d_in, n, correlated=True)
    _staged_check(W, xb, bits, gs, 128, act_order, f"b{bits} g{gs} ao{act_order}")


@pytest.mark.parametrize("d_out,d_in,gs,block", [(33, 200, 8, 64), (1, 392, 56, 8), (130, 264, 24, 24),
                                                 (257, 136, -1, 128), (64, 1000, 40, 40),
                                                 (40, 8, -1, 8)])
def test_quantize_ragged_shapes(d_out, d_in, gs, block):
    W, xb = synth.random_layer(d_out + d_in, d_out, d_in, max(512, 2 * d_in), correlated=True)
    _staged_check(W, xb, 4, gs, block, True, f"{d_out}x{d_in} g{gs} B{block}")


def test_tiny_workload_end_to_end_from_scratch():
    """S4: the checker computes its own H, U and order."""
    spec = synth.WORKLOADS["tiny"]
    xb = synth.x_bf16(spec)
    W = synth.weight_f32(spec)
    q = LayerQuantizer(spec.d_out, spec.d_in, spec.bits, spec.group_size, spec.block_size,
                       spec.damp, spec.act_order, keep_err=True)
    q.reset()
    q.add_batch(_x_dev(xb))
    res = q.run(torch.from_numpy(W).to(DEV))
    torch.cuda.synchronize()
    ref = oracle.layer(W.astype(np.float64), xb, spec.bits, spec.group_size)
    mse_g = oracle.output_mse(W, res.W_hat.cpu().numpy(), ref["H"], spec.n_tokens)
    P.check_mse(mse_g, ref["mse"], "tiny")
    codes = res.codes.cpu().numpy()
    rate = 1.0 - np.mean(codes != ref["codes"])
    assert rate >= P.CODE_MATCH
    rtn = oracle.rtn(W.astype(np.float64), spec.bits, spec.group_size)
    assert mse_g < oracle.output_mse(W, rtn["W_hat"], ref["H"], spec.n_tokens)


def test_quantize_is_deterministic():
    W, xb = synth.random_layer(77, 64, 256, 1024)
    Hg = _gpu_hessian(xb)
    perm, Ug = _gpu_prepare(Hg, True)
    a = _gpu_quantize(W, Ug, perm, 4, 64, 64)
    b = _gpu_quantize(W, Ug, perm, 4, 64, 64)
    for k in ("codes", "scales", "zeros", "W_hat", "packed"):
        np.testing.assert_array_equal(a[k], b[k])


def test_diagonal_hessian_gives_rtn_on_gpu():
    """With a diagonal H no error is carried: codes equal round-to-nearest."""
    d_out, d_in = 64, 256
    g = np.random.default_rng(3)
    W = (g.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    H = np.diag(g.uniform(0.5, 5.0, d_in)).astype(np.float32)
    perm, Ug = _gpu_prepare(H, False)
    gq = _gpu_quantize(W, Ug, None, 4, 64, 128)
    rt = oracle.rtn(W.astype(np.float64), 4, 64)
    np.testing.assert_array_equal(gq["codes"], rt["codes"])
    np.testing.assert_array_equal(gq["scales"], rt["scales"])
    np.testing.assert_array_equal(gq["zeros"], rt["zeros"])


def test_launch_count_increases():
    before = B.gptq_launch_count()
    _gpu_hessian(_rand_x(1, 128, 64))
    assert B.gptq_launch_count() >= before + 2
    assert B.gptq_device_status() == 0


def test_bounded_wait_times_out_and_device_stays_usable():
    """A wait nothing satisfies gives up after its limit (~1 ms here), records
    GPTQ_ERR_TIMEOUT, and later work on the device still runs correctly."""
    assert B.gptq_selftest_bounded_wait(2_000_000) == 5
    assert B.gptq_device_status() == 0          # the word was read and cleared
    xb = _rand_x(9, 256, 64)
    np.testing.assert_allclose(_gpu_hessian(xb), oracle.hessian(xb), rtol=1e-5, atol=1e-3)


def test_division_free_quotient_matches_ieee_division():
    """The column loop decides each code from w / s rounded without a
    division instruction; on the device it must agree with IEEE division on
    random, all-ones-significand and near-tie operands."""
    assert B.gptq_selftest_quotient(3 << 26, seed=7) == 0


def test_minimum_workspace_gives_the_same_results():
    """gptq_quantize with the smallest accepted workspace forms the tf32 low
    parts inside the lazy-batch products instead of keeping them in the
    workspace; the per-element accumulation order is the same, so the results
    match the full-workspace call."""
    d_out, d_in, bits, gs = 256, 1024, 4, 128
    W, xb = synth.random_layer(21, d_out, d_in, 2 * d_in, correlated=True)
    H = torch.zeros(d_in, d_in, dtype=torch.float32, device=DEV)
    B.gptq_hessian_accumulate(H, torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16))
    U = torch.empty(d_in, d_in, dtype=torch.float32, device=DEV)
    perm = torch.empty(d_in, dtype=torch.int32, device=DEV)
    B.gptq_prepare(H, 0.01, 1, perm, U, B.workspace(d_out, d_in, 128))
    outs = []
    for n in (B.gptq_workspace_bytes(d_out, d_in, 128), B.gptq_workspace_min_bytes(d_out, d_in, 128)):
        ws = torch.empty(n, dtype=torch.uint8, device=DEV)
        Wt = torch.from_numpy(W.astype(np.float32)).to(DEV)
        ng = d_in // gs
        sc = torch.empty(d_out, ng, device=DEV)
        zr = torch.empty(d_out, ng, device=DEV)
        codes = torch.empty(d_out, d_in, dtype=torch.uint8, device=DEV)
        B.gptq_quantize(Wt, U, perm, bits, gs, 128, sc, zr, ws, codes=codes)
        torch.cuda.synchronize()
        outs.append((Wt.cpu().numpy(), sc.cpu().numpy(), codes.cpu().numpy()))
    assert B.gptq_device_status() == 0
    np.testing.assert_array_equal(outs[0][2], outs[1][2])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    np.testing.assert_allclose(outs[0][0], outs[1][0], rtol=1e-6, atol=1e-8)


def test_timed_quantize_matches_and_reports_times():
    """The timing diagnostic runs the same launches as gptq_quantize (direct
    enqueue instead of a graph replay): identical codes, and positive times
    for the column loop and the lazy-batch products."""
    d_out, d_in, bits, gs = 256, 1024, 4, 128
    W, xb = synth.random_layer(22, d_out, d_in, 2 * d_in, correlated=True)
    H = torch.zeros(d_in, d_in, dtype=torch.float32, device=DEV)
    B.gptq_hessian_accumulate(H, torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16))
    U = torch.empty(d_in, d_in, dtype=torch.float32, device=DEV)
    perm = torch.empty(d_in, dtype=torch.int32, device=DEV)
    ws = B.workspace(d_out, d_in, 128)
    B.gptq_prepare(H, 0.01, 0, perm, U, ws)
    res = []
    for timed in (False, True):
        Wt = torch.from_numpy(W.astype(np.float32)).to(DEV)
        sc = torch.empty(d_out, d_in // gs, device=DEV)
        zr = torch.empty(d_out, d_in // gs, device=DEV)
        codes = torch.empty(d_out, d_in, dtype=torch.uint8, device=DEV)
        if timed:
            loop_ms, upd_ms, other_ms = B.gptq_quantize_timed(Wt, U, None, bits, gs, 128, sc, zr, ws, codes=codes)
            assert loop_ms > 0 and upd_ms > 0 and other_ms >= 0
        else:
            B.gptq_quantize(Wt, U, None, bits, gs, 128, sc, zr, ws, codes=codes)
        torch.cuda.synchronize()
        res.append(codes.cpu().numpy())
    np.testing.assert_array_equal(res[0], res[1])
