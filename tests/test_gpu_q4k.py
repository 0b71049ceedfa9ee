"""GPTQ onto the two-level Q4_K grid on the device against the float64
checker, given the device's own factor and order (the staged parity of the
one-level grid, with the same bar): walking each row in processing order,
its first divergence is a code or a 6-bit level one step off at a rounding
tie; the 4-bit codes agree on >= 99.9% of entries and every code mismatch is
one level; at most 3% of the rows diverge (the 6-bit levels carry a tie
through the rest of a row); super-block scales agree to 1e-5 before a row's
first divergence; and the layer-output MSE agrees to 0.5%.  The device's outputs obey
w^ = d sc q - dmin m.  A full-size 4096 x 4096 layer is checked on sampled
rows."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import synth

import parity as P

pytestmark = pytest.mark.gpu


def _run(d_out, d_in, n, act_order, seed):
    W, xb = synth.random_layer(seed, d_out, d_in, n, correlated=True)
    dev = torch.device("cuda")
    X = torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
    H = torch.zeros(d_in, d_in, dtype=torch.float32, device=dev)
    B.gptq_hessian_accumulate(H, X)
    perm = torch.empty(d_in, dtype=torch.int32, device=dev)
    U = torch.empty(d_in, d_in, dtype=torch.float32, device=dev)
    ws = B.workspace(d_out, d_in, 128, device=dev)
    B.gptq_prepare(H, 0.01, act_order, perm, U, ws)
    Wt = torch.from_numpy(W.astype(np.float32)).to(dev)
    nb, ns = d_in // 32, d_in // 256
    out = {"sc6": torch.empty(d_out, nb, dtype=torch.uint8, device=dev),
           "m6": torch.empty(d_out, nb, dtype=torch.uint8, device=dev),
           "dsup": torch.empty(d_out, ns, dtype=torch.float32, device=dev),
           "dmin": torch.empty(d_out, ns, dtype=torch.float32, device=dev),
           "scales": torch.empty(d_out, nb, dtype=torch.float32, device=dev),
           "offsets": torch.empty(d_out, nb, dtype=torch.float32, device=dev)}
    codes = torch.empty(d_out, d_in, dtype=torch.uint8, device=dev)
    packed = torch.empty(d_out, d_in // 2, dtype=torch.uint8, device=dev)
    g_idx = torch.empty(d_in, dtype=torch.int32, device=dev)
    B.gptq_quantize_q4k(Wt, U, perm if act_order else None, out, ws, codes=codes,
                        packed_int4=packed, g_idx=g_idx)
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
    g = {k: v.cpu().numpy() for k, v in out.items()}
    g.update(codes=codes.cpu().numpy(), packed=packed.cpu().numpy(), g_idx=g_idx.cpu().numpy(),
             W_hat=Wt.cpu().numpy(), H=H.cpu().numpy().astype(np.float64),
             U=U.cpu().numpy().astype(np.float64), perm=perm.cpu().numpy())
    return W, g


@pytest.mark.parametrize("d_out,d_in,act_order", [(256, 1024, False), (200, 2048, True), (64, 256, False)])
def test_q4k_matches_checker(d_out, d_in, act_order):
    W, g = _run(d_out, d_in, 4096, act_order, d_in + d_out)
    perm = g["perm"] if act_order else None
    ref = oracle.quantize_q4k(W, g["U"], perm)
    P.check_q4k(g, ref, g["perm"] if act_order else np.arange(d_in), f"q4k {d_out}x{d_in} ao{act_order}")
    n = 4096
    mse_g = oracle.output_mse(W, g["W_hat"].astype(np.float64), g["H"], n)
    mse_r = oracle.output_mse(W, ref["W_hat"], g["H"], n)
    P.check_mse(mse_g, mse_r, f"q4k {d_out}x{d_in}")
    # the device's own outputs: levels in range and w^ = scales q - offsets
    assert g["codes"].max() <= 15 and g["sc6"].min() >= 1 and g["sc6"].max() <= 63 and g["m6"].max() <= 63
    blk = np.arange(d_in) // 32
    sup = np.arange(d_in) // 256
    np.testing.assert_array_equal(g["scales"], (g["dsup"][:, sup[::32]] * g["sc6"].astype(np.float32)))
    np.testing.assert_array_equal(g["offsets"], (g["dmin"][:, sup[::32]] * g["m6"].astype(np.float32)))
    pk = perm if perm is not None else np.arange(d_in)
    codes_p = g["codes"][:, pk]
    what_p = (g["scales"][:, blk].astype(np.float64) * codes_p - g["offsets"][:, blk]).astype(np.float32)
    # one rounding of s q - o (fused on the device): within one ulp of the float64 form
    assert (np.abs(g["W_hat"][:, pk] - what_p) <= np.spacing(np.abs(what_p))).all()
    np.testing.assert_array_equal(oracle.unpack_int4(g["packed"]), g["codes"])
    np.testing.assert_array_equal(g["g_idx"], oracle.g_idx(pk, 32))


def test_q4k_through_the_layer_wrapper():
    """LayerQuantizer.quantize_q4k (act_order) against the checker with the
    wrapper's own factor and order."""
    from post_weight_quantization_accumulate_b200.layer import LayerQuantizer
    d_out, d_in = 96, 512
    W, xb = synth.random_layer(77, d_out, d_in, 2048, correlated=True)
    q = LayerQuantizer(d_out, d_in, act_order=True)
    q.add_batch(torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16))
    q.prepare()
    r = q.quantize_q4k(torch.from_numpy(W.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
    perm = q.perm.cpu().numpy()
    ref = oracle.quantize_q4k(W, q.U.cpu().numpy().astype(np.float64), perm)
    g = {k: r[k].cpu().numpy() for k in ("codes", "sc6", "m6", "dsup", "dmin")}
    P.check_q4k(g, ref, perm, "q4k layer wrapper")
    np.testing.assert_array_equal(oracle.unpack_int4(r["packed"].cpu().numpy()), r["codes"].cpu().numpy())


@pytest.mark.slow
def test_q4k_full_size_q_proj_sampled_rows():
    """The q_proj workload (4096 x 4096, 262144 tokens) onto the Q4_K grid in
    the launch configuration of the benchmark's layer: sampled rows rerun by
    the checker with the device's factor, under the same bar."""
    from post_weight_quantization_accumulate_b200.layer import LayerQuantizer
    spec = synth.WORKLOADS["q_proj_4096"]
    xb = synth.x_bf16(spec)
    W = synth.weight_f32(spec)
    q = LayerQuantizer(spec.d_out, spec.d_in, 4, 32, 128, spec.damp, spec.act_order)
    q.reset()
    q.add_batch(torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16))
    del xb
    q.prepare()
    r = q.quantize_q4k(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
    rows = np.sort(np.random.default_rng(3).choice(spec.d_out, 24, replace=False))
    perm = q.perm.cpu().numpy()
    U = q.U.cpu().numpy().astype(np.float64)
    ref = oracle.quantize_q4k(W[rows].astype(np.float64), U, perm, block=128)
    g = {k: r[k].cpu().numpy()[rows] for k in ("codes", "sc6", "m6", "dsup", "dmin")}
    P.check_q4k(g, ref, perm, "q4k q_proj_4096")
    H64 = q.H.cpu().numpy().astype(np.float64)
    mse_g = oracle.output_mse(W[rows], r["W_hat"].cpu().numpy()[rows].astype(np.float64), H64, spec.n_tokens)
    mse_r = oracle.output_mse(W[rows], ref["W_hat"], H64, spec.n_tokens)
    P.check_mse(mse_g, mse_r, "q4k q_proj_4096")
