"""gptq_quantize_static_scratch: the workspace-free variant of gptq_quantize
for callers that cannot allocate device memory (an engine plugin that gets
only input/output pointers, a loop that must avoid cudaMalloc's device-wide
synchronisation, a process whose memory is all reserved up front).

Two calls in a row through the C ABI are compared with gptq_quantize (caller
workspace) on the same inputs, within the parity tolerances of the other
tests.  The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import build as build_mod
from post_weight_quantization_accumulate_b200 import synth

import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_mod.build()
    B.lib()


def _factor(seed, d_out, d_in, act_order):
    W, xb = synth.random_layer(seed, d_out, d_in, 2 * d_in, correlated=True)
    H = torch.zeros(d_in, d_in, dtype=torch.float32, device=DEV)
    B.gptq_hessian_accumulate(H, torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16))
    U = torch.empty(d_in, d_in, dtype=torch.float32, device=DEV)
    perm = torch.empty(d_in, dtype=torch.int32, device=DEV)
    B.gptq_prepare(H, 0.01, act_order, perm, U, B.workspace(d_out, d_in, 128))
    return torch.from_numpy(W.astype(np.float32)).to(DEV), U, perm if act_order else None


def _outputs(d_out, d_in, bits, gs):
    ng = d_in // gs if gs > 0 else 1
    return dict(scales=torch.empty(d_out, ng, device=DEV), zeros=torch.empty(d_out, ng, device=DEV),
                codes=torch.empty(d_out, d_in, dtype=torch.uint8, device=DEV),
                packed_int4=torch.empty(d_out, d_in // 2, dtype=torch.uint8, device=DEV),
                g_idx=torch.empty(d_in, dtype=torch.int32, device=DEV),
                err_sq=torch.empty(d_out, device=DEV))


def _compare(ref_W, ref, W, out, bits, gs, perm, where):
    torch.cuda.synchronize()
    # the same kernels run behind both entry points: results agree exactly,
    # which is inside every tolerance of the parity tests
    np.testing.assert_array_equal(out["codes"].cpu().numpy(), ref["codes"].cpu().numpy())
    np.testing.assert_allclose(out["scales"].cpu().numpy(), ref["scales"].cpu().numpy(), rtol=P.SZ_RTOL)
    np.testing.assert_array_equal(out["zeros"].cpu().numpy(), ref["zeros"].cpu().numpy())
    np.testing.assert_allclose(W.cpu().numpy(), ref_W.cpu().numpy(), rtol=1e-5, atol=1e-7)
    np.testing.assert_array_equal(out["packed_int4"].cpu().numpy(), ref["packed_int4"].cpu().numpy())
    np.testing.assert_array_equal(out["g_idx"].cpu().numpy(), ref["g_idx"].cpu().numpy())
    np.testing.assert_allclose(out["err_sq"].cpu().numpy(), ref["err_sq"].cpu().numpy(), rtol=1e-5)


def test_static_scratch_matches_workspace_entry_point_twice_in_a_row():
    cases = [(11, 256, 1024, 4, 128, True), (12, 300, 512, 3, 64, False)]
    for seed, d_out, d_in, bits, gs, act in cases:
        W0, U, perm = _factor(seed, d_out, d_in, act)
        # existing entry point with a caller workspace
        W_ref = W0.clone()
        ref = _outputs(d_out, d_in, bits, gs)
        B.gptq_quantize(W_ref, U, perm, bits, gs, 128, ref["scales"], ref["zeros"],
                        B.workspace(d_out, d_in, 128), codes=ref["codes"],
                        packed_int4=ref["packed_int4"], g_idx=ref["g_idx"], err_sq=ref["err_sq"])
        # the workspace-free entry point, called twice in a row on the same layer
        for call in range(2):
            W = W0.clone()
            out = _outputs(d_out, d_in, bits, gs)
            torch.cuda.synchronize()
            free0, torch0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
            B.gptq_quantize_static_scratch(W, U, perm, bits, gs, 128, out["scales"], out["zeros"],
                                           codes=out["codes"], packed_int4=out["packed_int4"],
                                           g_idx=out["g_idx"], err_sq=out["err_sq"])
            torch.cuda.synchronize()
            if call == 1:
                # once the first call has created the array, a call takes no
                # device memory: neither from the device nor from torch's pool
                assert torch.cuda.mem_get_info()[0] == free0
                assert torch.cuda.memory_allocated() == torch0
            _compare(W_ref, ref, W, out, bits, gs, perm, f"static scratch {d_out}x{d_in} call {call}")


def test_static_scratch_refuses_layers_larger_than_the_array():
    """A layer whose working set exceeds the fixed array (4096 x 11008) is
    refused with GPTQ_ERR_WORKSPACE.  The buffers handed over are real device
    tensors of the declared shapes, so even a refusal that came too late
    could not touch memory outside them."""
    d_out, d_in = 4096, 11008
    W = torch.zeros(d_out, d_in, device=DEV)
    U = torch.zeros(d_in, d_in, device=DEV)
    out = _outputs(d_out, d_in, 4, 128)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = B.lib().gptq_quantize_static_scratch(ptr(W), ptr(U), None, d_out, d_in, 4, 128, 128,
                                               ptr(out["codes"]), ptr(out["scales"]),
                                               ptr(out["zeros"]), None, None, None, None)
    assert st == 6  # GPTQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert B.gptq_device_status() == 0
