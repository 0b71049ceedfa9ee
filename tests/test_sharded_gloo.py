"""The sharded single-layer path (tokens for the Hessian, one all-reduce,
replicated factorisation, rows for the column loop) on two gloo ranks, with
the float64 checker as the compute: the gathered result equals the checker's
single-process layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from post_weight_quantization_accumulate_b200 import sharded, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, act_order, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = synth.WORKLOADS["tiny"]
        xb = synth.x_bf16(spec)
        W = synth.weight_f32(spec).astype(np.float64)
        t0, t1 = sharded.token_range(spec.n_tokens, rank, world)
        r0, r1 = sharded.row_range(spec.d_out, rank, world)
        H, (perm, U, _, _), res = sharded.run_sharded(
            xb[t0:t1], W[r0:r1],
            hessian_fn=lambda X: torch.from_numpy(oracle.hessian(X)),
            prepare_fn=lambda H: oracle.prepare(H.numpy(), 0.01, act_order),
            quantize_fn=lambda Wr, st: oracle.quantize(Wr, st[1], st[0], spec.bits, spec.group_size))
        codes = sharded.gather_rows(torch.from_numpy(res["codes"]), spec.d_out)
        what = sharded.gather_rows(torch.from_numpy(res["W_hat"]), spec.d_out)
        out[rank] = (H.numpy(), perm, codes.numpy(), what.numpy(), (t0, t1), (r0, r1))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("act_order", [False, True])
def test_two_ranks_reproduce_the_single_process_layer(act_order):
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), act_order, out), nprocs=world, join=True)
    spec = synth.WORKLOADS["tiny"]
    xb = synth.x_bf16(spec)
    W = synth.weight_f32(spec).astype(np.float64)
    ref = oracle.layer(W, xb, spec.bits, spec.group_size, 0.01, act_order)
    (H0, p0, c0, w0, tr0, rr0), (H1, p1, c1, w1, tr1, rr1) = out[0], out[1]
    assert tr0 == (0, 1024) and tr1 == (1024, 2048)          # every token once
    assert rr0 == (0, 128) and rr1 == (128, 256)              # every row once
    np.testing.assert_array_equal(H0, H1)                     # the all-reduce agrees
    np.testing.assert_allclose(H0, ref["H"], rtol=1e-12, atol=1e-9)
    np.testing.assert_array_equal(p0, p1)
    np.testing.assert_array_equal(c0, c1)                     # every rank gathers the same
    assert (c0 == ref["codes"]).mean() >= 0.999
    np.testing.assert_allclose(w0, ref["W_hat"], rtol=0, atol=1e-6)


def test_ranges_partition_and_single_process_identity():
    for n, world in [(2048, 2), (1000, 3), (7, 8)]:
        spans = [sharded.token_range(n, r, world) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    for d_out, world in [(4096, 8), (200, 3), (40, 4)]:
        rows = [sharded.row_range(d_out, r, world) for r in range(world)]
        assert rows[0][0] == 0 and rows[-1][1] == d_out
        assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
        assert all(r0 % 32 == 0 for r0, _ in rows)
    H = torch.ones(3, 3)
    assert sharded.all_reduce_hessian(H) is H and float(H.sum()) == 9.0
    t = torch.arange(6).reshape(3, 2)
    assert sharded.gather_rows(t, 3) is t
