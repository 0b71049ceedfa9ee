"""The multi-GPU host logic on CPU: two gloo ranks on 127.0.0.1."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

from post_weight_quantization_accumulate_b200 import ranks, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        base = synth.WORKLOADS["tiny"]
        spec = ranks.rank_workload(base, rank)
        x = synth.x_bf16(spec, tokens=slice(0, 64))
        times = [1.0 + rank, 5.0 - rank]          # rank-dependent "measurements"
        mx = ranks.max_over_ranks(times)
        out[rank] = (spec.tensor_id, int(x.astype(np.int64).sum()), mx)
    finally:
        dist.destroy_process_group()


def test_two_ranks_get_independent_layers_and_max_timing():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (t0, s0, m0), (t1, s1, m1) = out[0], out[1]
    assert t0 != t1                      # distinct layers
    assert s0 != s1                      # distinct activation draws
    assert m0 == m1 == [2.0, 5.0]        # max over ranks, same on every rank


def test_job_rate_and_single_process_identity():
    assert ranks.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert ranks.job_rate(4, 4096, 4096, 10.0) == 4 * 4096 * 4096 / 0.01
