"""Host logic for running the per-layer path on several GPUs of one node.

Layers are independent (GPTQ overview page, "Równoległość": columns are
sequential inside a layer, layers can be processed independently), so each
rank quantizes a layer of its own and no data crosses between GPUs.  The only
collectives are the timing barrier and the max-over-ranks reduction of the
measured times.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import synth


def rank_workload(base: synth.LayerSpec, rank: int) -> synth.LayerSpec:
    """The layer rank `rank` quantizes: the base recipe with its own tensor id
    (so its weights and activations are independent draws)."""
    return synth.scaled(base, tensor_id=base.tensor_id + rank)


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise maximum of `values` over all ranks (identity when not
    distributed)."""
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate(world: int, d_out: int, d_in: int, ms_per_step: float) -> float:
    """Quantized weights per second of the whole job: every rank finishes one
    d_out x d_in layer per step; the step time is the slowest rank's."""
    return world * d_out * d_in / (ms_per_step / 1e3)
