"""One layer over several GPUs of a node: tokens sharded for the Hessian, the
factorisation replicated, the rows of W sharded for the column loop.

GPTQ overview page, "Równoległość": inside a layer the columns are sequential,
but the Hessian is a sum over calibration tokens and the rows of W are
independent given the factor.  So:
  1. each rank accumulates H over its own contiguous slice of the tokens;
  2. one all-reduce (sum) of the d x d fp32 H, the only exchange;
  3. every rank runs the damping, ordering and factorisation on the same H
     (the all-reduce hands every rank the same bits), and the factorisation
     has no unordered reduction, so all ranks hold the same perm and the same
     U bit for bit, without a broadcast;
  4. each rank quantizes its own contiguous block of rows of W;
  5. optionally one all-gather of the per-row outputs.

The steps take the compute functions as arguments: `ShardedLayer` wires in
libgptq.so through `LayerQuantizer`; the CPU tests wire in the float64 checker
and run the same host logic on gloo ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .layer import LayerQuantizer, QuantizedLayer


def _world(group=None) -> tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


def token_range(n_tokens: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous slice [t0, t1) of the calibration tokens for `rank`; the
    slices cover every token once and differ in size by at most one."""
    return n_tokens * rank // world, n_tokens * (rank + 1) // world


def row_range(d_out: int, rank: int, world: int, align: int = 32) -> tuple[int, int]:
    """Contiguous rows [r0, r1) of W for `rank`, in whole multiples of `align`
    (the column loop's row tile) except for the last rank."""
    units = (d_out + align - 1) // align
    u0, u1 = units * rank // world, units * (rank + 1) // world
    return min(d_out, u0 * align), min(d_out, u1 * align)


def all_reduce_hessian(H: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of the ranks' partial Hessians, in place (identity on one rank)."""
    _, world = _world(group)
    if world > 1:
        dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    return H


def gather_rows(local: torch.Tensor, d_out: int, group=None, align: int = 32) -> torch.Tensor:
    """The full [d_out, ...] tensor from each rank's row block (all-gather of
    equal-sized padded blocks, then the padding dropped)."""
    rank, world = _world(group)
    if world == 1:
        return local
    sizes = [row_range(d_out, r, world, align) for r in range(world)]
    cap = max(r1 - r0 for r0, r1 in sizes)
    pad = torch.zeros((cap,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[: r1 - r0] for p, (r0, r1) in zip(parts, sizes)], dim=0)


def run_sharded(X_local, W_rows, hessian_fn, prepare_fn, quantize_fn, group=None):
    """Steps 1-4 with caller-supplied compute: hessian_fn(X_local) -> partial
    H (a tensor, summed in place across ranks); prepare_fn(H) -> state shared
    by all rows; quantize_fn(W_rows, state) -> this rank's rows' result."""
    H = hessian_fn(X_local)
    all_reduce_hessian(H, group)
    state = prepare_fn(H)
    return H, state, quantize_fn(W_rows, state)


class ShardedLayer:
    """One linear layer quantized by all ranks of the default group, each on
    its own GPU: `add_batch` takes this rank's tokens, `prepare` all-reduces H
    and factorises it, `quantize` takes the full W (every rank holds it) and
    quantizes this rank's rows."""

    def __init__(self, d_out: int, d_in: int, bits: int = 4, group_size: int = 128,
                 block_size: int = 128, damp: float = 0.01, act_order: bool = False,
                 device="cuda", group=None):
        self.rank, self.world = _world(group)
        self.group = group
        self.d_out = d_out
        self.r0, self.r1 = row_range(d_out, self.rank, self.world)
        self.q = LayerQuantizer(max(1, self.r1 - self.r0), d_in, bits, group_size, block_size,
                                damp, act_order, device=device)

    def reset(self):
        self.q.reset()

    def add_batch(self, X_local: torch.Tensor):
        self.q.add_batch(X_local)

    def prepare(self):
        all_reduce_hessian(self.q.H, self.group)
        self.q.prepare()

    def quantize(self, W: torch.Tensor) -> QuantizedLayer | None:
        """W [d_out, d_in] (all rows); returns this rank's rows [r0, r1), or
        None when the rank has no rows (more ranks than 32-row tiles)."""
        if self.r1 <= self.r0:
            return None
        return self.q.quantize(W[self.r0:self.r1].contiguous())
