"""Host-side logic of a multi-GPU run: one process per GPU.

Every (batch, head) pair of block-causal linear attention is independent: its
own q, k, v tokens and its own 32x33 state ("Nvidia, MIT ve diğerleri video
yapay zeka devrimini başlattı", section "Sabit Bellekli KV önbelleğe alma
mekanizması": the cached KV is a per-head sum).  A multi-GPU job therefore
needs no data-path collective: either every rank runs an independent problem
of the same shape (weak scaling: ``rank_workload``), or the heads of one
problem are split across ranks (strong scaling: ``head_slice``), each rank
owning its heads' tensors and state.  The only collectives are the host's:
agreeing on a step count and taking the slowest rank's time.

A block with too few (batch, head) pairs to fill the GPUs can instead be split
by tokens (``token_slice``, ``split_call``): splitting along tokens leaves the
block's KV a sum of the slices' KV (KV_{1-2} = KV_1 + KV_2 in the same
section), so the ranks exchange one [S | Z] partial per (batch, head), an
all-gather of 4,224 bytes each, and every rank commits the same state.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch

from .synth import Workload

RANK_SEED_STRIDE = 1000


def rank_workload(w: Workload, rank: int) -> Workload:
    """The problem rank `rank` runs in a weak-scaling job: the same shape with
    its own seed (rank 0 keeps the workload's seed)."""
    if rank < 0:
        raise ValueError("rank must be >= 0")
    return w.shrink(seed=w.seed + RANK_SEED_STRIDE * rank) if rank else w


def head_slice(H: int, world: int, rank: int, group: int = 4) -> Tuple[int, int]:
    """Heads [h0, h1) of rank `rank` when the H heads of one problem are split
    over `world` ranks: contiguous, as even as possible, and in whole groups of
    `group` heads when H allows it (the tensor-core kernels take 4-head
    groups).  Ranks beyond the available groups get an empty range."""
    if world < 1 or not 0 <= rank < world or H < 1:
        raise ValueError("need H >= 1 and 0 <= rank < world")
    unit = group if H % group == 0 else 1
    units = H // unit
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return u0 * unit, u1 * unit


def _reduce(values: Sequence[float], dist, device, op) -> List[float]:
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=op)
    return [float(x) for x in t.tolist()]


def max_over_ranks(values: Sequence[float], dist=None, device="cpu") -> List[float]:
    """Elementwise MAX over ranks (the slowest rank's times)."""
    op = dist.ReduceOp.MAX if dist is not None else None
    return _reduce(values, dist, device, op)


def agree_steps(steps: int, dist=None, device="cpu") -> int:
    """The smallest step count any rank asked for, so that every rank takes the
    same collective steps in the same order."""
    op = dist.ReduceOp.MIN if dist is not None else None
    return int(_reduce([float(steps)], dist, device, op)[0])


def token_slice(N: int, world: int, rank: int, align: int = 1) -> Tuple[int, int]:
    """Tokens [t0, t1) of rank `rank` when one block of N tokens is split over
    `world` ranks: contiguous, in whole units of `align` tokens (a frame, for
    RoPE), as even as possible."""
    if world < 1 or not 0 <= rank < world or N < 0 or align < 1:
        raise ValueError("need N >= 0, align >= 1 and 0 <= rank < world")
    units = (N + align - 1) // align
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(u0 * align, N), min(u1 * align, N)


def token_split_block(q, k, v, reduce_fn, gather_fn, apply_fn):
    """One block whose tokens are split over the ranks: this rank's q, k, v
    slice -> its partial sums (reduce_fn) -> every rank's partials in rank
    order (gather_fn, the one collective) -> this rank's outputs (apply_fn,
    which adds the partials to the state in rank order and commits).  The
    steps are passed in so that the exchange can run with any backend."""
    partial = reduce_fn(k, v)
    gathered = gather_fn(partial)
    return apply_fn(q, gathered)


def split_call(q_slices, kv_slices, reduce_fn, gather_fn, apply_fn):
    """One call of a block whose tokens are split over the ranks, for the ranks
    this process holds (one, or several emulated ranks on one GPU): their
    partial sums in local rank order (reduce_fn(j, k, v)), one exchange
    (gather_fn: the local partials -> every rank's partials in global rank
    order), then their outputs (apply_fn(j, q, gathered)).  Every rank adds the
    same gathered partials to the same state, so all commit the same state."""
    partials = [reduce_fn(j, k, v) for j, (k, v) in enumerate(kv_slices)]
    gathered = gather_fn(partials)
    return [apply_fn(j, q, gathered) for j, q in enumerate(q_slices)]


def split_frame_offsets(frames_before: int, N: int, world: int, align: int) -> List[Tuple[int, int, int]]:
    """(t0, t1, first frame) of every rank's slice of a block of N tokens that
    follows `frames_before` frames of the stream, split in whole frames of
    `align` tokens (RoPE positions continue across the ranks' slices)."""
    out = []
    for r in range(world):
        t0, t1 = token_slice(N, world, r, align)
        out.append((t0, t1, frames_before + t0 // align))
    return out


def nccl_gather(partial, dist):
    """All-gather of the partial sums, stacked in rank order: [R, *partial.shape]."""
    world = dist.get_world_size()
    out = partial.new_empty((world,) + tuple(partial.shape))
    dist.all_gather_into_tensor(out, partial.contiguous())
    return out


def job_throughput(units_per_rank_step: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's
    time."""
    if total_ms <= 0:
        raise ValueError("total_ms must be > 0")
    return units_per_rank_step * world * steps / (total_ms / 1e3)
