"""Context (sequence) parallel SSD forward over a process group.

The sequence is cut into contiguous segments, one per rank, as in the SSD write-up's
"序列并行": every rank runs the chunked forward on its own segment, then the ranks
pass states. Here the passing is one all-gather of every rank's local end state and
total log-decay (NCCL over NVLink on GPUs), after which each rank forms its incoming
state by an exclusive scan over the ranks before it and adds that state's term to
its outputs (the state-to-output step of the chunked algorithm). All arithmetic runs
in libssd's kernels (ssd_fwd, ssd_cp_decay, ssd_cp_combine, ssd_cp_correct); this
module orders the calls and issues the collective.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding


class CudaSteps:
    """The four per-rank steps, on libssd's CUDA kernels."""

    def fwd(self, x, dt, A, B, C, D, h0, chunk):
        return _binding.ssd_fwd(x, dt, A, B, C, D, h0, chunk=chunk)

    def decay(self, dt, A):
        return _binding.ssd_cp_decay(dt, A)

    def combine(self, states, totals, rank):
        return _binding.ssd_cp_combine(states, totals, rank)

    def correct(self, dt, A, C, block_decay, s_in, y):
        return _binding.ssd_cp_correct(dt, A, C, block_decay, s_in, y)


def segment_bounds(seqlen: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of rank's segment: contiguous, in rank order, lengths differing by at most one."""
    q, r = divmod(seqlen, world)
    start = rank * q + min(rank, r)
    return start, start + q + (1 if rank < r else 0)


def ssd_fwd_context_parallel(x, dt, A, B, C, D=None, h0=None, *, chunk: int, group=None, steps=None):
    """y, h_end = the SSD forward of this rank's segment within the whole sequence.

    x [B,L_r,H,P], dt [B,L_r,H], B/C [B,L_r,G,N] are this rank's segment (rank order =
    sequence order); A, D are per head; h0 [B,H,P,N] is the state before the whole
    sequence and is read on rank 0 only. Returns this segment's outputs and the state at
    its end (on the last rank, the sequence's final state). Every rank of `group` must call
    it with the same batch, head and state sizes. `steps` supplies the per-rank steps
    (default: CudaSteps).
    """
    steps = steps or CudaSteps()
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    y, h_loc = steps.fwd(x, dt, A, B, C, D, h0 if rank == 0 else None, chunk)
    if world == 1:
        return y, h_loc
    block_decay, total = steps.decay(dt, A)
    # gathered along dim 0 in rank order, then viewed as [R, ...]
    states = torch.empty((world * h_loc.shape[0],) + tuple(h_loc.shape[1:]), dtype=h_loc.dtype, device=h_loc.device)
    totals = torch.empty((world * total.shape[0],) + tuple(total.shape[1:]), dtype=total.dtype, device=total.device)
    dist.all_gather_into_tensor(states, h_loc.contiguous(), group=group)
    dist.all_gather_into_tensor(totals, total.contiguous(), group=group)
    s_in, h_end = steps.combine(states.view((world,) + tuple(h_loc.shape)), totals.view((world,) + tuple(total.shape)),
                                rank)
    if rank > 0:
        steps.correct(dt, A, C, block_decay, s_in, y)
    return y, h_end
