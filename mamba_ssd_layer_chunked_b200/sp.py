"""Sequence-parallel SSD forward over the ranks of a process group.

Rank r holds tokens [t_r, t_{r+1}) of every batch row (X, log_a, B, C and
seq_idx of that segment; segments may differ in length). The state after a
segment is affine in the state before it, E = dec * H_start + loc, so one
exchange of the per-segment (loc, dec, ids) suffices ("Mamba-2: writing the
recurrent state as a structured matrix", wq-win section 3, a block's local end
state and block decay, for a block that is a whole segment):

  1. ``sp_summary``   this rank's (loc, dec, ids)              (kernel)
  2. all-gather of the three over the group, in rank order     (NCCL)
  3. ``sp_combine``   the initial states of this rank's segment (kernel)
  4. ``ssd_fwd``      the ordinary forward pass with them      (kernels)
  5. final states: ``sp_own_finals`` keeps the sequences whose last token
     this rank holds, and a sum over the ranks assembles them  (kernel, NCCL)

The collectives are arguments, so that the same driver runs over
torch.distributed (``torch_collectives``) or over ranks emulated in one
process. Every step of the computation runs in the library's kernels.
"""
from typing import Callable, Optional, Tuple

import torch

from . import ssd


class GpuOps:
    """The library's entry points for the steps above."""

    @staticmethod
    def summary(X, log_a, B, seq_idx, nseq, chunk):
        return ssd.sp_summary(X, log_a, B, seq_idx=seq_idx, nseq=nseq, chunk=chunk)

    @staticmethod
    def combine(X, B, g_loc, g_dec, g_ids, rank, init_states, nseq, chunk):
        return ssd.sp_combine(X, B, g_loc, g_dec, g_ids, rank, init_states=init_states, nseq=nseq, chunk=chunk)

    @staticmethod
    def forward(X, log_a, B, C, chunk, D, init_local, seq_idx, nseq, return_final_states):
        return ssd.ssd_fwd(X, log_a, B, C, chunk, D=D, init_states=init_local, seq_idx=seq_idx, nseq=nseq,
                           return_final_states=return_final_states)

    @staticmethod
    def own_finals(X, B, final, g_ids, rank, nseq, chunk):
        return ssd.sp_own_finals(X, B, final, g_ids, rank, nseq=nseq, chunk=chunk)


def ssd_fwd_sp(X: torch.Tensor, log_a: torch.Tensor, B: torch.Tensor, C: torch.Tensor, chunk: int, *,
               rank: int, all_gather: Callable[[torch.Tensor], torch.Tensor],
               all_reduce_sum: Optional[Callable[[torch.Tensor], torch.Tensor]] = None,
               D: Optional[torch.Tensor] = None, init_states: Optional[torch.Tensor] = None,
               seq_idx: Optional[torch.Tensor] = None, nseq: Optional[int] = None,
               return_final_states: bool = True, ops=GpuOps) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """This rank's Y [b, T_r, H, P] and, when return_final_states, the final
    states [b, nseq, H, N, P] of the whole sequence (identical on every rank).

    ``all_gather(t)`` returns the ranks' t stacked in rank order ([R, *t.shape]);
    ``all_reduce_sum(t)`` the element-wise sum over the ranks. init_states are
    the per-sequence initial states of the whole sequence (the same tensor on
    every rank). nseq is required with seq_idx, as in ssd_fwd."""
    if nseq is None:
        if seq_idx is not None:
            raise ValueError("nseq is required with seq_idx")
        nseq = 1
    loc, dec, ids = ops.summary(X, log_a, B, seq_idx, nseq, chunk)
    g_loc, g_dec, g_ids = all_gather(loc), all_gather(dec), all_gather(ids)
    init_local = ops.combine(X, B, g_loc, g_dec, g_ids, rank, init_states, nseq, chunk)
    Y, final = ops.forward(X, log_a, B, C, chunk, D, init_local, seq_idx, nseq, return_final_states)
    if not return_final_states:
        return Y, None
    if all_reduce_sum is None:
        raise ValueError("all_reduce_sum is required for the final states")
    ops.own_finals(X, B, final, g_ids, rank, nseq, chunk)
    return Y, all_reduce_sum(final)


def torch_collectives(group=None):
    """(all_gather, all_reduce_sum) over a torch.distributed process group
    (NCCL for CUDA tensors, gloo for CPU tensors)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)

    def all_gather(t):
        t = t.contiguous()
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t, group=group)
        return torch.stack(parts)

    def all_reduce_sum(t):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        return t

    return all_gather, all_reduce_sum
