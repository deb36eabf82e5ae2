"""Sequences cut along T across ranks: one process per GPU, each holding a
contiguous stretch of tokens of every (b, h) sequence.

The recurrence over a stretch is affine in the state entering it (xLSTM page,
"mLSTM (matrix LSTM)" eq. 1-2 with the "sLSTM" stabilizer), so the forward pass
needs exactly one exchange:
  1. each rank summarises its stretch (F, m_seg, C_seg, n_seg from a zero state
     with the stabilizer at -inf: xlstm_mlstm_segment_summary);
  2. one all-gather of the summaries over the process group (NCCL over NVLink on
     GPUs; d_v*d_qk + d_qk floats and two doubles per head and rank);
  3. rank r chains the summaries of ranks 0..r-1 onto the sequence's initial
     state (xlstm_mlstm_combine_states): its entry state, with the canonical m;
  4. rank r runs the chunkwise forward over its stretch from that entry state.
The final state of the whole sequence is the chain of all R summaries; every
rank forms it, so no second exchange is needed.

The arithmetic runs in the CUDA library (``ops=CudaOps()``); this module only
orders the calls and the collective.  ``ops`` is a parameter so that the host
plumbing can be exercised on CPU ranks (gloo) with another implementation of
the three operations.
"""
from __future__ import annotations


class CudaOps:
    """The three per-rank operations through the C ABI (torch CUDA tensors)."""

    def summary(self, k, v, i_pre, f_pre):
        from . import capi
        return capi.summary(k, v, i_pre, f_pre)

    def combine(self, C_seg, n_seg, F_m, state):
        from . import capi
        return capi.combine(C_seg, n_seg, F_m, state)

    def forward(self, q, k, v, i_pre, f_pre, state, qk_scale):
        from . import capi
        return capi.fwd(q, k, v, i_pre, f_pre, state=state, qk_scale=qk_scale)


def dist_gather(group=None):
    """The exchange step over a torch.distributed process group: all_gather of
    one tensor, returning (every rank's tensor in rank order, this rank)."""
    def gather(x):
        import torch
        import torch.distributed as dist
        parts = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, x.contiguous(), group=group)
        return parts, dist.get_rank(group)
    return gather


def fwd_tsharded(q, k, v, i_pre, f_pre, state=None, qk_scale=None, group=None, ops=None, gather=None):
    """Forward of this rank's stretch of tokens.

    q, k [B,H,T_r,d_qk], v [B,H,T_r,d_v], i_pre, f_pre [B,H,T_r]: tokens
    [t_r, t_r + T_r) of every sequence, rank r of the group holding the r-th
    stretch in order.  state: the sequence's initial (C, n, m), the same on
    every rank, or None (zero state).  Returns (h of the stretch, final state of
    the whole sequence); every rank returns the same final state.
    gather: the exchange step (default: all_gather over ``group``).
    """
    import torch

    ops = ops or CudaOps()
    gather = gather or dist_gather(group)
    summaries = ops.summary(k, v, i_pre, f_pre)
    stacked = []
    rank = 0
    for x in summaries:
        parts, rank = gather(x)
        stacked.append(torch.stack(parts))
    Cs, ns, Fs = stacked
    entry = state if rank == 0 else ops.combine(Cs[:rank], ns[:rank], Fs[:rank], state)
    h, _ = ops.forward(q, k, v, i_pre, f_pre, entry, qk_scale)
    final = ops.combine(Cs, ns, Fs, state)
    return h, final
