"""Context-parallel prefill: one batch of long sequences split along time
across the ranks of a process group, one segment per rank.

The KDA recurrence (Kimi Linear paper notes, section 2) is affine in the
state, so a segment of tokens maps any start state S to M S + B, where B is
the segment's final state from S = 0 and M its final state from S = I with
v = 0 (both computed by the chunked prefill on the segment).  With one
exchange step -- an all-gather of every rank's (M, B) -- rank r folds the
maps of ranks 0..r-1 into its true start state, then runs its segment from
it.  The pages describe no multi-device prefill; this is built on the
checkpoint semantics they do give (a state summarises its prefix exactly).

Every rank passes the same ``initial_state`` (or None for zeros); rank r
returns its segment's output and the state at its segment's end (the last
rank's is the whole sequence's final state).  The device work runs in the
library's kernels (``ops`` defaults to them); the collective is
``torch.distributed.all_gather`` (NCCL on GPUs).
"""
from __future__ import annotations

import torch


class KernelOps:
    """The library's kernels, for tensors on a CUDA device."""

    @staticmethod
    def chunk_fwd(q, k, v, g, beta, initial_state):
        from . import kda_chunk_fwd
        return kda_chunk_fwd(q, k, v, g, beta, initial_state=initial_state)

    @staticmethod
    def affine(M, B, S):
        from . import kda_state_affine
        return kda_state_affine(M, B, S)


def segment_map(q, k, v, g, beta, ops=KernelOps):
    """(M, B) of this segment's chunk map S_end = M S_start + B, per
    (sequence, head): M [B, H, dk, dk], B [B, H, dk, dv]."""
    Bn, T, H, dk = q.shape
    _, Bmap = ops.chunk_fwd(q, k, v, g, beta, None)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(Bn, H, dk, dk).contiguous()
    zero_v = torch.zeros(Bn, T, H, dk, dtype=v.dtype, device=v.device)
    _, M = ops.chunk_fwd(q, k, zero_v, g, beta, eye)
    return M, Bmap


def start_state(maps, S0, ops=KernelOps):
    """The state after applying the segment maps (M_0, B_0), (M_1, B_1), ...
    in order to S0 (a tensor of the B shape)."""
    S = S0
    for M, Bm in maps:
        S = ops.affine(M, Bm, S)
    return S


def cp_chunk_fwd(q, k, v, g, beta, initial_state=None, group=None, ops=KernelOps):
    """This rank's segment of a batch of sequences split along time across
    ``group``: q, k, g [B, T_r, H, dk]; v [B, T_r, H, dv]; beta [B, T_r, H].
    Returns (out [B, T_r, H, dv], state at this segment's end)."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    M, Bmap = segment_map(q, k, v, g, beta, ops)
    Ms = [torch.empty_like(M) for _ in range(world)]
    Bs = [torch.empty_like(Bmap) for _ in range(world)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Bs, Bmap.contiguous(), group=group)
    S0 = initial_state if initial_state is not None else torch.zeros_like(Bmap)
    S = start_state(list(zip(Ms[:rank], Bs[:rank])), S0, ops)
    return ops.chunk_fwd(q, k, v, g, beta, S)
