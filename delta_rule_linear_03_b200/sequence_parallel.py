"""Prefill of one sequence sharded along L over the ranks of a process group.

Rank r holds the contiguous segment r of every (b, h) sequence (segments in
rank order).  The state after a segment is affine in the state before it,
S_out = M_r S_in + S_r, because the recurrence of the pages' 关键设计 2 is
linear in S.  Each rank therefore:

1. runs its segment from zero and from the identity (rank 0 from the true S0
   instead, which also gives its final outputs);
2. exchanges the two final states with every rank in one ``all_gather``;
3. composes the maps of the ranks before it into its true initial state,
   S_in(r+1) = (S_I - S_Z)_r S_in(r) + S_Z,r  (``efla_state_affine``);
4. reruns its segment from that state, which gives its outputs and final
   state.

The only collective is step 2: 2 * B * H * d * d fp32 per rank.  Computation
runs in the library's kernels; torch.distributed carries the exchange.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

Segment = Callable[..., Tuple[torch.Tensor, torch.Tensor]]
Affine = Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor]


def _gpu_segment(q, k, v, beta, S0, mode, out_dtype):
    from . import chunk_fwd
    return chunk_fwd(q, k, v, beta, S0, mode=mode, out_dtype=out_dtype)


def _gpu_affine(SI, SZ, X):
    from . import state_affine
    return state_affine(SI, SZ, X)


def initial_state(maps, S0: torch.Tensor, upto: int, affine: Affine) -> torch.Tensor:
    """True initial state of segment ``upto`` from the per-segment final
    states ``maps[r] = (S_Z, S_I)`` of the segments before it and the
    sequence's S0 (segment 0 contributes its true final state as both)."""
    S = S0
    for r in range(upto):
        SZ, SI = maps[r]
        S = affine(SI, SZ, S) if r > 0 else SZ
    return S


def chunk_fwd_sequence_sharded(q, k, v, beta, S0=None, mode: str = "exact", group=None,
                               out_dtype=torch.float32, segment: Optional[Segment] = None,
                               affine: Optional[Affine] = None):
    """``q, k`` [B,H,L_r,d], ``v`` [B,H,L_r,d], ``beta`` [B,H,L_r]: this rank's
    segment.  ``S0`` [B,H,d,d] fp32 (the sequence's initial state, the same
    on every rank) or None.  Returns (o of this segment, final state of this
    segment); on the last rank the latter is the sequence's S_L.

    ``segment`` / ``affine`` default to the library's kernels; tests pass
    other implementations of the same contracts."""
    segment = segment or _gpu_segment
    affine = affine or _gpu_affine
    B, H, _, d = k.shape
    if v.shape[-1] != d:
        raise ValueError("sequence sharding needs d_k == d_v (the identity as an initial state)")
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    zeros = torch.zeros(B, H, d, d, dtype=torch.float32, device=k.device)
    S0 = zeros if S0 is None else S0
    if world == 1:
        return segment(q, k, v, beta, S0, mode, out_dtype)
    if rank == 0:
        o, S_end = segment(q, k, v, beta, S0, mode, out_dtype)
        SZ, SI = S_end, S_end
    else:
        eye = torch.eye(d, dtype=torch.float32, device=k.device).expand(B, H, d, d).contiguous()
        _, SZ = segment(q, k, v, beta, zeros, mode, out_dtype)
        _, SI = segment(q, k, v, beta, eye, mode, out_dtype)
    mine = torch.stack([SZ.contiguous(), SI.contiguous()])
    gathered = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(gathered, mine, group=group)
    if rank == 0:
        return o, S_end
    maps = [(g[0], g[1]) for g in gathered]
    S_in = initial_state(maps, S0, rank, affine)
    return segment(q, k, v, beta, S_in.contiguous(), mode, out_dtype)
