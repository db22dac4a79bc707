"""Context-parallel prefill: every sequence is split into contiguous segments, one per rank.

Eq. (5) of "On the design of Qwen3.8-Next architecture", section 2.1.1, makes each token's
update affine in the state, S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, so a
segment maps its initial state to S_end = M S_start + B.  Each rank

1. forms its segment's maps with two chunked passes (`segment_maps`): M = S_T from S0 = I with
   v = 0 and B = S_T from S0 = 0,
2. exchanges them with one all-gather (`gather_maps`; NCCL over NVLink between GPUs, no
   multicast),
3. folds the maps of the ranks before it onto the sequences' initial state (`fold_maps`, one
   `gdn_state_map_apply` launch per earlier rank), and
4. runs the chunked pass over its segment from that state (`finish`).

Every step on the device is a libgdn launch.  This module only orders the calls and the
exchange.  The fold is host logic over a list of maps, so `fold_maps` takes the apply step as an
argument and can be exercised on any backend.
"""
from __future__ import annotations

import torch

from . import gdn


def segment_maps(q, k, v, g, beta, cu_seqlens=None, num_seqs=None, chunk=64, workspace=None, stream=None):
    """(M, B) of this rank's segment of every sequence: M [num_seqs, H, dk, dk] is the state the
    segment leaves when it starts from I with v = 0, B [num_seqs, H, dk, dv] the state it leaves
    from zero (both through gdn_chunk_fwd)."""
    N, H, dk = q.shape
    if cu_seqlens is not None:
        num_seqs = cu_seqlens.numel() - 1
    elif num_seqs is None:
        num_seqs = 1
    dev = q.device
    eye = torch.eye(dk, device=dev, dtype=torch.float32).expand(num_seqs, H, dk, dk).contiguous()
    zero_v = torch.zeros(N, H, dk, device=dev, dtype=v.dtype)
    _, M = gdn.chunk_fwd(q, k, zero_v, g, beta, S0=eye, cu_seqlens=cu_seqlens, num_seqs=num_seqs, chunk=chunk,
                         workspace=workspace, stream=stream)
    _, B = gdn.chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=cu_seqlens, num_seqs=num_seqs, chunk=chunk,
                         workspace=workspace, stream=stream)
    return M, B


def gather_maps(M, B, group=None):
    """All ranks' (M, B), in rank order, from one all-gather of the packed pair (every rank's
    maps have the same shape: its segment of the same sequences and heads)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    packed = torch.cat([M.reshape(-1), B.reshape(-1)])
    out = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(out, packed, group=group)
    nm = M.numel()
    return [(o[:nm].view_as(M), o[nm:].view_as(B)) for o in out]


def fold_maps(maps, rank, S0, apply):
    """The initial state of segment `rank`: S0 with the maps of segments 0 .. rank-1 applied in
    order, S <- M_j S + B_j, through apply(M, B, S)."""
    S = S0
    for j in range(rank):
        S = apply(maps[j][0], maps[j][1], S)
    return S


def finish(maps, rank, q, k, v, g, beta, S0=None, cu_seqlens=None, num_seqs=None, chunk=64, y=None, S_T=None,
           workspace=None, stream=None):
    """y and the final state of segment `rank`, from the gathered maps and the sequences'
    initial state S0 (None: zero)."""
    if S0 is None:
        S0 = torch.zeros_like(maps[0][1])
    S_start = fold_maps(maps, rank, S0, lambda M, B, S: gdn.state_map_apply(M, B, S, stream=stream))
    return gdn.chunk_fwd(q, k, v, g, beta, S0=S_start, cu_seqlens=cu_seqlens, num_seqs=num_seqs, chunk=chunk, y=y,
                         S_T=S_T, workspace=workspace, stream=stream)


def cp_prefill(q, k, v, g, beta, S0=None, cu_seqlens=None, num_seqs=None, chunk=64, group=None, workspace=None,
               stream=None):
    """One rank's part of a context-parallel prefill.  q, k, v, g, beta hold this rank's
    segment of every sequence (packed by cu_seqlens); S0 is the sequences' initial state, the
    same on every rank.  Returns this segment's y and final state; the last rank's final state
    is the sequences' S_T."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    M, B = segment_maps(q, k, v, g, beta, cu_seqlens=cu_seqlens, num_seqs=num_seqs, chunk=chunk, workspace=workspace,
                        stream=stream)
    maps = gather_maps(M, B, group=group)
    return finish(maps, rank, q, k, v, g, beta, S0=S0, cu_seqlens=cu_seqlens, num_seqs=num_seqs, chunk=chunk,
                  workspace=workspace, stream=stream)
