"""Sequence-parallel KDA forward over ranks of a torch.distributed group.

The worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and
Anthropic Systems on Independent Benchmarks", paragraph 3: FlashKDA
reconstructs the sequential states across GPUs with a prefix scan.  Here rank r
holds the r-th contiguous time segment of every sequence (all ranks the same
batch, heads and segment length).  Over a segment the state map is affine,
S_end = M S_start + N, so:

1. every rank but the last computes its segment's maps [M | N]
   (kda_segment_maps, one tensor-core launch);
2. the maps are all-gathered (the one data-path exchange: d_k (d_k + d_v) fp32
   values per sequence and head, 128 KiB at d = 128);
3. rank r applies the maps of ranks 0 .. r-1 to S0 (kda_segment_scan, fp32) to
   get its start state;
4. rank r runs kda_forward on its segment from that state.

The last rank's final state is the sequence's final state.  Every step that
touches the data runs in the library's kernels; this module only moves tensors
and calls the collective.  With a gloo group the maps travel through host
memory; with NCCL they stay on the device.
"""
from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import kda


def kda_forward_sequence_parallel(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  alpha: torch.Tensor, beta: torch.Tensor,
                                  S0: Optional[torch.Tensor] = None, group=None,
                                  stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's outputs [B, T_r, H, d_v] and the state after its segment.

    q, k, alpha [B, T_r, H, d_k], v [B, T_r, H, d_v], beta [B, T_r, H]: this
    rank's segment (bf16, d_k = d_v = 128).  S0: fp32 [B, H, d_k, d_v] or None,
    the state before rank 0's segment; every rank passes the same values (or
    None).  Collective: every rank of `group` calls it with the same B, H, T_r.
    Without a process group (one process) it is kda_forward.
    """
    single = group is None and not (dist.is_available() and dist.is_initialized())
    world = 1 if single else dist.get_world_size(group)
    rank = 0 if single else dist.get_rank(group)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    start = S0
    if world > 1:
        if rank < world - 1:
            maps = kda.kda_segment_maps(k, v, alpha, beta, stream=stream)
        else:   # the last segment's map is not needed by anyone
            maps = torch.zeros(B, H, dk, dk + dv, dtype=torch.float32, device=q.device)
        if dist.get_backend(group) == "gloo":   # host-memory exchange
            parts = [torch.empty(maps.shape, dtype=maps.dtype) for _ in range(world)]
            dist.all_gather(parts, maps.cpu(), group=group)
            gathered = torch.stack(parts).to(q.device)
        else:
            gathered = torch.empty((world,) + tuple(maps.shape), dtype=maps.dtype, device=q.device)
            dist.all_gather_into_tensor(gathered, maps, group=group)
        if rank > 0:
            start = kda.kda_segment_scan(gathered[:rank].contiguous(), S0, stream=stream)
    return kda.kda_forward(q, k, v, alpha, beta, start, stream=stream)


def split_time(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """Rank `rank`'s contiguous slice of dimension 1 (time) of x, split into
    `world` equal segments (T must be a multiple of world)."""
    T = x.shape[1]
    if T % world:
        raise ValueError("T must be a multiple of the world size")
    n = T // world
    return x[:, rank * n:(rank + 1) * n].contiguous()
