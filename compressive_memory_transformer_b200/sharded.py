"""Sequence sharding of the Linear-mode forward over the ranks of a process group
(one GPU per rank).

The Linear memory after a stretch of segments is the incoming memory plus a plain
sum of per-segment terms (M_s = M_{s-1} + sigma(K_s)^T V_s, z likewise: "Leave No
Context Behind", arXiv 2404.07143, as quoted on llm-papers-study.pages.dev, section
3.4). So a sequence cut into consecutive ranges, one per rank in rank order, needs a
single exchange: every rank sums its own range from the zero state
(infini_attn_state_update), the ranks all-gather those sums (d*d + d floats per
head), and every rank runs its forward from the incoming state plus the sums of the
ranges before it (infini_attn_state_sum, then infini_attn_forward). All arithmetic
runs in the CUDA library; this module only moves tensors and calls the collective.
The Linear+Delta memory is not such a sum (each segment's update reads the memory
before it), so it has no sharded form here.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import LINEAR, infini_attn_forward, infini_attn_state_sum, infini_attn_state_update


def gather_states(dM: torch.Tensor, dz: torch.Tensor, group=None):
    """All-gathers every rank's (dM [B, H, d, d], dz [B, H, d]) into
    ([world, B, H, d, d], [world, B, H, d]) in rank order."""
    world = dist.get_world_size(group)
    flat = torch.cat([dM.reshape(-1), dz.reshape(-1)])
    parts = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(parts, flat, group=group)
    allf = torch.stack(parts)
    nM = dM.numel()
    return (allf[:, :nM].reshape(world, *dM.shape).contiguous(),
            allf[:, nM:].reshape(world, *dz.shape).contiguous())


def sequence_sharded_linear_forward(q, k, v, beta, N, M_in=None, z_in=None, group=None,
                                    out=None, stream=None):
    """This rank's part of a Linear-mode forward over a sequence whose consecutive
    ranges are held by the ranks in rank order. q, k, v: this rank's range, [B, H, L_r,
    d] bf16, L_r a multiple of N on every rank but the last. (M_in, z_in): the state
    before the whole sequence (None: zero), the same on every rank. Returns (out_r, M,
    z) with M, z the state after the whole sequence (every rank gets it)."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    L_r = q.shape[2]
    if rank < world - 1 and L_r % N != 0:
        raise ValueError("every range but the last must hold whole segments (L_r % N == 0)")
    dM, dz = infini_attn_state_update(k, v, N, LINEAR, stream=stream)
    dM_all, dz_all = gather_states(dM, dz, group)
    M_pre, z_pre = infini_attn_state_sum(dM_all[:rank], dz_all[:rank], M_in, z_in, stream=stream)
    M_end, z_end = infini_attn_state_sum(dM_all, dz_all, M_in, z_in, stream=stream)
    out, _, _ = infini_attn_forward(q, k, v, beta, N, LINEAR, M_pre, z_pre, out=out,
                                    state_out=False, stream=stream)
    return out, M_end, z_end
