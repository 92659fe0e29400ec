"""Sequence sharding of the Linear-mode forward over the ranks of a process group
(one GPU per rank).

The Linear memory after a stretch of segments is the incoming memory plus a plain
sum of per-segment terms (M_s = M_{s-1} + sigma(K_s)^T V_s, z likewise: "Leave No
Context Behind", arXiv 2404.07143, as quoted on llm-papers-study.pages.dev, section
3.4). So a sequence cut into consecutive ranges, one per rank in rank order, needs a
single exchange: every rank sums its own range from the zero state
(infini_attn_state_update), the ranks all-gather those sums (d*d + d floats per
head, plus the range's length), and every rank runs its forward from the incoming
state plus the sums of the ranges before it (infini_attn_state_sum, then
infini_attn_forward). All arithmetic runs in the CUDA library; this module only
moves tensors and calls the collective.
The Linear+Delta memory is not such a sum (each segment's update reads the memory
before it), so it has no sharded form here.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import LINEAR, infini_attn_forward, infini_attn_state_sum, infini_attn_state_update


def _all_gather_rows(flat: torch.Tensor, group=None) -> torch.Tensor:
    """[world, n] stack of every rank's 1-D tensor, in rank order, on flat's device.
    The gloo backend moves host tensors, so a device payload is staged through host
    memory there; NCCL gathers device memory directly."""
    world = dist.get_world_size(group)
    staged = flat.is_cuda and dist.get_backend(group) == dist.Backend.GLOO
    send = flat.cpu() if staged else flat
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    return torch.stack(parts).to(flat.device)


def gather_states(dM: torch.Tensor, dz: torch.Tensor, group=None, length: int = 0):
    """All-gathers every rank's (dM [B, H, d, d], dz [B, H, d] float32) and its range
    length in one collective. Returns ([world, B, H, d, d], [world, B, H, d], lengths)
    in rank order; the floats travel bit for bit (as int32 words)."""
    words = torch.cat([dM.reshape(-1).view(torch.int32), dz.reshape(-1).view(torch.int32),
                       torch.tensor([length], dtype=torch.int32, device=dM.device)])
    allw = _all_gather_rows(words, group)
    nM, nz = dM.numel(), dz.numel()
    world = allw.shape[0]
    dM_all = allw[:, :nM].contiguous().view(torch.float32).reshape(world, *dM.shape)
    dz_all = allw[:, nM:nM + nz].contiguous().view(torch.float32).reshape(world, *dz.shape)
    return dM_all, dz_all, [int(x) for x in allw[:, -1].tolist()]


def sequence_sharded_linear_forward(q, k, v, beta, N, M_in=None, z_in=None, group=None,
                                    out=None, stream=None):
    """This rank's part of a Linear-mode forward over a sequence whose consecutive
    ranges are held by the ranks in rank order. q, k, v: this rank's range, [B, H, L_r,
    d] bf16, L_r a multiple of N on every rank but the last. (M_in, z_in): the state
    before the whole sequence (None: zero), the same on every rank. Returns (out_r, M,
    z) with M, z the state after the whole sequence (every rank gets it).

    Every rank learns every range's length from the one all-gather, so a range that
    breaks the rule raises ValueError on all ranks together (none is left waiting in a
    collective)."""
    rank = dist.get_rank(group)
    L_r = q.shape[2]
    dM, dz = infini_attn_state_update(k, v, N, LINEAR, stream=stream)
    dM_all, dz_all, lengths = gather_states(dM, dz, group, L_r)
    bad = [r for r, n in enumerate(lengths[:-1]) if n % N != 0]
    if bad:
        raise ValueError(f"ranges of ranks {bad} do not hold whole segments: every range but "
                         f"the last must have a length that is a multiple of N = {N}")
    M_pre, z_pre = infini_attn_state_sum(dM_all[:rank], dz_all[:rank], M_in, z_in, stream=stream)
    M_end, z_end = infini_attn_state_sum(dM_all, dz_all, M_in, z_in, stream=stream)
    out, _, _ = infini_attn_forward(q, k, v, beta, N, LINEAR, M_pre, z_pre, out=out,
                                    state_out=False, stream=stream)
    return out, M_end, z_end
