"""Sequence-parallel index branch over torch.distributed (one process per GPU, NCCL).

Rank p of P holds tokens [tok0_p, tok0_p + ntok_p) of every sequence's keys, the ranges tiling
[0, N) in rank order ("4.1.1 · 监督与联合训练", section 3: local top candidates, exchange of
(score, index) pairs only, and the global log-sum-exp from each rank's local maximum and exp-sum,
eq (16)). Every rank ends with the same selection and LSE_idx as the single-device index pass.
The computation runs in libmsa's kernels; this module only moves the candidates between ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (MsaDims, msa_index_topk_local, msa_lse_combine, msa_lse_idx_local, msa_topk_merge)


def split_range(N: int, block_k: int, world: int, rank: int):
    """(tok0, ntok) of rank `rank`: whole blocks, as even as possible, the last range ending at N."""
    nb = -(-N // block_k)
    b0 = rank * nb // world
    b1 = (rank + 1) * nb // world
    tok0 = b0 * block_k
    return tok0, min(b1 * block_k, N) - tok0


def gather(t: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' copies of `t`, stacked in rank order: [P, *t.shape]."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def sp_index_topk(dims: MsaDims, q_idx, k_idx_local, tok0: int, want_lse: bool = False, group=None):
    """Selection blocks [B, N, H_kv, topk+1] (and LSE_idx [B, N, H_kv]) of all N tokens from this
    rank's key range; q_idx [B, N, H_kv, d_idx] is replicated on every rank."""
    empty = k_idx_local.shape[1] == 0  # more ranks than blocks: this rank holds no key
    cs, ci = no_candidates(dims, q_idx.device) if empty else msa_index_topk_local(dims, q_idx, k_idx_local, tok0)
    blocks = msa_topk_merge(dims, gather(cs, group), gather(ci, group))
    if not want_lse:
        return blocks
    ml = no_lse_pairs(dims, q_idx.device) if empty else msa_lse_idx_local(dims, q_idx, k_idx_local, tok0, blocks)
    return blocks, msa_lse_combine(dims, gather(ml, group))


def no_candidates(dims: MsaDims, device):
    """The candidates of a rank that holds no key: scores -inf and ids -1 [B, N, H_kv, topk], the
    padding of a row without candidates."""
    shape = (dims.B, dims.N, dims.H_kv, dims.topk)
    return (torch.full(shape, float("-inf"), dtype=torch.float32, device=device),
            torch.full(shape, -1, dtype=torch.int32, device=device))


def no_lse_pairs(dims: MsaDims, device):
    """The (max, exp-sum) pairs of a rank that holds no key: (-inf, 0), which eq (16) ignores."""
    ml = torch.zeros(dims.B, dims.N, dims.H_kv, 2, dtype=torch.float32, device=device)
    ml[..., 0] = float("-inf")
    return ml
