"""Sequence-parallel index branch over torch.distributed (one process per GPU, NCCL).

Each rank holds one or two ranges of every sequence's keys (whole blocks; across the ranks the
ranges tile [0, N)). "4.1.1 · 监督与联合训练", section 3: every rank takes its local top candidates,
only (score, index) pairs are exchanged, and the global log-sum-exp comes from each rank's local
maximum and exp-sum, eq (16). Every rank ends with the same selection and LSE_idx as the
single-device index pass. The computation runs in libmsa's kernels; this module only decides which
keys a rank holds and moves the candidates between ranks.

Work balance: under the causal mask, block c is a complete past block of the queries after it, so
a rank's local Top-k costs about the number of (query, held past block) pairs. Contiguous ranges
give the first rank the blocks every later query scores; the zig-zag assignment (chunk p and chunk
2P-1-p of 2P equal chunks) pairs an early chunk with a late one and evens the ranks out.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (MsaDims, msa_index_topk_local, msa_lse_combine, msa_lse_idx_local, msa_topk_merge)


def _chunk_tokens(N: int, block_k: int, parts: int, j: int):
    """(tok0, ntok) of chunk j of `parts` near-equal chunks of whole blocks (the last ends at N)."""
    nb = -(-N // block_k)
    b0, b1 = j * nb // parts, (j + 1) * nb // parts
    tok0 = b0 * block_k
    return tok0, min(b1 * block_k, N) - tok0


def contiguous_ranges(N: int, block_k: int, world: int, rank: int):
    """Rank `rank`'s key ranges [(tok0, ntok)] under the contiguous assignment: one range of about
    nb / world blocks, in rank order ([] for a rank that gets no block)."""
    r = _chunk_tokens(N, block_k, world, rank)
    return [r] if r[1] > 0 else []


def zigzag_ranges(N: int, block_k: int, world: int, rank: int):
    """Rank `rank`'s key ranges [(tok0, ntok), ...] under the zig-zag assignment: chunks `rank` and
    2 * world - 1 - rank of 2 * world near-equal chunks of blocks, empty chunks left out."""
    parts = 2 * world
    held = [_chunk_tokens(N, block_k, parts, rank), _chunk_tokens(N, block_k, parts, parts - 1 - rank)]
    return [r for r in held if r[1] > 0]


def local_keys(k_idx: torch.Tensor, held) -> torch.Tensor:
    """The K_idx a rank stores for its ranges, [B, sum ntok, d_idx]: the first range's tokens, then
    the second's (the layout msa_index_topk_local / msa_lse_idx_local read)."""
    return torch.cat([k_idx[:, t0:t0 + n] for t0, n in held], dim=1).contiguous()


def gather(t: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' copies of `t`, stacked in rank order: [P, *t.shape]. NCCL gathers device memory in
    place; gloo moves host memory, so a device tensor is staged through the host there."""
    world = dist.get_world_size(group)
    if t.is_cuda and dist.get_backend(group) == "nccl":
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out
    src = t.detach().cpu().contiguous()
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    return torch.stack(parts).to(t.device)


def sp_index_topk(dims: MsaDims, q_idx, k_idx_local, held, want_lse: bool = False, group=None):
    """Selection blocks [B, N, H_kv, topk+1] (and LSE_idx [B, N, H_kv]) of all N tokens from this
    rank's keys: `held` its ranges [(tok0, ntok), ...] (one or two; [] for none) and k_idx_local
    their tokens in that order (local_keys). q_idx [B, N, H_kv, d_idx] is replicated on every
    rank. Every rank of the group must call it."""
    empty = len(held) == 0  # more ranks than blocks: this rank holds no key
    cs, ci = no_candidates(dims, q_idx.device) if empty else msa_index_topk_local(dims, q_idx, k_idx_local, held)
    blocks = msa_topk_merge(dims, gather(cs, group), gather(ci, group))
    if not want_lse:
        return blocks
    ml = no_lse_pairs(dims, q_idx.device) if empty else msa_lse_idx_local(dims, q_idx, k_idx_local, held, blocks)
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
