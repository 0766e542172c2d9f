"""Sequence-parallel indexer: plain float64 restatement of the exchange that lets P ranks, each
holding some ranges of every sequence's key blocks, reproduce the single-device selection
and LSE_idx ("4.1.1 · 监督与联合训练", section 3: each rank takes its local top candidates and
only the (score, index) pairs are exchanged and merged; the global log-sum-exp comes from each
rank's local maximum a_p and exp-sum z_p by eq (16)).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle``. Small cases: Python loops over rows.
"""
from __future__ import annotations

import math

import numpy as np

from . import Dims, block_max_row, index_scores_row


def held_blocks(held):
    """The block ids of a rank's held ranges [(blk0, blk1), ...] (each half-open)."""
    return sorted({c for b0, b1 in held for c in range(b0, b1)})


def local_topk(dims: Dims, q_idx, k_idx, held):
    """For every (b, i, r): the Top-k of the complete past blocks c < b_i that the rank holds (c in
    one of its block ranges `held` = [(blk0, blk1), ...]) by (M desc, id asc). Returns scores
    [B, N, H_kv, k] (M with scale_idx, -inf padded) and ids (int32, -1 padded)."""
    mine = held_blocks(held)
    k = dims.topk
    scores = np.full((dims.B, dims.N, dims.H_kv, k), -np.inf)
    ids = np.full((dims.B, dims.N, dims.H_kv, k), -1, dtype=np.int32)
    for b in range(dims.B):
        for i in range(dims.N):
            bi = i // dims.block_k
            for r in range(dims.H_kv):
                M = block_max_row(dims, index_scores_row(dims, q_idx, k_idx, b, i, r), i)
                cand = sorted((c for c in mine if c < bi), key=lambda c: (-M[c], c))[:k]
                for p, c in enumerate(cand):
                    scores[b, i, r, p] = M[c]
                    ids[b, i, r, p] = c
    return scores, ids


def merge(dims: Dims, cand_scores, cand_ids):
    """Union of the P ranks' candidate lists, Top-k by (score desc, id asc), plus each row's local
    block; ascending, -1 padded: blocks [B, N, H_kv, k + 1]."""
    k = dims.topk
    S = np.concatenate(list(cand_scores), axis=-1)
    I = np.concatenate(list(cand_ids), axis=-1)
    blocks = np.full((dims.B, dims.N, dims.H_kv, k + 1), -1, dtype=np.int32)
    for b in range(dims.B):
        for i in range(dims.N):
            for r in range(dims.H_kv):
                pairs = [(S[b, i, r, x], I[b, i, r, x]) for x in range(S.shape[-1]) if I[b, i, r, x] >= 0]
                top = [c for _, c in sorted(pairs, key=lambda p: (-p[0], p[1]))[:k]]
                sel = sorted(top + [i // dims.block_k])
                blocks[b, i, r, :len(sel)] = sel
    return blocks


def local_lse(dims: Dims, q_idx, k_idx, blocks, held):
    """Per (b, i, r): (a_p, z_p) = (max, sum of exp(s - a_p)) of the index scores over the causal
    tokens of the selected blocks the rank holds (block ranges `held`); (-inf, 0) when there are
    none."""
    mine = set(held_blocks(held))
    out = np.zeros((dims.B, dims.N, dims.H_kv, 2))
    for b in range(dims.B):
        for i in range(dims.N):
            for r in range(dims.H_kv):
                s = index_scores_row(dims, q_idx, k_idx, b, i, r)
                J = [j for c in blocks[b, i, r] if c in mine
                     for j in range(c * dims.block_k, min((c + 1) * dims.block_k, i + 1))]
                if not J:
                    out[b, i, r] = (-np.inf, 0.0)
                    continue
                a = max(s[j] for j in J)
                out[b, i, r] = (a, sum(math.exp(s[j] - a) for j in J))
    return out


def combine_lse(pairs):
    """Eq (16): a = max_p a_p, z = sum_p exp(a_p - a) z_p, LSE = a + log z. pairs: [P, ..., 2]."""
    P = np.asarray(pairs, dtype=np.float64)
    a = P[..., 0].max(axis=0)
    w = np.where(np.isneginf(P[..., 0]), 0.0, np.exp(P[..., 0] - a))
    z = (w * P[..., 1]).sum(axis=0)
    return a + np.log(z)
