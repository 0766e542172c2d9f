"""Host-side selection metrics of the oracle (test infrastructure only).

- ``topk_ids``: Top-k positions of a score vector; equal scores go to the lower position
  ("4.1.1 supervision and joint training", section 2: fix a secondary sort key for ties).
- ``recall_at_k``: R_i@k = |S_i ∩ G_i| / |G_i|  (same page, eq (2)).
- ``coverage``: C_i = sum_{j in S_i} p_ij, the teacher probability mass covered  (same page, eq (3)).
- ``output_error``: E_i = ||o_sparse - o_dense||_2 / (||o_dense||_2 + eps)  (same page, eq (14)).
- ``cutoff_margin``: Delta_i = r_(k) - r_(k+1)  (same page, eq (9)).
"""
from __future__ import annotations

import numpy as np


def topk_ids(scores, k: int) -> list[int]:
    """Positions of the k largest scores, ranked by (score desc, position asc)."""
    s = np.asarray(scores, dtype=np.float64)
    order = sorted(range(len(s)), key=lambda j: (-s[j], j))
    return order[:k]


def recall_at_k(selected, ideal) -> float:
    S, G = set(int(x) for x in selected), set(int(x) for x in ideal)
    return len(S & G) / len(G)


def coverage(selected, p) -> float:
    p = np.asarray(p, dtype=np.float64)
    return float(sum(p[int(j)] for j in set(int(x) for x in selected)))


def cutoff_margin(scores, k: int) -> float:
    s = sorted(np.asarray(scores, dtype=np.float64), reverse=True)
    return float(s[k - 1] - s[k]) if len(s) > k else float("inf")


def output_error(o_sparse, o_dense, eps: float = 1e-12) -> np.ndarray:
    a = np.asarray(o_sparse, dtype=np.float64)
    b = np.asarray(o_dense, dtype=np.float64)
    return np.linalg.norm(a - b, axis=-1) / (np.linalg.norm(b, axis=-1) + eps)
