"""Seeded synthetic inputs for the MSA workloads (shared by the tests, the oracle runs and bench.py).

This module draws random numbers and plants structure; it holds none of the method's arithmetic.
Workload ``c`` draws from ``torch.Generator(device).manual_seed(1000 + c)`` (or a caller seed), in
the order Q, K, V, Q_idx, K_idx, with float32 normal draws rounded to bfloat16.

Workloads (sizes from the MSA main configuration: H_q=64, H_kv=4, d=128, d_idx=64, B_k=128, k=16):

1. ``tiny``: N=512, H_q=4, H_kv=2, d=64, d_idx=32, B_k=32, k=4; i.i.d. N(0,1).
2. ``prefill_8k``: N=8192, i.i.d. N(0,1). With the 1/sqrt(d) factors the scores already have
   unit variance, so no further scaling is applied.
3. ``prefill_32k_needles``: N=32768. Needle blocks = {0} plus 32 distinct blocks drawn from
   1..nb-1. Per KV head r a direction u_r ~ N(0, I_d) and for the index branch u_idx ~ N(0, I_didx).
   Every token j of a needle block gets K[j,r] = 3 u_r + eps and K_idx[j] = 3 u_idx + eps (eps are
   the i.i.d. draws). A Bernoulli(1/2) subset of query rows gets Q[i,h] = (u_{r(h)} + eps)/sqrt(2)
   and Q_idx[i,r] = (u_idx + eps)/sqrt(2). Selection is skewed towards the needles (hot blocks).
4. ``train_64k``: N=65536, i.i.d. N(0,1); forward plus KL alignment.
5. ``decode_16x256k``: 16 sequences with 262144 cached tokens each, one new query token per
   sequence (already appended, so the query sits at position L-1). Caches i.i.d. N(0,1); per
   sequence 8 distinct planted blocks in 0..nb-2 get K = 3 u_r + eps and K_idx = 3 u_idx + eps;
   the decode query carries the directions as in workload 3.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    B: int
    N: int
    H_q: int
    H_kv: int
    d: int
    d_idx: int
    block_k: int
    topk: int
    kind: str  # "prefill", "train" or "decode"
    needles: bool = False


WORKLOADS = {
    "tiny": Workload(1, "tiny", 1, 512, 4, 2, 64, 32, 32, 4, "train"),
    "prefill_8k": Workload(2, "prefill_8k", 1, 8192, 64, 4, 128, 64, 128, 16, "prefill"),
    "prefill_32k_needles": Workload(3, "prefill_32k_needles", 1, 32768, 64, 4, 128, 64, 128, 16, "prefill",
                                    needles=True),
    "train_64k": Workload(4, "train_64k", 1, 65536, 64, 4, 128, 64, 128, 16, "train"),
    "decode_16x256k": Workload(5, "decode_16x256k", 16, 262144, 64, 4, 128, 64, 128, 16, "decode", needles=True),
}


def _randn(shape, gen, device, chunk_elems: int = 1 << 27) -> torch.Tensor:
    """Normal draws rounded to bfloat16, generated in float32 chunks to bound temporary memory."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def make_generator(w: Workload, device, seed: int | None = None) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1000 + w.cid if seed is None else seed)
    return g


def prefill_inputs(w: Workload, device="cpu", seed: int | None = None, N: int | None = None) -> dict:
    """Q [B,N,H_q,d], K/V [B,N,H_kv,d], Q_idx [B,N,H_kv,d_idx], K_idx [B,N,d_idx] in bfloat16.

    ``N`` overrides the sequence length (same recipe, smaller size) for quick cases.
    """
    N = w.N if N is None else N
    g = make_generator(w, device, seed)
    q = _randn((w.B, N, w.H_q, w.d), g, device)
    k = _randn((w.B, N, w.H_kv, w.d), g, device)
    v = _randn((w.B, N, w.H_kv, w.d), g, device)
    q_idx = _randn((w.B, N, w.H_kv, w.d_idx), g, device)
    k_idx = _randn((w.B, N, w.d_idx), g, device)
    out = {"q": q, "k": k, "v": v, "q_idx": q_idx, "k_idx": k_idx}
    if w.needles:
        nb = -(-N // w.block_k)
        G = w.H_q // w.H_kv
        perm = torch.randperm(nb - 1, generator=g, device=device)[: min(32, nb - 1)] + 1
        needle_blocks = torch.cat([torch.zeros(1, dtype=torch.long, device=device), perm.to(torch.long)])
        u = torch.randn(w.H_kv, w.d, generator=g, device=device)
        u_idx = torch.randn(w.d_idx, generator=g, device=device)
        tok = (needle_blocks[:, None] * w.block_k + torch.arange(w.block_k, device=device)[None, :]).reshape(-1)
        tok = tok[tok < N]
        k[:, tok] = (3.0 * u[None, None] + k[:, tok].float()).to(torch.bfloat16)
        k_idx[:, tok] = (3.0 * u_idx[None, None] + k_idx[:, tok].float()).to(torch.bfloat16)
        carry = torch.rand(w.B, N, generator=g, device=device) < 0.5
        u_h = u.repeat_interleave(G, dim=0)  # direction of each query head's group
        qf = q.float()
        q.copy_(torch.where(carry[..., None, None], (u_h[None, None] + qf) / math.sqrt(2.0), qf).to(torch.bfloat16))
        qif = q_idx.float()
        q_idx.copy_(torch.where(carry[..., None, None], (u_idx[None, None, None] + qif) / math.sqrt(2.0), qif)
                    .to(torch.bfloat16))
        out["needle_blocks"] = needle_blocks
        out["needle_rows"] = carry
    return out


def decode_inputs(w: Workload, device="cpu", seed: int | None = None, L: int | None = None,
                  B: int | None = None) -> dict:
    """Caches k_cache/v_cache [B,L,H_kv,d], k_idx_cache [B,L,d_idx]; queries q [B,H_q,d],
    q_idx [B,H_kv,d_idx]; cache_len [B] int32 (all full). ``L`` / ``B`` override the sizes."""
    L = w.N if L is None else L
    B = w.B if B is None else B
    g = make_generator(w, device, seed)
    G = w.H_q // w.H_kv
    q = _randn((B, w.H_q, w.d), g, device)
    k = _randn((B, L, w.H_kv, w.d), g, device)
    v = _randn((B, L, w.H_kv, w.d), g, device)
    q_idx = _randn((B, w.H_kv, w.d_idx), g, device)
    k_idx = _randn((B, L, w.d_idx), g, device)
    nb = -(-L // w.block_k)
    u = torch.randn(w.H_kv, w.d, generator=g, device=device)
    u_idx = torch.randn(w.d_idx, generator=g, device=device)
    planted = []
    for b in range(B):
        blk = torch.randperm(max(nb - 1, 1), generator=g, device=device)[: min(8, max(nb - 1, 1))]
        planted.append(blk)
        tok = (blk[:, None] * w.block_k + torch.arange(w.block_k, device=device)[None, :]).reshape(-1)
        tok = tok[tok < L]
        k[b, tok] = (3.0 * u[None] + k[b, tok].float()).to(torch.bfloat16)
        k_idx[b, tok] = (3.0 * u_idx[None] + k_idx[b, tok].float()).to(torch.bfloat16)
    u_h = u.repeat_interleave(G, dim=0)
    q.copy_(((u_h[None] + q.float()) / math.sqrt(2.0)).to(torch.bfloat16))
    q_idx.copy_(((u_idx[None, None] + q_idx.float()) / math.sqrt(2.0)).to(torch.bfloat16))
    cache_len = torch.full((B,), L, dtype=torch.int32, device=device)
    return {"q": q, "q_idx": q_idx, "k_cache": k, "v_cache": v, "k_idx_cache": k_idx, "cache_len": cache_len,
            "planted_blocks": torch.stack(planted)}


def small_prefill(N: int, H_q: int, H_kv: int, d: int, d_idx: int, block_k: int, topk: int, seed: int,
                  B: int = 1, device="cpu", dtype=torch.bfloat16) -> dict:
    """i.i.d. N(0,1) inputs of arbitrary small sizes (edge cases, ragged tails)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g, device=device, dtype=torch.float32).to(dtype)
    return {"q": mk(B, N, H_q, d), "k": mk(B, N, H_kv, d), "v": mk(B, N, H_kv, d),
            "q_idx": mk(B, N, H_kv, d_idx), "k_idx": mk(B, N, d_idx)}
