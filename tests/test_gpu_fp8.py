"""FP8 (e4m3) index keys on the GPU, through the C ABI, against the float64 oracle:

- the row quantiser: codes and scales bit-exact (both sides round the same fp32 quotients);
- the decode step with FP8 index scoring: selection bit-exact except near-ties, attention on the
  rows whose selection matches, and the cutoff margins r_(k) - r_(k+1);
- the cutoff margins of the bf16 decode step;
- flips between the bf16 and the FP8 selection happen only where the bf16 margin is within the
  quantisation's own bound on the score change ("4.1.1 · 监督与联合训练", section 2 and eq (9)).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from parity import NEAR_TIE, check_attention, compare_blocks

pytestmark = pytest.mark.gpu

DEV = "cuda"


def zero_sign(codes):
    """e4m3 codes with -0 (0x80) written as +0: the sign of a zero is not part of the contract."""
    c = np.array(codes, dtype=np.uint8, copy=True)
    c[c == 0x80] = 0
    return c


def spread_rows(rows, n, seed):
    """Rows of N(0,1) values times 2^p with p from -24 to 12 per row (subnormal codes, large
    scales), a zero row and a row with a single non-zero entry."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, n, generator=g) * torch.exp2(torch.randint(-24, 13, (rows, 1), generator=g).float())
    if rows > 2:
        x[1] = 0.0
        x[2] = 0.0
        x[2, n // 2] = -3.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,n", [(1000, 64), (7, 32), (33, 16), (5, 128), (3, 256), (4097, 64), (0, 64)])
def test_quantize_rows_matches_oracle(rows, n):
    x = spread_rows(rows, n, seed=rows * 7 + n)
    codes, scale = msa.msa_quantize_e4m3_rows(x.to(DEV))
    torch.cuda.synchronize()
    oc, osc = oracle.quantize_e4m3_rows(x)
    np.testing.assert_array_equal(zero_sign(codes.cpu().numpy()), zero_sign(oc))
    np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), osc.view(np.uint32))


def test_quantize_three_dim_cache_layout():
    """A K_idx cache [B, L, d_idx] quantises row by row: scales [B, L]."""
    x = spread_rows(2 * 333, 64, seed=5).reshape(2, 333, 64)
    codes, scale = msa.msa_quantize_e4m3_rows(x.to(DEV))
    oc, osc = oracle.quantize_e4m3_rows(x)
    assert tuple(codes.shape) == (2, 333, 64) and tuple(scale.shape) == (2, 333)
    np.testing.assert_array_equal(zero_sign(codes.cpu().numpy()), zero_sign(oc))
    np.testing.assert_array_equal(scale.cpu().numpy(), osc)


DECODE_SHAPES = [(3, 1000, 64, 4, 128, 64, 128, 16), (2, 700, 4, 2, 64, 32, 32, 4), (2, 901, 16, 2, 64, 64, 64, 8),
                 (1, 300, 8, 8, 128, 32, 128, 1), (2, 1001, 8, 2, 64, 64, 128, 4), (2, 702, 8, 2, 64, 64, 32, 6),
                 (2, 900, 8, 4, 64, 64, 64, 5)]


def decode_case(shape, seed):
    B, L, H_q, H_kv, d, d_idx, bk, k = shape
    gen = torch.Generator().manual_seed(seed + L)
    mkr = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    kc, vc, kic = mkr(B, L, H_kv, d), mkr(B, L, H_kv, d), mkr(B, L, d_idx)
    q, qi = mkr(B, H_q, d), mkr(B, H_kv, d_idx)
    lens = torch.tensor([L, L // 2 + 17, 130][:B], dtype=torch.int32)
    dm = msa.MsaDims(B, L, H_q, H_kv, d, d_idx, bk, k)
    od = oracle.Dims(B, L, H_q, H_kv, d, d_idx, bk, k)
    return dm, od, dict(q=q, q_idx=qi, k_cache=kc, v_cache=vc, k_idx_cache=kic, cache_len=lens)


def check_margins(gm, om):
    """Cutoff margins: +inf exactly where every candidate is taken, else within NEAR_TIE."""
    gm = np.asarray(gm, dtype=np.float64)
    om = np.asarray(om, dtype=np.float64)
    assert np.array_equal(np.isinf(gm), np.isinf(om))
    fin = np.isfinite(om)
    if fin.any():
        err = np.abs(gm[fin] - om[fin]).max()
        assert err <= NEAR_TIE, f"margin max abs error {err:.3e}"


@pytest.mark.parametrize("shape", DECODE_SHAPES)
def test_decode_fp8idx_matches_oracle(shape):
    dm, od, x = decode_case(shape, seed=199)
    g = {k: v.to(DEV) for k, v in x.items()}
    kcodes, kscale = msa.msa_quantize_e4m3_rows(g["k_idx_cache"])
    out, blocks, margin = msa.msa_sparse_attn_decode_fp8idx(dm, g["cache_len"], g["q"], g["q_idx"], g["k_cache"],
                                                            g["v_cache"], kcodes, kscale, want_margin=True)
    torch.cuda.synchronize()
    okc, oks = oracle.quantize_e4m3_rows(x["k_idx_cache"])
    ob, om, oo, _ = oracle.decode_fp8idx(od, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                         okc, oks)
    bad, near = compare_blocks(blocks.cpu().numpy(), ob, om)
    assert bad == 0, f"{bad} selection rows differ (near-ties excluded: {near})"
    check_margins(margin.cpu().numpy(), om)
    same = np.all(blocks.cpu().numpy() == ob, axis=-1)
    G = dm.H_q // dm.H_kv
    og = out.cpu().numpy()
    for b in range(dm.B):
        for r in range(dm.H_kv):
            if same[b, r]:
                check_attention(og[b, r * G:(r + 1) * G], oo[b, r * G:(r + 1) * G])


@pytest.mark.parametrize("shape", DECODE_SHAPES[:2])
def test_decode_bf16_margins_match_oracle(shape):
    dm, od, x = decode_case(shape, seed=299)
    g = {k: v.to(DEV) for k, v in x.items()}
    out, blocks, margin = msa.msa_sparse_attn_decode(dm, g["cache_len"], g["q"], g["q_idx"], g["k_cache"],
                                                     g["v_cache"], g["k_idx_cache"], want_margin=True)
    out2, blocks2 = msa.msa_sparse_attn_decode(dm, g["cache_len"], g["q"], g["q_idx"], g["k_cache"], g["v_cache"],
                                               g["k_idx_cache"])
    torch.cuda.synchronize()
    ob, om, _, _ = oracle.decode(od, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                 x["k_idx_cache"])
    check_margins(margin.cpu().numpy(), om)
    # asking for the margins changes nothing else
    assert torch.equal(blocks, blocks2) and torch.equal(out, out2)


def score_change_bound(od, x, okc, oks):
    """Per (sequence, group): max over the complete past tokens of |S_fp8 - S_bf16|, from the
    oracle's dequantised index vectors in float64. A block maximum moves by at most this much."""
    qc, qs = oracle.quantize_e4m3_rows(x["q_idx"])
    qd = oracle.dequantize_e4m3_rows(qc, qs).numpy()
    kd = oracle.dequantize_e4m3_rows(okc, oks).numpy()
    q16 = x["q_idx"].double().numpy()
    k16 = x["k_idx_cache"].double().numpy()
    sc = 1.0 / np.sqrt(od.d_idx)
    eps = np.zeros((od.B, od.H_kv))
    for b in range(od.B):
        n = (int(x["cache_len"][b]) - 1) // od.block_k * od.block_k
        for r in range(od.H_kv):
            if n > 0:
                eps[b, r] = np.abs(kd[b, :n] @ qd[b, r] - k16[b, :n] @ q16[b, r]).max() * sc
    return eps


def test_fp8_flips_only_within_the_quantisation_bound():
    """A row's FP8 selection can differ from its bf16 selection only if the bf16 cutoff margin is
    at most twice the largest change quantisation makes to one of its scores (plus the near-tie
    tolerance of the GPU's own rounding). Also reports how many rows flip."""
    shape = (3, 4000, 16, 4, 128, 64, 32, 16)
    dm, od, x = decode_case(shape, seed=7)
    g = {k: v.to(DEV) for k, v in x.items()}
    kcodes, kscale = msa.msa_quantize_e4m3_rows(g["k_idx_cache"])
    _, b16 = msa.msa_sparse_attn_decode(dm, g["cache_len"], g["q"], g["q_idx"], g["k_cache"], g["v_cache"],
                                        g["k_idx_cache"])
    _, b8 = msa.msa_sparse_attn_decode_fp8idx(dm, g["cache_len"], g["q"], g["q_idx"], g["k_cache"], g["v_cache"],
                                              kcodes, kscale)
    torch.cuda.synchronize()
    _, om16, _, _ = oracle.decode(od, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                  x["k_idx_cache"])
    okc, oks = oracle.quantize_e4m3_rows(x["k_idx_cache"])
    eps = score_change_bound(od, x, okc, oks)
    flipped = np.any(b16.cpu().numpy() != b8.cpu().numpy(), axis=-1)
    assert np.all(om16[flipped] <= 2 * eps[flipped] + 2 * NEAR_TIE), (om16[flipped], eps[flipped])
    print(f"fp8 vs bf16 selection: {int(flipped.sum())} of {flipped.size} rows differ; "
          f"median bf16 margin {np.median(om16):.3e}, score change bound median {np.median(eps):.3e}")


def test_decode_short_caches_both_scorings():
    """Edge cases of the decode step in both scorings: a cache of one token (no past block, the
    local block only), exactly one block, one block plus one token, and a cache with exactly topk
    complete past blocks (every candidate taken: margin +inf)."""
    B, L, H_q, H_kv, d, d_idx, bk, k = 4, 700, 16, 2, 128, 64, 64, 5
    gen = torch.Generator().manual_seed(5150)
    mkr = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    kc, vc, kic = mkr(B, L, H_kv, d), mkr(B, L, H_kv, d), mkr(B, L, d_idx)
    q, qi = mkr(B, H_q, d), mkr(B, H_kv, d_idx)
    lens = torch.tensor([1, bk, bk + 1, k * bk + 3], dtype=torch.int32)
    dm = msa.MsaDims(B, L, H_q, H_kv, d, d_idx, bk, k)
    od = oracle.Dims(B, L, H_q, H_kv, d, d_idx, bk, k)
    g = {n: t.to(DEV) for n, t in dict(q=q, qi=qi, kc=kc, vc=vc, kic=kic, lens=lens).items()}
    codes, kscale = msa.msa_quantize_e4m3_rows(g["kic"])
    out16, b16, m16 = msa.msa_sparse_attn_decode(dm, g["lens"], g["q"], g["qi"], g["kc"], g["vc"], g["kic"],
                                                 want_margin=True)
    out8, b8, m8 = msa.msa_sparse_attn_decode_fp8idx(dm, g["lens"], g["q"], g["qi"], g["kc"], g["vc"], codes, kscale,
                                                     want_margin=True)
    torch.cuda.synchronize()
    ob, om, oo, _ = oracle.decode(od, lens, q, qi, kc, vc, kic)
    okc, oks = oracle.quantize_e4m3_rows(kic)
    ob8, om8, oo8, _ = oracle.decode_fp8idx(od, lens, q, qi, kc, vc, okc, oks)
    for gb, gm, go, rb, rm, ro in ((b16, m16, out16, ob, om, oo), (b8, m8, out8, ob8, om8, oo8)):
        bad, _ = compare_blocks(gb.cpu().numpy(), rb, rm)
        assert bad == 0
        check_margins(gm.cpu().numpy(), rm)
        assert np.isinf(gm.cpu().numpy()).all()  # at most topk complete past blocks in every row
        check_attention(go.cpu().numpy(), ro)
