"""Randomised shapes, every one checked against the float64 oracle: a seeded sweep over the sizes
the library supports (batch 1-3, ragged N up to ~3000, 1-8 KV groups, 1-32 query heads per group,
d in {64, 128}, d_idx in {32, 64}, B_k in {32, 64, 128}, k in 1..16) so that no combination of
tile edges, group sizes and block sizes is only ever exercised by the handful of fixed cases.

Per case: the selection (bit-exact outside near-ties) and LSE_idx; the attention on the oracle's
selection (fp32 output on sampled rows, and the bf16 output equal to it rounded); the KL loss and
both index gradients where the KL kernel supports the group size; the backward where its kernel
supports it. Decode: random cache lengths per sequence against the oracle's decode."""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from msa_inputs import small_prefill
from parity import KL_REL, check_attention, check_bwd, check_grad, compare_blocks, report

pytestmark = pytest.mark.gpu

DEV = "cuda"


def draw_case(seed):
    """A supported configuration drawn from `seed` (numpy's generator, nothing of the method)."""
    rng = np.random.default_rng(10_000 + seed)
    d, d_idx = [(128, 64), (64, 32), (128, 32), (64, 64)][rng.integers(4)]
    bk = int(rng.choice([32, 64, 128]))
    H_kv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4, 8, 16, 32]))
    while H_kv * G > 64:
        G //= 2
    B = int(rng.integers(1, 4))
    N = int(np.exp(rng.uniform(np.log(2), np.log(3000))))
    k = int(rng.integers(1, 17))
    return B, N, H_kv * G, H_kv, d, d_idx, bk, k


CASES = list(range(32))


def case_id(seed):
    B, N, H_q, H_kv, d, d_idx, bk, k = draw_case(seed)
    return f"s{seed}-B{B}-N{N}-G{H_q // H_kv}x{H_kv}-d{d}-di{d_idx}-bk{bk}-k{k}"


@pytest.mark.parametrize("seed", CASES, ids=[case_id(s) for s in CASES])
def test_random_shape_matches_oracle(seed):
    B, N, H_q, H_kv, d, d_idx, bk, k = draw_case(seed)
    G = H_q // H_kv
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=20_000 + seed, B=B)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, k)
    g = {kk: vv.to(DEV) for kk, vv in x.items()}

    # selection and LSE_idx
    blocks, lse_idx = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"], want_lse=True)
    torch.cuda.synchronize()
    ob, om, ol = oracle.index_topk(od, x["q_idx"], x["k_idx"], want_lse=True)
    bad, near = compare_blocks(blocks.cpu().numpy(), ob, om)
    report(f"random case {case_id(seed)}: {near} of {om.size} (row, group) pairs near-tied")
    assert bad == 0
    same = np.all(blocks.cpu().numpy().reshape(ob.shape) == ob, axis=-1)
    assert np.abs(lse_idx.cpu().numpy().reshape(ol.shape) - ol)[same].max() <= 1e-3

    # attention on the oracle's selection (every input independent of the CUDA path)
    obb = ob.reshape(B, N, H_kv, k + 1)
    bo = torch.from_numpy(obb).to(DEV)
    out, lse = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], bo)
    o16, _ = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], bo, want_lse=False, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(o16, out.to(torch.bfloat16))
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, B * N - 1], rng.choice(B * N, size=min(96, B * N), replace=False)]))
    oo, olse = oracle.sparse_attn(od, x["q"], x["k"], x["v"], obb, rows=rows)
    check_attention(out.cpu().numpy().reshape(B * N, H_q, d)[rows], oo,
                    lse.cpu().numpy().reshape(B * N, H_q)[rows], olse)

    # KL alignment where its kernel supports the group size
    if ((d, d_idx) in ((128, 64), (64, 32))) and G in (2, 16):
        gs = float(B * N * H_kv)
        loss, dq, dk = msa.msa_kl_fwd_grad(dm, g["q"], g["k"], g["q_idx"], g["k_idx"], bo, lse, None, grad_scale=gs)
        torch.cuda.synchronize()
        l_o, _, odq, odk = oracle.kl(od, x["q"], x["k"], x["q_idx"], x["k_idx"], obb, grad_scale=gs)
        assert abs(loss.item() - l_o) <= KL_REL * abs(l_o), f"loss {loss.item()} vs {l_o}"
        check_grad(dq.cpu().numpy().reshape(odq.shape), odq, "dq_idx")
        check_grad(dk.cpu().numpy(), odk, "dk_idx")

    # backward where its kernel supports the group size
    if G in (8, 16, 32):
        gen = torch.Generator().manual_seed(30_000 + seed)
        dout = torch.randn(B, N, H_q, d, generator=gen).to(torch.bfloat16)
        dq, dk, dv = msa.msa_sparse_attn_bwd(dm, g["q"], g["k"], g["v"], bo, out, lse, dout.to(DEV))
        torch.cuda.synchronize()
        rq, rk, rv = oracle.sparse_attn_bwd(od, x["q"], x["k"], x["v"], obb, dout)
        check_bwd(dq.cpu().numpy(), rq, "dq")
        check_bwd(dk.cpu().numpy(), rk, "dk")
        check_bwd(dv.cpu().numpy(), rv, "dv")


DECODE_CASES = list(range(10))


@pytest.mark.parametrize("seed", DECODE_CASES)
def test_random_decode_matches_oracle(seed):
    rng = np.random.default_rng(40_000 + seed)
    d, d_idx = [(128, 64), (64, 32), (128, 32), (64, 64)][rng.integers(4)]
    bk = int(rng.choice([32, 64, 128]))
    H_kv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4, 8, 16]))
    while H_kv * G > 64:
        G //= 2
    H_q = H_kv * G
    B = int(rng.integers(1, 5))
    L = int(rng.integers(200, 5000))
    k = int(rng.integers(1, 17))
    lens = rng.integers(1, L + 1, size=B).astype(np.int32)
    lens[0] = L  # one sequence at the caches' capacity
    gen = torch.Generator().manual_seed(50_000 + seed)
    mk = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    x = dict(q=mk(B, H_q, d), q_idx=mk(B, H_kv, d_idx), k_cache=mk(B, L, H_kv, d), v_cache=mk(B, L, H_kv, d),
             k_idx_cache=mk(B, L, d_idx), cache_len=torch.from_numpy(lens))
    g = {kk: vv.to(DEV) for kk, vv in x.items()}
    dm = msa.MsaDims(B, L, H_q, H_kv, d, d_idx, bk, k)
    out, blocks = msa.msa_sparse_attn_decode(dm, g["cache_len"], g["q"], g["q_idx"], g["k_cache"], g["v_cache"],
                                             g["k_idx_cache"])
    torch.cuda.synchronize()
    od = oracle.Dims(B, L, H_q, H_kv, d, d_idx, bk, k)
    ob, om, oo, _ = oracle.decode(od, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                  x["k_idx_cache"])
    gb = blocks.cpu().numpy()
    bad, near = compare_blocks(gb, ob, om)
    report(f"random decode case {seed} (B={B}, L={L}, G={G}x{H_kv}, d={d}, d_idx={d_idx}, bk={bk}, k={k}): "
           f"{near} of {om.size} pairs near-tied")
    assert bad == 0
    same = np.all(gb == ob, axis=-1)
    og = out.cpu().numpy()
    for b in range(B):
        for r in range(H_kv):
            if same[b, r]:
                check_attention(og[b, r * G:(r + 1) * G], oo[b, r * G:(r + 1) * G])


SP_CASES = list(range(8))


@pytest.mark.parametrize("seed", SP_CASES)
def test_random_sequence_parallel_matches_single_device(seed):
    """P emulated ranks (2-8) on random shapes, zig-zag and contiguous key assignments: the merged
    selection is the single-device selection bit for bit, LSE_idx the same value summed in
    another order."""
    from block_sparse_attention_idx_b200 import sp
    B, N, H_q, H_kv, d, d_idx, bk, k = draw_case(100 + seed)
    P = int(np.random.default_rng(60_000 + seed).integers(2, 9))
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=70_000 + seed, B=B, device=DEV)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    ref_blocks, ref_lse = msa.msa_index_topk(dm, x["q_idx"], x["k_idx"], want_lse=True)
    for ranges_of in (sp.zigzag_ranges, sp.contiguous_ranges):
        helds = [ranges_of(N, bk, P, p) for p in range(P)]
        cs, ci = [], []
        for h in helds:
            c = (msa.msa_index_topk_local(dm, x["q_idx"], sp.local_keys(x["k_idx"], h), h) if h
                 else sp.no_candidates(dm, x["q_idx"].device))
            cs.append(c[0])
            ci.append(c[1])
        blocks = msa.msa_topk_merge(dm, torch.stack(cs), torch.stack(ci))
        ml = torch.stack([msa.msa_lse_idx_local(dm, x["q_idx"], sp.local_keys(x["k_idx"], h), h, blocks) if h
                          else sp.no_lse_pairs(dm, x["q_idx"].device) for h in helds])
        lse = msa.msa_lse_combine(dm, ml)
        torch.cuda.synchronize()
        assert torch.equal(blocks, ref_blocks), ranges_of.__name__
        assert torch.allclose(lse, ref_lse, rtol=0, atol=2e-5 * max(1.0, float(ref_lse.abs().max())))


DENSE_CASES = list(range(6))


@pytest.mark.parametrize("seed", DENSE_CASES)
def test_random_dense_warmup_matches_oracle(seed):
    """The dense warm-up KL on random shapes its kernels support (G in {2, 16}, matching head
    dims, every block size): loss, both index gradients and the teacher LSE against the oracle's KL
    with every causal block selected."""
    rng = np.random.default_rng(80_000 + seed)
    d, d_idx = [(128, 64), (64, 32)][rng.integers(2)]
    G = int(rng.choice([2, 16]))
    H_kv = int(rng.choice([1, 2, 4]))
    bk = int(rng.choice([32, 64, 128]))
    B = int(rng.integers(1, 3))
    N = int(rng.integers(2, 900))
    H_q = G * H_kv
    nb = -(-N // bk)
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, 4, seed=90_000 + seed, B=B)
    g = {kk: vv.to(DEV) for kk, vv in x.items()}
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, 1)
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, max(nb - 1, 1))
    gs = float(B * N * H_kv)
    loss, dq, dk, lse = msa.msa_kl_dense_fwd_grad(dm, g["q"], g["k"], g["q_idx"], g["k_idx"], grad_scale=gs,
                                                  want_lse=True)
    torch.cuda.synchronize()
    ids = np.arange(nb, dtype=np.int32)[None, :].repeat(N, 0)
    ids[ids > (np.arange(N) // bk)[:, None]] = -1
    # one more slot than the oracle's k + 1 is never needed: k + 1 = max(nb, 2) >= nb
    full = np.full((N, od.topk + 1), -1, dtype=np.int32)
    full[:, :nb] = ids
    blocks = np.broadcast_to(full[None, :, None, :], (B, N, H_kv, od.topk + 1)).copy()
    ol, _, odq, odk = oracle.kl(od, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, grad_scale=gs)
    _, olse = oracle.sparse_attn(od, x["q"], x["k"], x["v"], blocks)
    assert abs(float(loss.item()) - ol) <= KL_REL * max(abs(ol), 1e-12), f"loss {loss.item()} vs {ol}"
    check_grad(dq.cpu().numpy().reshape(odq.shape), odq, "dq_idx")
    check_grad(dk.cpu().numpy(), odk, "dk_idx")
    assert np.abs(lse.cpu().numpy().reshape(olse.shape) - olse).max() <= 2e-3


FP8_CASES = list(range(6))


@pytest.mark.parametrize("seed", FP8_CASES)
def test_random_fp8_decode_matches_oracle(seed):
    """The FP8-index decode step on random shapes: the quantiser's codes and scales bit-exact, then
    selection (outside near-ties), cutoff margins and attention against the oracle's FP8 decode."""
    rng = np.random.default_rng(95_000 + seed)
    d, d_idx = [(128, 64), (64, 32), (128, 32), (64, 64)][rng.integers(4)]
    bk = int(rng.choice([32, 64, 128]))
    H_kv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4, 8, 16]))
    while H_kv * G > 64:
        G //= 2
    H_q = H_kv * G
    B = int(rng.integers(1, 5))
    L = int(rng.integers(200, 5000))
    k = int(rng.integers(1, 17))
    lens = rng.integers(1, L + 1, size=B).astype(np.int32)
    lens[-1] = L
    gen = torch.Generator().manual_seed(96_000 + seed)
    mk = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    x = dict(q=mk(B, H_q, d), q_idx=mk(B, H_kv, d_idx), k_cache=mk(B, L, H_kv, d), v_cache=mk(B, L, H_kv, d),
             k_idx_cache=mk(B, L, d_idx), cache_len=torch.from_numpy(lens))
    g = {kk: vv.to(DEV) for kk, vv in x.items()}
    dm = msa.MsaDims(B, L, H_q, H_kv, d, d_idx, bk, k)
    kcodes, kscale = msa.msa_quantize_e4m3_rows(g["k_idx_cache"])
    out, blocks, margin = msa.msa_sparse_attn_decode_fp8idx(dm, g["cache_len"], g["q"], g["q_idx"], g["k_cache"],
                                                            g["v_cache"], kcodes, kscale, want_margin=True)
    torch.cuda.synchronize()
    okc, oks = oracle.quantize_e4m3_rows(x["k_idx_cache"])
    gc = kcodes.cpu().numpy().copy()
    gc[gc == 0x80] = 0  # a negative value rounded to zero may keep its sign bit (either code is zero)
    okc0 = okc.copy()
    okc0[okc0 == 0x80] = 0
    np.testing.assert_array_equal(gc, okc0)
    np.testing.assert_array_equal(kscale.cpu().numpy(), oks)
    od = oracle.Dims(B, L, H_q, H_kv, d, d_idx, bk, k)
    ob, om, oo, _ = oracle.decode_fp8idx(od, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"], okc,
                                         oks)
    gb = blocks.cpu().numpy()
    bad, near = compare_blocks(gb, ob, om)
    assert bad == 0
    gm = margin.cpu().numpy()
    assert np.array_equal(np.isinf(gm), np.isinf(om))
    fin = np.isfinite(om)
    assert np.abs(gm[fin] - om[fin]).max(initial=0.0) <= 1e-4
    same = np.all(gb == ob, axis=-1)
    og = out.cpu().numpy()
    for b in range(B):
        for r in range(H_kv):
            if same[b, r]:
                check_attention(og[b, r * G:(r + 1) * G], oo[b, r * G:(r + 1) * G])
