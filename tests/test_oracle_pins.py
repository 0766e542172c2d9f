"""Pins of the float64 oracle against what the pages and the mathematics fix (CPU only).

Each test ties one part of the oracle to something other than itself: a worked example printed
on the pages, a closed form, an identity, a special case that reduces to a library routine, or
brute force written independently here on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import metrics
from msa_inputs import small_prefill

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


# ----------------------------------------------------------------------------- worked examples
def test_fig1_recall_and_coverage():
    """4.1.1 · 监督与联合训练, Figure 1: student (0.7,-0.2,1.1), k=2 -> {1,3}; teacher top-2 {1,2};
    recall 1/2, coverage 0.70."""
    g = GOLDEN["fig1_recall_coverage"]
    s_top = sorted(j + 1 for j in metrics.topk_ids(g["student_scores"], g["k"]))
    t_top = sorted(j + 1 for j in metrics.topk_ids(g["teacher_probs"], g["k"]))
    assert s_top == g["student_topk"] and t_top == g["teacher_topk"]
    sel0 = [j - 1 for j in s_top]
    assert metrics.recall_at_k(sel0, [j - 1 for j in t_top]) == pytest.approx(g["recall"], abs=1e-15)
    assert metrics.coverage(sel0, g["teacher_probs"]) == pytest.approx(g["coverage"], abs=1e-12)
    # Top-k on raw scores equals Top-k on softmaxed scores (MSA blog, softmax-free Top-K)
    sm = torch.softmax(torch.tensor(g["student_scores"], dtype=torch.float64), 0).numpy()
    assert sorted(metrics.topk_ids(sm, g["k"])) == sorted(metrics.topk_ids(g["student_scores"], g["k"]))


def test_fig1_through_the_oracle_selection():
    """The same example through the C oracle's block selection: three complete past blocks with
    maxima (0.7,-0.2,1.1), k=2, query in block 3 -> past blocks {0,2} plus the local block 3."""
    g = GOLDEN["fig1_recall_coverage"]
    dims = oracle.Dims(B=1, N=64, H_q=1, H_kv=1, d=8, d_idx=8, block_k=8, topk=2)
    M = np.array(g["student_scores"] + [-5.0])  # local block's max is irrelevant under reading 0
    sel, margin, n = oracle.select_from_max(dims, M, i=3 * 8 + 2)
    assert n == 3 and list(sel) == [0, 2, 3]
    assert margin == pytest.approx(0.7 - (-0.2), abs=1e-15)


def test_sec1_recall_vs_mass():
    g = GOLDEN["sec1_recall_vs_mass"]
    ideal = metrics.topk_ids(g["teacher_probs"], g["k"])
    for c in ("A", "B"):
        sel = [j - 1 for j in g[f"candidate_{c}"]]
        assert metrics.recall_at_k(sel, ideal) == pytest.approx(g[f"{c}_recall"], abs=1e-15)
        assert metrics.coverage(sel, g["teacher_probs"]) == pytest.approx(g[f"{c}_mass"], abs=1e-12)


def test_sec1_2_budget_quality():
    g = GOLDEN["sec1_2_budget_quality"]
    p = g["teacher_probs"]
    ideal = metrics.topk_ids(p, g["k"])
    assert metrics.coverage(ideal, p) == pytest.approx(g["oracle_coverage"], abs=1e-12)
    sel = [j - 1 for j in g["student_blocks"]]
    assert metrics.recall_at_k(sel, ideal) == pytest.approx(g["student_recall"], abs=1e-12)
    assert metrics.coverage(sel, p) == pytest.approx(g["student_coverage"], abs=1e-12)


def test_eq11_two_position_example():
    """2.4 · 训练原生稀疏 eq (11): weights (0.75,0.25) (a logit gap of ln 3), v1=(2,0), v2=(0,2)
    give o=(1.5,0.5); with upstream g=(1,-1) the logit gradients are 0.75 and -0.75. The gradient
    is taken here by central differences of the oracle's attention output."""
    g = GOLDEN["eq11_two_position"]
    q = np.array([1.0, 0.0])
    k = np.array([[math.log(3.0), 0.0], [0.0, 0.0]])
    v = np.array(g["values"])
    o, lse = oracle.attend_tokens(q, k, v, [0, 1], scale=1.0)
    np.testing.assert_allclose(o, g["output"], atol=1e-14)
    assert lse == pytest.approx(math.log(4.0), abs=1e-14)
    up = np.array(g["upstream_grad"])
    h = 1e-6
    for s, want in enumerate(g["logit_grads"]):
        kp, km = k.copy(), k.copy()
        kp[s, 0] += h  # q = e_0, so this moves logit s by exactly h
        km[s, 0] -= h
        lp = up @ oracle.attend_tokens(q, kp, v, [0, 1], 1.0)[0]
        lm = up @ oracle.attend_tokens(q, km, v, [0, 1], 1.0)[0]
        assert (lp - lm) / (2 * h) == pytest.approx(want, abs=1e-8)


# ----------------------------------------------------------------------------- identities
def test_deletion_identity():
    """4.1.1 eq (17): o^(-j) - o = p_j/(1-p_j) (o - v_j), with p_j recovered from the two LSEs."""
    rng = np.random.default_rng(7)
    d, n = 16, 40
    q, k, v = rng.normal(size=d), rng.normal(size=(n, d)), rng.normal(size=(n, d))
    J = list(range(n))
    o, lse = oracle.attend_tokens(q, k, v, J, 0.25)
    for j in (0, 13, 39):
        oj, lsej = oracle.attend_tokens(q, k, v, [t for t in J if t != j], 0.25)
        pj = 1.0 - math.exp(lsej - lse)
        np.testing.assert_allclose(oj - o, pj / (1 - pj) * (o - v[j]), atol=1e-12)


def test_partition_merge_identity():
    """2.4 eq (18) / 4.1.1 eq (16): attention over J1 ∪ J2 equals the softmax-state merge of the two
    parts (m, l folded into each part's LSE)."""
    rng = np.random.default_rng(3)
    d, n = 8, 50
    q, k, v = rng.normal(size=d), rng.normal(size=(n, d)) * 2, rng.normal(size=(n, d))
    J1, J2 = list(range(0, 50, 3)), [t for t in range(50) if t % 3]
    o, lse = oracle.attend_tokens(q, k, v, list(range(n)), 0.5)
    o1, l1 = oracle.attend_tokens(q, k, v, J1, 0.5)
    o2, l2 = oracle.attend_tokens(q, k, v, J2, 0.5)
    a = max(l1, l2)
    z = math.exp(l1 - a) + math.exp(l2 - a)
    assert lse == pytest.approx(a + math.log(z), abs=1e-12)
    np.testing.assert_allclose(o, (math.exp(l1 - a) * o1 + math.exp(l2 - a) * o2) / z, atol=1e-12)


# ----------------------------------------------------------------------------- selection
def _brute_selection(dims, q_idx, k_idx):
    """Independent brute force: dense causal index scores with a matmul, block max by slicing,
    ranking with Python's sort; returns blocks [B*N, H_kv, k+1], margins, LSE_idx over J."""
    qi = q_idx.double().numpy()
    ki = k_idx.double().numpy()
    sc = dims.scale_idx or 1.0 / math.sqrt(dims.d_idx)
    Bk, k = dims.block_k, dims.topk
    out, marg, lses = [], [], []
    for b in range(dims.B):
        S = np.einsum("nrc,mc->nrm", qi[b], ki[b]) * sc
        for i in range(dims.N):
            bi = i // Bk
            row_b, row_m, row_l = [], [], []
            for r in range(dims.H_kv):
                s = S[i, r, : i + 1]
                M = [s[c * Bk: min((c + 1) * Bk, i + 1)].max() for c in range(bi + 1)]
                cand = sorted(range(bi), key=lambda c: (-M[c], c))
                sel = sorted(cand[:k] + [bi])
                row_m.append(M[cand[k - 1]] - M[cand[k]] if bi > k else math.inf)
                J = np.concatenate([np.arange(c * Bk, min((c + 1) * Bk, i + 1)) for c in sel])
                row_l.append(float(torch.logsumexp(torch.from_numpy(s[J]), 0)))
                row_b.append(sel + [-1] * (k + 1 - len(sel)))
            out.append(row_b)
            marg.append(row_m)
            lses.append(row_l)
    return np.array(out, dtype=np.int32), np.array(marg), np.array(lses)


@pytest.mark.parametrize("N,Bk,k,Hkv", [(100, 8, 3, 2), (64, 16, 2, 1), (37, 4, 5, 3), (129, 32, 4, 2)])
def test_selection_brute_force(N, Bk, k, Hkv):
    """Selection (scores, causal block max, Top-k with ties to the lower id, local block added),
    cutoff margins and LSE_idx match an independent brute force, including a ragged last block."""
    dims = oracle.Dims(B=2, N=N, H_q=Hkv, H_kv=Hkv, d=8, d_idx=8, block_k=Bk, topk=k)
    x = small_prefill(N, Hkv, Hkv, 8, 8, Bk, k, seed=N + Bk, B=2)
    blocks, margin, lse = oracle.index_topk(dims, x["q_idx"], x["k_idx"], want_lse=True)
    bb, bm, bl = _brute_selection(dims, x["q_idx"], x["k_idx"])
    np.testing.assert_array_equal(blocks, bb)
    np.testing.assert_allclose(margin, bm, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-10)


def test_ties_go_to_lower_block_id():
    dims = oracle.Dims(B=1, N=64, H_q=1, H_kv=1, d=8, d_idx=8, block_k=8, topk=2)
    sel, margin, n = oracle.select_from_max(dims, np.array([1.0, 2.0, 2.0, 2.0, 0.5, 0.0]), i=5 * 8)
    assert list(sel) == [1, 2, 5] and margin == 0.0
    sel, _, _ = oracle.select_from_max(dims, np.array([3.0, 3.0, 3.0]), i=2 * 8 + 7)
    assert list(sel) == [0, 1, 2]


def test_early_rows_and_row_zero():
    """Rows of the first blocks: fewer complete past blocks than k -> all of them plus the local
    block, -1 padded; rows of block 0 see only the local block."""
    dims = oracle.Dims(B=1, N=40, H_q=1, H_kv=1, d=8, d_idx=8, block_k=8, topk=3)
    x = small_prefill(40, 1, 1, 8, 8, 8, 3, seed=5)
    blocks, margin, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    assert list(blocks[0, 0]) == [0, -1, -1, -1] and list(blocks[7, 0]) == [0, -1, -1, -1]
    assert list(blocks[8, 0]) == [0, 1, -1, -1]
    assert list(blocks[31, 0]) == [0, 1, 2, 3] and np.isinf(margin[31, 0])
    assert len(set(blocks[39, 0])) == 4 and blocks[39, 0, -1] == 4  # local block always present


def test_local_mode_readings():
    """Reading 1 (local block inside k) equals reading 0 with k-1; reading 2 contains reading 0's
    local block and at most k+1 blocks."""
    x = small_prefill(96, 2, 2, 8, 8, 8, 4, seed=11)
    d0 = oracle.Dims(1, 96, 2, 2, 8, 8, 8, 3, local_mode=0)
    d1 = oracle.Dims(1, 96, 2, 2, 8, 8, 8, 4, local_mode=1)
    d2 = oracle.Dims(1, 96, 2, 2, 8, 8, 8, 4, local_mode=2)
    b0, _, _ = oracle.index_topk(d0, x["q_idx"], x["k_idx"])
    b1, _, _ = oracle.index_topk(d1, x["q_idx"], x["k_idx"])
    b2, _, _ = oracle.index_topk(d2, x["q_idx"], x["k_idx"])
    np.testing.assert_array_equal(b0, b1[..., :4])
    for i in range(96):
        for r in range(2):
            s = [c for c in b2[i, r] if c >= 0]
            assert i // 8 in s and len(s) <= 5


def test_raw_topk_equals_softmax_topk():
    """MSA blog (softmax-free Top-K): ranking block maxima or their softmax gives the same set."""
    dims = oracle.Dims(B=1, N=256, H_q=1, H_kv=1, d=8, d_idx=16, block_k=8, topk=6)
    x = small_prefill(256, 1, 1, 8, 16, 8, 6, seed=21)
    for i in (100, 200, 255):
        s = oracle.index_scores_row(dims, x["q_idx"], x["k_idx"], 0, i, 0)
        M = oracle.block_max_row(dims, s, i)
        sel, _, _ = oracle.select_from_max(dims, M, i)
        past = M[: i // 8]
        sm = torch.softmax(torch.from_numpy(past), 0).numpy()
        want = sorted(metrics.topk_ids(sm, 6) + [i // 8])
        assert list(sel) == want


# ----------------------------------------------------------------------------- attention
@pytest.mark.parametrize("N,Bk,G", [(70, 8, 2), (128, 32, 4)])
def test_all_blocks_is_dense_causal_attention(N, Bk, G):
    """k >= number of blocks: the selection is every causal block and the output is dense causal
    attention, checked against torch's scaled_dot_product_attention in float64."""
    Hkv = 2
    dims = oracle.Dims(B=1, N=N, H_q=Hkv * G, H_kv=Hkv, d=16, d_idx=8, block_k=Bk, topk=N // Bk + 1)
    x = small_prefill(N, Hkv * G, Hkv, 16, 8, Bk, dims.topk, seed=N)
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    for i in range(N):
        assert [c for c in blocks[i, 0] if c >= 0] == list(range(i // Bk + 1))
    out, lse = oracle.sparse_attn(dims, x["q"], x["k"], x["v"], blocks)
    q = x["q"].double().transpose(1, 2)
    k = x["k"].double().repeat_interleave(G, dim=2).transpose(1, 2)
    v = x["v"].double().repeat_interleave(G, dim=2).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    np.testing.assert_allclose(out, ref.transpose(1, 2)[0].numpy(), atol=1e-12)
    logits = (q @ k.transpose(-1, -2)) / 4.0
    logits = logits.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1)[0].T.numpy(), atol=1e-12)


def test_sparse_attention_brute_force():
    """Attention on a sparse selection equals masked dense attention (mask = selected causal
    tokens of the head's group), computed with torch in float64."""
    N, Bk, G, Hkv = 96, 8, 2, 2
    dims = oracle.Dims(B=1, N=N, H_q=G * Hkv, H_kv=Hkv, d=16, d_idx=8, block_k=Bk, topk=3)
    x = small_prefill(N, G * Hkv, Hkv, 16, 8, Bk, 3, seed=9)
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    out, lse = oracle.sparse_attn(dims, x["q"], x["k"], x["v"], blocks)
    for h in range(G * Hkv):
        r = h // G
        mask = torch.zeros(N, N, dtype=torch.bool)
        for i in range(N):
            for c in blocks[i, r]:
                if c >= 0:
                    mask[i, c * Bk: min((c + 1) * Bk, i + 1)] = True
        lg = (x["q"][0, :, h].double() @ x["k"][0, :, r].double().T) * 0.25
        lg = lg.masked_fill(~mask, -math.inf)
        p = torch.softmax(lg, -1)
        np.testing.assert_allclose(out[:, h], (p @ x["v"][0, :, r].double()).numpy(), atol=1e-12)
        np.testing.assert_allclose(lse[:, h], torch.logsumexp(lg, -1).numpy(), atol=1e-12)


# ----------------------------------------------------------------------------- KL alignment
def _f64(x):
    return {k: v.double() for k, v in x.items()}


def test_kl_brute_force():
    """KL(P || P_idx) per (row, group), with P the group average of per-head softmaxes (probability
    space, not logits) and P_idx the index softmax on the same token set, against torch float64."""
    N, Bk, G, Hkv = 64, 8, 3, 2
    dims = oracle.Dims(B=1, N=N, H_q=G * Hkv, H_kv=Hkv, d=8, d_idx=4, block_k=Bk, topk=2)
    x = small_prefill(N, G * Hkv, Hkv, 8, 4, Bk, 2, seed=4)
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    loss, kl_rows, _, _ = oracle.kl(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks)
    tot = 0.0
    for i in range(N):
        for r in range(Hkv):
            J = [t for c in blocks[i, r] if c >= 0 for t in range(c * Bk, min((c + 1) * Bk, i + 1))]
            Kj = x["k"][0, J, r].double()
            P = sum(torch.softmax((x["q"][0, i, h].double() @ Kj.T) / math.sqrt(8), 0)
                    for h in range(r * G, (r + 1) * G)) / G
            s = (x["q_idx"][0, i, r].double() @ x["k_idx"][0, J].double().T) / 2.0
            kl = float((P * (P.log() - torch.log_softmax(s, 0))).sum())
            assert kl_rows[i, r] == pytest.approx(kl, abs=1e-12)
            assert kl_rows[i, r] >= -1e-15
            tot += kl
    assert loss == pytest.approx(tot / (N * Hkv), rel=1e-12)


def test_kl_gradient_finite_differences():
    """KL alignment's analytic gradient (P_idx - P chained to q_idx, k_idx) against central
    differences of the oracle's own loss, selection held fixed, float64 inputs."""
    N, Bk, G, Hkv = 40, 8, 2, 2
    dims = oracle.Dims(B=1, N=N, H_q=G * Hkv, H_kv=Hkv, d=8, d_idx=4, block_k=Bk, topk=2)
    x = _f64(small_prefill(N, G * Hkv, Hkv, 8, 4, Bk, 2, seed=13))
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    gs = 3.0
    loss, _, dq, dk = oracle.kl(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, grad_scale=gs)
    h = 1e-5
    rng = np.random.default_rng(0)
    for _ in range(12):
        i, r, c = rng.integers(N), rng.integers(Hkv), rng.integers(4)
        qp, qm = x["q_idx"].clone(), x["q_idx"].clone()
        qp[0, i, r, c] += h
        qm[0, i, r, c] -= h
        fd = (oracle.kl(dims, x["q"], x["k"], qp, x["k_idx"], blocks)[0]
              - oracle.kl(dims, x["q"], x["k"], qm, x["k_idx"], blocks)[0]) / (2 * h)
        assert dq[i, r, c] == pytest.approx(gs * fd, rel=1e-6, abs=1e-9)
        j = rng.integers(N)
        kp, km = x["k_idx"].clone(), x["k_idx"].clone()
        kp[0, j, c] += h
        km[0, j, c] -= h
        fd = (oracle.kl(dims, x["q"], x["k"], x["q_idx"], kp, blocks)[0]
              - oracle.kl(dims, x["q"], x["k"], x["q_idx"], km, blocks)[0]) / (2 * h)
        assert dk[0, j, c] == pytest.approx(gs * fd, rel=1e-6, abs=1e-9)


def test_kl_zero_when_student_equals_teacher():
    """With G=1, d_idx=d, Q_idx=Q, K_idx=K and equal scales, P_idx = P: KL = 0 and the gradients
    vanish."""
    N, Bk = 48, 8
    dims = oracle.Dims(B=1, N=N, H_q=1, H_kv=1, d=8, d_idx=8, block_k=Bk, topk=2)
    x = small_prefill(N, 1, 1, 8, 8, Bk, 2, seed=17)
    x["q_idx"] = x["q"].clone()
    x["k_idx"] = x["k"][:, :, 0].clone()
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    loss, kl_rows, dq, dk = oracle.kl(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks)
    assert abs(loss) < 1e-14 and np.abs(kl_rows).max() < 1e-13
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14


def test_kl_row_subset_matches_full():
    N, Bk, G, Hkv = 56, 8, 2, 2
    dims = oracle.Dims(B=2, N=N, H_q=G * Hkv, H_kv=Hkv, d=8, d_idx=4, block_k=Bk, topk=2)
    x = small_prefill(N, G * Hkv, Hkv, 8, 4, Bk, 2, seed=19, B=2)
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    blocks = blocks.reshape(2, N, Hkv, 3)
    loss, kl_rows, dq, dk = oracle.kl(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks)
    rows = [3, 60, 111]
    _, kr, dqr, _ = oracle.kl(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, rows=rows)
    np.testing.assert_allclose(kr, kl_rows[rows], atol=1e-15)
    np.testing.assert_allclose(dqr, dq[rows], atol=1e-15)



def test_kl_all_blocks_is_dense_causal_kl():
    """Dense warm-up limit (k >= the number of blocks; "MSA 中的 KL 对齐与局部知识蒸馏", section 5: the
    warm-up aligns over the whole causal context): the oracle's L_KL, KL rows
    and both index gradients equal a whole-matrix computation in torch float64 -- causal masks on
    the full score matrices, the teacher as the head average of per-head softmaxes, the student as
    the index log-softmax, and autograd (not the analytic P_idx - P) for the gradients."""
    N, Bk, G, Hkv, d, di = 48, 8, 3, 2, 8, 4
    nb = N // Bk
    dims = oracle.Dims(B=1, N=N, H_q=G * Hkv, H_kv=Hkv, d=d, d_idx=di, block_k=Bk, topk=nb)
    x = _f64(small_prefill(N, G * Hkv, Hkv, d, di, Bk, nb, seed=23))
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    loss, kl_rows, dq, dk = oracle.kl(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks)
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    qi = x["q_idx"][0].clone().requires_grad_(True)  # [N, H_kv, d_idx]
    ki = x["k_idx"][0].clone().requires_grad_(True)  # [N, d_idx]
    rows = []
    for r in range(Hkv):
        kr = x["k"][0, :, r]
        P = torch.stack([torch.softmax((x["q"][0, :, h] @ kr.T / math.sqrt(d)).masked_fill(~causal, -math.inf), -1)
                         for h in range(r * G, (r + 1) * G)]).mean(0)
        logq = torch.log_softmax((qi[:, r] @ ki.T / math.sqrt(di)).masked_fill(~causal, -math.inf), -1)
        terms = torch.where(causal, P * (P.clamp_min(1e-300).log() - logq), torch.zeros((), dtype=P.dtype))
        rows.append(terms.sum(-1))
    R = torch.stack(rows, -1)
    L = R.sum() / (N * Hkv)
    L.backward()
    assert (blocks[:, :, 0] == 0).all() and (blocks >= 0).sum() == sum(i // Bk + 1 for i in range(N)) * Hkv
    np.testing.assert_allclose(kl_rows, R.detach().numpy(), rtol=0, atol=1e-12)
    assert loss == pytest.approx(float(L.detach()), rel=1e-12)
    np.testing.assert_allclose(dq.reshape(N, Hkv, di), qi.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk[0], ki.grad.numpy(), rtol=0, atol=1e-12)

# ----------------------------------------------------------------------------- decode
def test_decode_equals_prefill_last_row():
    """Replaying one new token over the cache gives the parallel causal path's row L-1
    (2.4 · 训练原生稀疏, section 3.2: token-by-token replay must match the parallel path)."""
    L, Bk, G, Hkv = 77, 8, 2, 2
    dims = oracle.Dims(B=1, N=L, H_q=G * Hkv, H_kv=Hkv, d=16, d_idx=8, block_k=Bk, topk=3)
    x = small_prefill(L, G * Hkv, Hkv, 16, 8, Bk, 3, seed=23)
    blocks, margin, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    out, lse = oracle.sparse_attn(dims, x["q"], x["k"], x["v"], blocks, rows=[L - 1])
    # capacity larger than the live length: rows past cache_len must not matter
    cap = 96
    pad = lambda t: torch.cat([t, torch.randn(1, cap - L, *t.shape[2:]).to(t.dtype)], 1)
    dd = oracle.Dims(B=1, N=cap, H_q=G * Hkv, H_kv=Hkv, d=16, d_idx=8, block_k=Bk, topk=3)
    db, dm, do, dl = oracle.decode(dd, [L], x["q"][:, L - 1], x["q_idx"][:, L - 1], pad(x["k"]), pad(x["v"]),
                                   pad(x["k_idx"]))
    np.testing.assert_array_equal(db[0], blocks[L - 1])
    np.testing.assert_allclose(do[0], out[0], atol=1e-13)
    np.testing.assert_allclose(dl[0], lse[0], atol=1e-13)


# ----------------------------------------------------------------------------- FP8 index keys
def test_e4m3_code_values_match_the_format_table():
    """Every e4m3 code decodes as the format defines it (1 sign, 4 exponent bits with bias 7,
    3 mantissa bits, subnormals, 0x7f/0xff NaN): checked against torch's float8_e4m3fn table and
    a few values written out."""
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_values(codes)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert list(np.where(np.isnan(v))[0]) == [0x7F, 0xFF]
    fin = ~np.isnan(v)
    np.testing.assert_array_equal(v[fin], t[fin])
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0  # largest finite
    assert v[0x38] == 1.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x3F] == 1.875


def test_e4m3_rounding_nearest_even_and_saturation():
    """Rounding to the nearest e4m3 value with ties to the even mantissa, as torch's float8 cast
    does for |y| <= 448; beyond 448 the serving conversion saturates to +-448."""
    rng = np.random.default_rng(7)
    y = (rng.choice([-1.0, 1.0], 200000) * np.exp2(rng.uniform(-12, 9, 200000))).astype(np.float32)
    y = y[np.abs(y) <= 448]
    c = oracle.e4m3_round(y)
    tc = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(c, tc)
    v = lambda x: float(oracle.e4m3_values(oracle.e4m3_round([x]))[0])
    assert v(1.0 + 1 / 16) == 1.0          # tie between 1 and 1.125 -> even mantissa 0
    assert v(1.0 + 3 / 16) == 1.25         # tie between 1.125 and 1.25 -> even mantissa 2
    assert v(2.0 ** -10) == 0.0            # half the smallest subnormal -> 0
    assert v(3 * 2.0 ** -10) == 2.0 ** -8  # tie between 1 and 2 subnormal quanta -> 2
    assert v(-0.3) == -0.3125
    assert v(460.0) == 448.0 and v(1e6) == 448.0 and v(-1e6) == -448.0


def test_e4m3_row_quantisation_properties():
    """Row scale max|x| / 448: each row's largest magnitude becomes exactly +-448, every value is
    reproduced within half an e4m3 step (relative 2^-4 for normal codes), and a zero row keeps
    scale 1 with zero codes."""
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(64, 32, generator=g) * torch.exp2(torch.randint(-8, 8, (64, 1), generator=g).float()))
    x[5] = 0.0
    x = x.to(torch.bfloat16)
    codes, scale = oracle.quantize_e4m3_rows(x)
    xf = x.double().numpy()
    amax = np.abs(xf).max(1)
    np.testing.assert_array_equal(scale[amax > 0], (amax[amax > 0].astype(np.float32) / np.float32(448.0)))
    assert scale[5] == 1.0 and not codes[5].any()
    vals = oracle.e4m3_values(codes)
    arg = np.abs(xf).argmax(1)
    for r in range(64):
        if amax[r] > 0:
            assert abs(vals[r, arg[r]]) == 448.0
    deq = oracle.dequantize_e4m3_rows(codes, scale).numpy()
    y = np.abs(xf) / scale[:, None]
    normal = y >= 2.0 ** -6
    err = np.abs(deq - xf) / scale[:, None]
    assert np.all(err[normal] <= y[normal] * 2.0 ** -4 * (1 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 * (1 + 1e-6))


def test_decode_fp8_equals_bf16_decode_on_e4m3_grid():
    """When every index vector is already an e4m3 value times a power of two and each row holds
    +-448 times that power, quantisation is exact (scale 2^p, codes reproduce the values), so FP8
    decode must equal the bf16 decode: same blocks, margins and outputs. The powers differ per row,
    so a scale applied to the wrong row or a dropped scale fails."""
    L, Bk, G, Hkv, di = 150, 16, 2, 2, 16
    B = 2
    dims = oracle.Dims(B=B, N=L, H_q=G * Hkv, H_kv=Hkv, d=16, d_idx=di, block_k=Bk, topk=3)
    g = torch.Generator().manual_seed(31)
    fin = oracle.e4m3_values(np.arange(0x7F, dtype=np.uint8))  # finite non-negative values

    def grid_rows(*shape):
        idx = torch.randint(0, 0x7F, shape, generator=g).numpy()
        sign = np.where(torch.rand(shape, generator=g).numpy() < 0.5, -1.0, 1.0)
        v = fin[idx] * sign
        v[..., 0] = 448.0 * np.where(torch.rand(shape[:-1], generator=g).numpy() < 0.5, -1.0, 1.0)
        p = torch.randint(-9, 1, shape[:-1] + (1,), generator=g).numpy()
        return torch.from_numpy(v * np.exp2(p)).to(torch.bfloat16)

    q_idx = grid_rows(B, Hkv, di)
    k_idx = grid_rows(B, L, di)
    assert torch.equal(q_idx.double().to(torch.bfloat16), q_idx)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    q, kc, vc = mk(B, G * Hkv, 16), mk(B, L, Hkv, 16), mk(B, L, Hkv, 16)
    lens = [L, 97]
    kcodes, kscale = oracle.quantize_e4m3_rows(k_idx)
    assert np.all(np.log2(kscale) == np.round(np.log2(kscale)))
    np.testing.assert_array_equal(oracle.dequantize_e4m3_rows(kcodes, kscale).numpy(), k_idx.double().numpy())
    b8, m8, o8, l8 = oracle.decode_fp8idx(dims, lens, q, q_idx, kc, vc, kcodes, kscale)
    b16, m16, o16, l16 = oracle.decode(dims, lens, q, q_idx, kc, vc, k_idx)
    np.testing.assert_array_equal(b8, b16)
    np.testing.assert_allclose(m8, m16, rtol=1e-14, atol=0)
    np.testing.assert_allclose(o8, o16, atol=1e-13)
    np.testing.assert_allclose(l8, l16, atol=1e-13)


# ----------------------------------------------------------------------------- attention backward
def test_bwd_eq11_two_position_example():
    """2.4 · 训练原生稀疏 eq (11) through the backward: weights (0.75, 0.25) from a logit gap of ln 3,
    v = (2,0), (0,2), upstream g = (1,-1) at the second query. The logit gradients 0.75 / -0.75 of
    the page appear as dk (q = e_0), dv = alpha g, and dq = scale sum dz k."""
    gld = GOLDEN["eq11_two_position"]
    dims = oracle.Dims(B=1, N=2, H_q=1, H_kv=1, d=2, d_idx=2, block_k=1, topk=1, scale=1.0)
    q = torch.tensor([[[[0.0, 0.0]], [[1.0, 0.0]]]], dtype=torch.float64)        # [1,2,1,2]
    k = torch.tensor([[[[math.log(3.0), 0.0]], [[0.0, 0.0]]]], dtype=torch.float64)
    v = torch.tensor(gld["values"], dtype=torch.float64).reshape(1, 2, 1, 2)
    dout = torch.zeros(1, 2, 1, 2, dtype=torch.float64)
    dout[0, 1, 0] = torch.tensor(gld["upstream_grad"], dtype=torch.float64)
    blocks = np.array([[[[0, -1]], [[0, 1]]]], dtype=np.int32)  # row 1: past block 0 + local block 1
    o, _ = oracle.sparse_attn(dims, q, k, v, blocks)
    np.testing.assert_allclose(o[1, 0], gld["output"], atol=1e-14)
    dq, dk, dv = oracle.sparse_attn_bwd(dims, q, k, v, blocks, dout)
    dz = np.array(gld["logit_grads"])
    np.testing.assert_allclose(dk[0, :, 0, 0], dz, atol=1e-14)      # dk_j = dz_j q, q = e_0
    np.testing.assert_allclose(dk[0, :, 0, 1], 0.0, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0, 0], 0.75 * np.array(gld["upstream_grad"]), atol=1e-14)
    np.testing.assert_allclose(dv[0, 1, 0], 0.25 * np.array(gld["upstream_grad"]), atol=1e-14)
    np.testing.assert_allclose(dq[0, 1, 0], [0.75 * math.log(3.0), 0.0], atol=1e-14)
    np.testing.assert_allclose(dq[0, 0, 0], 0.0, atol=1e-14)         # row 0 has a zero upstream gradient


def _bwd_case(N=45, Bk=8, k=2, G=2, Hkv=2, d=8, seed=41):
    dims = oracle.Dims(B=1, N=N, H_q=G * Hkv, H_kv=Hkv, d=d, d_idx=4, block_k=Bk, topk=k)
    x = small_prefill(N, G * Hkv, Hkv, d, 4, Bk, k, seed=seed, dtype=torch.float64)
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(1, N, G * Hkv, d, generator=g, dtype=torch.float64)
    return dims, x, blocks, dout


def test_bwd_matches_central_differences():
    """The backward against central differences of the oracle's forward, L = sum(dout * o), on
    sampled entries of q, k and v (selection held fixed, ragged last block)."""
    dims, x, blocks, dout = _bwd_case()
    dq, dk, dv = oracle.sparse_attn_bwd(dims, x["q"], x["k"], x["v"], blocks, dout)
    grads = {"q": dq, "k": dk, "v": dv}
    L = lambda xx: float((torch.from_numpy(oracle.sparse_attn(dims, xx["q"], xx["k"], xx["v"], blocks)[0])
                          * dout.reshape(-1, dims.H_q, dims.d)).sum())
    rng = np.random.default_rng(3)
    h = 1e-6
    for name in ("q", "k", "v"):
        t = x[name]
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in t.shape)
            xp = dict(x); xm = dict(x)
            xp[name] = t.clone(); xm[name] = t.clone()
            xp[name][idx] += h
            xm[name][idx] -= h
            fd = (L(xp) - L(xm)) / (2 * h)
            assert grads[name][idx] == pytest.approx(fd, abs=1e-7, rel=1e-6), (name, idx)


def test_bwd_sums_over_tokens():
    """Closed forms from softmax normalisation: per (sequence, group), sum_j dv_j equals the sum of
    the group's upstream gradients (the weights of each row sum to one), and sum_j dk_j = 0 (the
    logit gradients of each row sum to zero)."""
    dims, x, blocks, dout = _bwd_case(N=70, Bk=16, k=2, G=4, Hkv=2, d=8, seed=9)
    dq, dk, dv = oracle.sparse_attn_bwd(dims, x["q"], x["k"], x["v"], blocks, dout)
    G = dims.H_q // dims.H_kv
    for r in range(dims.H_kv):
        want = dout[0, :, r * G:(r + 1) * G].sum(dim=(0, 1)).numpy()
        np.testing.assert_allclose(dv[0, :, r].sum(0), want, atol=1e-12)
        np.testing.assert_allclose(dk[0, :, r].sum(0), 0.0, atol=1e-12)


def test_bwd_dense_limit_matches_autograd():
    """k >= every block: the backward is that of dense causal attention, checked against torch
    autograd of scaled_dot_product_attention in float64 (GQA heads expanded)."""
    N, Bk, G, Hkv, d = 37, 8, 2, 2, 8
    dims = oracle.Dims(B=1, N=N, H_q=G * Hkv, H_kv=Hkv, d=d, d_idx=4, block_k=Bk, topk=8)
    x = small_prefill(N, G * Hkv, Hkv, d, 4, Bk, 8, seed=5, dtype=torch.float64)
    blocks, _, _ = oracle.index_topk(dims, x["q_idx"], x["k_idx"])
    g = torch.Generator().manual_seed(6)
    dout = torch.randn(1, N, G * Hkv, d, generator=g, dtype=torch.float64)
    dq, dk, dv = oracle.sparse_attn_bwd(dims, x["q"], x["k"], x["v"], blocks, dout)
    q = x["q"].clone().requires_grad_(True)
    k = x["k"].clone().requires_grad_(True)
    v = x["v"].clone().requires_grad_(True)
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.repeat_interleave(G, dim=2).transpose(1, 2), v.repeat_interleave(G, dim=2).transpose(1, 2),
        is_causal=True)
    (o.transpose(1, 2) * dout).sum().backward()
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-12)


# ----------------------------------------------------------------------------- sequence-parallel indexer
def test_sp_eq16_hand_values():
    """4.1.1 · 监督与联合训练 eq (16) on written-out values: ranks with (a_p, z_p) = (1, 2) and (3, 1)
    give a = 3, z = 2 e^-2 + 1; a rank with no tokens (-inf, 0) changes nothing."""
    from oracle import sp
    got = sp.combine_lse([[1.0, 2.0], [3.0, 1.0], [-np.inf, 0.0]])
    assert got == pytest.approx(3.0 + math.log(1.0 + 2.0 * math.exp(-2.0)), abs=1e-15)
    # it equals the log-sum-exp of the union of the ranks' scores
    s1, s2 = np.array([1.0, 1.0]), np.array([3.0])
    assert got == pytest.approx(math.log(np.exp(s1).sum() + np.exp(s2).sum()), abs=1e-14)


@pytest.mark.parametrize("held", [[[(0, 4)], [(4, 8)]], [[(0, 3)], [(3, 6)], [(6, 8)]],
                                  [[(0, 1)], [(1, 2)], [(2, 5)], [(5, 8)]], [[(0, 8)]],
                                  [[(0, 2), (6, 8)], [(2, 4), (4, 6)]], [[(0, 1), (7, 8)], [(1, 3), (5, 7)], [(3, 5)]]],
                         ids=["halves", "thirds", "uneven", "one_rank", "zigzag_2", "zigzag_3_uneven"])
def test_sp_merge_and_lse_equal_single_device(held):
    """Each rank's local Top-k of its held blocks, merged by (score desc, id asc), plus the local
    block, is the single-device selection; eq (16) over the ranks' (a_p, z_p) is the single-device
    LSE_idx (uneven ranges, two ranges per rank, a ragged last block, ranks without candidates for
    early rows)."""
    from oracle import sp
    N, Bk, k, Hkv = 61, 8, 3, 2
    dims = oracle.Dims(B=2, N=N, H_q=2 * Hkv, H_kv=Hkv, d=8, d_idx=8, block_k=Bk, topk=k)
    x = small_prefill(N, 2 * Hkv, Hkv, 8, 8, Bk, k, seed=71, B=2)
    blocks, _, lse = oracle.index_topk(dims, x["q_idx"], x["k_idx"], want_lse=True)
    blocks = blocks.reshape(2, N, Hkv, k + 1)
    cs, ci, ml = [], [], []
    assert sp.held_blocks([r for h in held for r in h]) == list(range(8))  # the ranks' blocks tile [0, 8)
    for h in held:
        s_, i_ = sp.local_topk(dims, x["q_idx"], x["k_idx"], h)
        cs.append(s_)
        ci.append(i_)
    merged = sp.merge(dims, cs, ci)
    np.testing.assert_array_equal(merged, blocks)
    for h in held:
        ml.append(sp.local_lse(dims, x["q_idx"], x["k_idx"], blocks, h))
    np.testing.assert_allclose(sp.combine_lse(ml), lse.reshape(2, N, Hkv), atol=1e-12)


def test_bwd_dq_rows_equal_full_backward():
    """The row-subset dq of the oracle is the full backward's dq on those rows (so that sampled rows
    of full-size problems can be checked)."""
    dims, x, blocks, dout = _bwd_case(N=50, Bk=8, k=2, G=2, Hkv=2, d=8, seed=13)
    dq, _, _ = oracle.sparse_attn_bwd(dims, x["q"], x["k"], x["v"], blocks, dout)
    rows = [0, 7, 8, 31, 49]
    sub = oracle.sparse_attn_bwd_dq_rows(dims, x["q"], x["k"], x["v"], blocks, dout, rows)
    np.testing.assert_allclose(sub, dq[0, rows], atol=1e-14)
