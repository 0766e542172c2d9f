"""Full-size workloads in the launch configuration the benchmark times (same entry points, same
workspaces, whole grids), checked against the float64 oracle on sampled rows and, where a value is
a reduction over the whole layer, through properties that hold at any size.

Workloads: the 8K and 32K (needle) prefills, the 64K training step (index Top-k with LSE_idx,
attention, KL alignment) and one decode step of 16 sequences over 256K-token caches."""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from msa_inputs import WORKLOADS, prefill_inputs, decode_inputs
from parity import compare_blocks, check_attention, check_grad, check_bwd

pytestmark = pytest.mark.gpu

DEV = "cuda"


def sampled_rows(N, n=40, seed=0, carry=None, n_carry=12):
    """First and last rows, rows at block edges, and uniformly drawn rows. With `carry` (the needle
    workload's mask of query rows that carry the needle direction), n_carry of those rows and as
    many of the others are added: the carrying rows select the hot needle blocks, block 0 among
    them, so the sample always reaches the hot-block path."""
    rng = np.random.default_rng(seed)
    rows = {0, 1, 127, 128, 129, N // 2, N - 2, N - 1}
    rows |= set(rng.choice(N, size=n, replace=False).tolist())
    if carry is not None:
        c = np.asarray(carry).reshape(-1)[:N]
        for pool in (np.flatnonzero(c), np.flatnonzero(~c)):
            pool = pool[pool >= 128 * 16]  # rows with more complete past blocks than topk
            rows |= set(rng.choice(pool, size=min(n_carry, len(pool)), replace=False).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N), dtype=np.int64)


def run_prefill(w, want_lse_idx=False):
    x = prefill_inputs(w, device=DEV)
    dm = msa.MsaDims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    ws_i = msa.workspace(msa.MSA_OP_INDEX_TOPK_LSE if want_lse_idx else msa.MSA_OP_INDEX_TOPK, dm, DEV)
    ws_a = msa.workspace(msa.MSA_OP_ATTN_FWD, dm, DEV)
    if want_lse_idx:
        blocks, lse_idx = msa.msa_index_topk(dm, x["q_idx"], x["k_idx"], want_lse=True, ws=ws_i)
    else:
        blocks, lse_idx = msa.msa_index_topk(dm, x["q_idx"], x["k_idx"], ws=ws_i), None
    out, lse = msa.msa_sparse_attn_fwd(dm, x["q"], x["k"], x["v"], blocks, ws=ws_a)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(ws_a) == msa.MSA_OK
    return dm, x, blocks, lse_idx, out, lse


def oracle_selection(w, rows, ob):
    """A full selection array holding the oracle's rows at `rows` (-1 elsewhere, never read)."""
    full = np.full((w.B * w.N, w.H_kv, w.topk + 1), -1, dtype=np.int32)
    full[rows] = ob
    return full.reshape(w.B, w.N, w.H_kv, w.topk + 1)


def check_sampled_prefill(w, x, blocks, out, lse, rows):
    od = oracle.Dims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    xc = {k: v.cpu() for k, v in x.items()}
    ob, om, _ = oracle.index_topk(od, xc["q_idx"], xc["k_idx"], rows=rows)
    gb = blocks.cpu().numpy().reshape(w.B * w.N, w.H_kv, w.topk + 1)
    bad, near = compare_blocks(gb[rows], ob, om)
    assert bad == 0, f"{bad} sampled selection rows differ (near-ties excluded: {near})"
    # attention on the oracle's own selection; compared where the GPU selected exactly the same
    # blocks (every (query, group) row of the sample, unless a near-tie went the other way)
    full = oracle_selection(w, rows, ob)
    same = np.all(gb[rows] == ob, axis=(1, 2))
    assert same.sum() >= len(rows) - near
    oo, ol = oracle.sparse_attn(od, xc["q"], xc["k"], xc["v"], full, rows=rows)
    og = out.cpu().numpy().reshape(w.B * w.N, w.H_q, w.d)[rows]
    lg = lse.cpu().numpy().reshape(w.B * w.N, w.H_q)[rows]
    check_attention(og[same], oo[same], lg[same], ol[same])
    return xc, od, full, same


@pytest.mark.parametrize("wname", ["prefill_8k", "prefill_32k_needles"])
def test_full_prefill_sampled_rows_match_oracle(wname):
    w = WORKLOADS[wname]
    dm, x, blocks, _, out, lse = run_prefill(w)
    carry = x["needle_rows"].cpu().numpy() if w.needles else None
    rows = sampled_rows(w.N, n=200, seed=w.cid, carry=carry, n_carry=40)
    if w.needles:
        # the sample reaches the hot blocks: some sampled rows select block 0 and other needle blocks
        gb = blocks.cpu().numpy().reshape(w.B * w.N, w.H_kv, w.topk + 1)[rows]
        needles = set(x["needle_blocks"].cpu().tolist())
        assert (gb == 0).any(axis=(1, 2)).sum() >= 8
        assert np.isin(gb, list(needles - {0})).any(axis=(1, 2)).sum() >= 8
    check_sampled_prefill(w, x, blocks, out, lse, rows)
    # the bf16 entry point (the benchmark's call) on the same selection: every output element is
    # the fp32 result rounded to nearest-even bf16, and the LSE is the same
    ws_a = msa.workspace(msa.MSA_OP_ATTN_FWD, dm, DEV)
    o16, l16 = msa.msa_sparse_attn_fwd(dm, x["q"], x["k"], x["v"], blocks, ws=ws_a, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(ws_a) == msa.MSA_OK
    assert torch.equal(o16, out.to(torch.bfloat16))
    assert torch.equal(l16, lse)


def test_full_training_step_sampled_rows_and_invariants():
    w = WORKLOADS["train_64k"]
    dm, x, blocks, lse_idx, out, lse = run_prefill(w, want_lse_idx=True)
    rows = sampled_rows(w.N, n=24, seed=w.cid)
    xc, od, full, same = check_sampled_prefill(w, x, blocks, out, lse, rows)
    gs = 1.0 / (w.N * w.H_kv)
    ws_k = msa.workspace(msa.MSA_OP_KL, dm, DEV)
    loss, dq, dk = msa.msa_kl_fwd_grad(dm, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, lse, lse_idx,
                                       grad_scale=gs, ws=ws_k)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(ws_k) == msa.MSA_OK
    # a KL divergence is never negative
    assert float(loss.item()) >= 0.0
    # dq_idx of the sampled rows against the oracle's gradient for those rows (oracle selection,
    # rows where the GPU selected the same blocks)
    _, _, odq, _ = oracle.kl(od, xc["q"], xc["k"], xc["q_idx"], xc["k_idx"], full, grad_scale=gs, rows=rows)
    gdq = dq.cpu().numpy().reshape(w.B * w.N, w.H_kv, w.d_idx)[rows]
    check_grad(gdq[same], odq[same], "dq_idx")
    # P and P_idx both sum to one over each row's token set, so the rows' contributions to dK_idx
    # cancel when summed over the tokens: sum_j dK_idx[b, j, :] = 0 up to rounding
    tot = dk.double().sum(dim=1).abs().max().item()
    scale = dk.double().abs().sum(dim=1).max().item()
    assert tot <= 1e-3 * max(scale, 1e-30), f"sum over tokens of dK_idx is {tot:.3e} (|dK_idx| sum {scale:.3e})"
    del dq, dk, ws_k
    # main-branch backward in the benchmark's configuration: dq of the sampled rows against the
    # oracle (its own selection, rows where the GPU chose the same blocks), and the sums over tokens
    # that hold at any size (sum_j dv_j = the group's upstream gradients, sum_j dk_j = 0)
    gen = torch.Generator().manual_seed(4242)
    dout = torch.randn(w.B, w.N, w.H_q, w.d, generator=gen).to(torch.bfloat16)
    ws_b = msa.workspace(msa.MSA_OP_ATTN_BWD, dm, DEV)
    gq, gk, gv = msa.msa_sparse_attn_bwd(dm, x["q"], x["k"], x["v"], blocks, out, lse, dout.to(DEV), ws=ws_b)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(ws_b) == msa.MSA_OK
    odq = oracle.sparse_attn_bwd_dq_rows(od, xc["q"], xc["k"], xc["v"], full, dout, rows)
    gqr = gq.cpu().numpy().reshape(w.B * w.N, w.H_q, w.d)[rows]
    check_bwd(gqr[same], odq[same], "dq (sampled rows)")
    G = w.H_q // w.H_kv
    for r in range(w.H_kv):
        want = dout[0, :, r * G:(r + 1) * G].double().sum(dim=(0, 1))
        got = gv[0, :, r].double().sum(0).cpu()
        assert (got - want).abs().max().item() <= 1e-3 * max(want.abs().max().item(), 1.0)
        ks = gk[0, :, r].double()
        assert ks.sum(0).abs().max().item() <= 1e-3 * ks.abs().sum(0).max().item()


def test_full_decode_sampled_sequences_match_oracle():
    w = WORKLOADS["decode_16x256k"]
    x = decode_inputs(w, device=DEV)
    dm = msa.MsaDims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    ws = msa.workspace(msa.MSA_OP_DECODE, dm, DEV)
    out, blocks = msa.msa_sparse_attn_decode(dm, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                             x["k_idx_cache"], ws=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    G = w.H_q // w.H_kv
    od = oracle.Dims(1, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    for b in (0, 5, 10, w.B - 1):
        sl = slice(b, b + 1)
        ob, om, oo, olse = oracle.decode(od, x["cache_len"][sl].cpu(), x["q"][sl].cpu(), x["q_idx"][sl].cpu(),
                                         x["k_cache"][sl].cpu(), x["v_cache"][sl].cpu(), x["k_idx_cache"][sl].cpu())
        gb = blocks[sl].cpu().numpy()
        bad, near = compare_blocks(gb, ob, om)
        assert bad == 0, f"sequence {b}: selection differs (near-ties excluded: {near})"
        same = np.all(gb == ob, axis=-1)[0]
        og = out[sl].cpu().numpy()[0]
        for r in range(w.H_kv):
            if same[r]:
                check_attention(og[r * G:(r + 1) * G], oo[0, r * G:(r + 1) * G])


def test_full_decode_fp8idx_sampled_sequences_match_oracle():
    """The FP8-scored decode step over the full 16 x 256K caches: the GPU quantiser's codes and
    scales bit-exact for the sampled sequences' whole caches, selection, margins and attention
    against the oracle, and every planted block selected by every group in both scorings."""
    w = WORKLOADS["decode_16x256k"]
    x = decode_inputs(w, device=DEV)
    dm = msa.MsaDims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    ws = msa.workspace(msa.MSA_OP_DECODE, dm, DEV)
    kcodes, kscale = msa.msa_quantize_e4m3_rows(x["k_idx_cache"])
    out, blocks, margin = msa.msa_sparse_attn_decode_fp8idx(dm, x["cache_len"], x["q"], x["q_idx"], x["k_cache"],
                                                            x["v_cache"], kcodes, kscale, ws=ws, want_margin=True)
    _, b16 = msa.msa_sparse_attn_decode(dm, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                        x["k_idx_cache"], ws=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    planted = x["planted_blocks"].cpu().numpy()
    for sel in (blocks.cpu().numpy(), b16.cpu().numpy()):
        for b in range(w.B):
            for r in range(w.H_kv):
                assert set(planted[b].tolist()) <= set(sel[b, r].tolist()), f"sequence {b} group {r}"
    G = w.H_q // w.H_kv
    od = oracle.Dims(1, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    for b in (0, w.B - 1):
        sl = slice(b, b + 1)
        kic = x["k_idx_cache"][sl].cpu()
        okc, oks = oracle.quantize_e4m3_rows(kic)
        gc = kcodes[sl].cpu().numpy()
        gc[gc == 0x80] = 0
        okc0 = okc.copy()
        okc0[okc0 == 0x80] = 0
        np.testing.assert_array_equal(gc, okc0)
        np.testing.assert_array_equal(kscale[sl].cpu().numpy(), oks)
        ob, om, oo, _ = oracle.decode_fp8idx(od, x["cache_len"][sl].cpu(), x["q"][sl].cpu(), x["q_idx"][sl].cpu(),
                                             x["k_cache"][sl].cpu(), x["v_cache"][sl].cpu(), okc, oks)
        gb = blocks[sl].cpu().numpy()
        bad, near = compare_blocks(gb, ob, om)
        assert bad == 0, f"sequence {b}: selection differs (near-ties excluded: {near})"
        gm = margin[sl].cpu().numpy()
        assert np.array_equal(np.isinf(gm), np.isinf(om))
        fin = np.isfinite(om)
        assert np.abs(gm[fin] - om[fin]).max(initial=0.0) <= 1e-4
        same = np.all(gb == ob, axis=-1)[0]
        og = out[sl].cpu().numpy()[0]
        for r in range(w.H_kv):
            if same[r]:
                check_attention(og[r * G:(r + 1) * G], oo[0, r * G:(r + 1) * G])
