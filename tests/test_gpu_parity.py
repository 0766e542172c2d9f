"""GPU (libmsa, through the C ABI) vs the float64 oracle on seeded inputs: selection, LSE_idx,
sparse attention, KL alignment and decode, at sizes spanning several tiles and a ragged tail."""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from msa_inputs import small_prefill
from parity import compare_blocks, check_attention, check_attention_bf16, check_grad, KL_REL, NEAR_TIE

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (N, H_q, H_kv, d, d_idx, block_k, topk, B)
SHAPES = {
    "tiny_cfg": (512, 4, 2, 64, 32, 32, 4, 1),
    "main_ragged": (1000, 64, 4, 128, 64, 128, 16, 1),
    "main_two_seqs": (777, 64, 4, 128, 64, 128, 4, 2),
    "main_one_token": (1, 64, 4, 128, 64, 128, 16, 1),
    "main_short": (130, 64, 4, 128, 64, 128, 16, 1),
    "small_bk64": (300, 16, 2, 128, 64, 64, 3, 1),
    "small_d64_bk128": (390, 8, 4, 64, 32, 128, 2, 1),
}


def mk(name, seed=0):
    N, H_q, H_kv, d, d_idx, bk, k, B = SHAPES[name]
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=1234 + seed + N, B=B)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, k)
    return dm, od, x


def to_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def sample_rows(B, N, n, seed=0):
    rng = np.random.default_rng(seed)
    rows = set([0, N - 1, B * N - 1] + [b * N + min(N - 1, 127) for b in range(B)])
    rows |= set(rng.choice(B * N, size=min(n, B * N), replace=False).tolist())
    return sorted(r for r in rows if r < B * N)


@pytest.mark.parametrize("name", list(SHAPES))
def test_index_topk_matches_oracle(name):
    dm, od, x = mk(name)
    g = to_dev(x)
    blocks, lse_idx = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"], want_lse=True)
    torch.cuda.synchronize()
    ob, om, ol = oracle.index_topk(od, x["q_idx"], x["k_idx"], want_lse=True)
    bad, near = compare_blocks(blocks.cpu().numpy(), ob, om)
    assert bad == 0, f"{bad} selection rows differ (near-ties excluded: {near})"
    # LSE_idx over the selected set, on rows whose selection matches
    same = np.all(blocks.cpu().numpy().reshape(ob.shape) == ob, axis=-1)
    err = np.abs(lse_idx.cpu().numpy().reshape(ol.shape) - ol)[same]
    assert err.max() <= 1e-3, f"LSE_idx max abs error {err.max():.3e}"


def test_index_topk_matches_oracle_on_a_grid_of_two_ctas_per_sm():
    """Ten sequences of 1000 tokens: 320 row tiles, enough for the launch that puts two index CTAs on
    every SM (the smaller cases above run one per SM)."""
    B, N, H_q, H_kv, d, d_idx, bk, k = 10, 1000, 64, 4, 128, 64, 128, 16
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=4242, B=B)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, k)
    g = to_dev(x)
    blocks, lse_idx = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"], want_lse=True)
    torch.cuda.synchronize()
    ob, om, ol = oracle.index_topk(od, x["q_idx"], x["k_idx"], want_lse=True)
    bad, near = compare_blocks(blocks.cpu().numpy(), ob, om)
    assert bad == 0, f"{bad} selection rows differ (near-ties excluded: {near})"
    same = np.all(blocks.cpu().numpy().reshape(ob.shape) == ob, axis=-1)
    assert np.abs(lse_idx.cpu().numpy().reshape(ol.shape) - ol)[same].max() <= 1e-3


@pytest.mark.parametrize("name", list(SHAPES))
def test_sparse_attention_matches_oracle(name):
    dm, od, x = mk(name, seed=1)
    ob, _, _ = oracle.index_topk(od, x["q_idx"], x["k_idx"])
    ob = ob.reshape(dm.B, dm.N, dm.H_kv, dm.topk + 1)
    g = to_dev(x)
    out, lse = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], torch.from_numpy(ob).to(DEV))
    torch.cuda.synchronize()
    rows = sample_rows(dm.B, dm.N, 160)
    oo, ol = oracle.sparse_attn(od, x["q"], x["k"], x["v"], ob, rows=rows)
    og = out.float().cpu().reshape(dm.B * dm.N, dm.H_q, dm.d).numpy()[rows]
    lg = lse.cpu().reshape(dm.B * dm.N, dm.H_q).numpy()[rows]
    check_attention(og, oo, lg, ol)


@pytest.mark.parametrize("name", ["tiny_cfg", "main_ragged", "main_two_seqs", "small_bk64"])
def test_sparse_attention_bf16_output_is_the_rounded_fp32_output(name):
    """msa_sparse_attn_fwd_bf16 writes the fp32 entry point's values rounded to nearest-even bf16,
    bit for bit, and stays within the fp32 bound plus half a bf16 unit of the oracle."""
    dm, od, x = mk(name, seed=2)
    ob, _, _ = oracle.index_topk(od, x["q_idx"], x["k_idx"])
    ob = ob.reshape(dm.B, dm.N, dm.H_kv, dm.topk + 1)
    g = to_dev(x)
    blocks = torch.from_numpy(ob).to(DEV)
    o32, l32 = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], blocks)
    o16, l16 = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], blocks, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(l16, l32)
    rows = sample_rows(dm.B, dm.N, 120, seed=5)
    oo, _ = oracle.sparse_attn(od, x["q"], x["k"], x["v"], ob, rows=rows)
    check_attention_bf16(o16.float().cpu().reshape(dm.B * dm.N, dm.H_q, dm.d).numpy()[rows], oo)


def test_dense_limit_k_covers_all_blocks():
    """k >= number of blocks: every causal block is selected and the output is dense causal attention."""
    N, H_q, H_kv, d, d_idx, bk, k = 256, 4, 2, 64, 32, 32, 16
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=77)
    dm = msa.MsaDims(1, N, H_q, H_kv, d, d_idx, bk, k)
    g = to_dev(x)
    blocks = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"])
    out, lse = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], blocks)
    b = blocks.cpu().numpy()[0]
    for i in range(N):
        assert [c for c in b[i, 0] if c >= 0] == list(range(i // bk + 1))
    q = x["q"].double().transpose(1, 2)
    kk = x["k"].double().repeat_interleave(2, dim=2).transpose(1, 2)
    vv = x["v"].double().repeat_interleave(2, dim=2).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True).transpose(1, 2)[0]
    check_attention(out.float().cpu()[0].numpy(), ref.numpy())


@pytest.mark.parametrize("name,gs", [("tiny_cfg", 1.0), ("main_short", 1.0), ("main_ragged", 0.5),
                                     ("main_two_seqs", 1.0)])
def test_kl_matches_oracle(name, gs):
    """KL loss and index gradients on the oracle's selection (LSE_idx computed inside the call),
    and the full GPU pipeline (GPU selection and GPU LSE_idx) where it selects the same blocks."""
    dm, od, x = mk(name, seed=2)
    g = to_dev(x)
    ob, om, _ = oracle.index_topk(od, x["q_idx"], x["k_idx"])
    ob = ob.reshape(dm.B, dm.N, dm.H_kv, dm.topk + 1)
    ol, okr, odq, odk = oracle.kl(od, x["q"], x["k"], x["q_idx"], x["k_idx"], ob, grad_scale=gs)
    bo = torch.from_numpy(ob).to(DEV)
    _, lse = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], bo)
    loss, dq, dk = msa.msa_kl_fwd_grad(dm, g["q"], g["k"], g["q_idx"], g["k_idx"], bo, lse, None, grad_scale=gs)
    torch.cuda.synchronize()
    assert abs(loss.item() - ol) <= KL_REL * abs(ol), f"loss {loss.item()} vs {ol}"
    check_grad(dq.cpu().numpy().reshape(odq.shape), odq, "dq_idx")
    check_grad(dk.cpu().numpy(), odk, "dk_idx")
    # full pipeline: GPU selection + GPU LSE_idx from the index pass
    blocks, lse_idx = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"], want_lse=True)
    if torch.equal(blocks.cpu(), torch.from_numpy(ob)):
        _, lse2 = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], blocks)
        loss2, dq2, dk2 = msa.msa_kl_fwd_grad(dm, g["q"], g["k"], g["q_idx"], g["k_idx"], blocks, lse2, lse_idx,
                                              grad_scale=gs)
        assert abs(loss2.item() - ol) <= KL_REL * abs(ol)
        check_grad(dq2.cpu().numpy().reshape(odq.shape), odq, "dq_idx (pipeline)")
    else:
        bad, near = compare_blocks(blocks.cpu().numpy(), ob, om)
        assert bad == 0


@pytest.mark.parametrize("shape", [(3, 1000, 64, 4, 128, 64, 128, 16), (2, 700, 4, 2, 64, 32, 32, 4)])
def test_decode_matches_oracle(shape):
    B, L, H_q, H_kv, d, d_idx, bk, k = shape
    gen = torch.Generator().manual_seed(99 + L)
    mkr = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    kc, vc, kic = mkr(B, L, H_kv, d), mkr(B, L, H_kv, d), mkr(B, L, d_idx)
    q, qi = mkr(B, H_q, d), mkr(B, H_kv, d_idx)
    lens = torch.tensor([L, L // 2 + 17, 130][:B], dtype=torch.int32)
    dm = msa.MsaDims(B, L, H_q, H_kv, d, d_idx, bk, k)
    od = oracle.Dims(B, L, H_q, H_kv, d, d_idx, bk, k)
    out, blocks, margin = msa.msa_sparse_attn_decode(dm, lens.to(DEV), q.to(DEV), qi.to(DEV), kc.to(DEV),
                                                     vc.to(DEV), kic.to(DEV), want_margin=True)
    torch.cuda.synchronize()
    ob, om, oo, olse = oracle.decode(od, lens, q, qi, kc, vc, kic)
    bad, near = compare_blocks(blocks.cpu().numpy(), ob, om)
    assert bad == 0
    gm = margin.cpu().numpy()
    assert np.array_equal(np.isinf(gm), np.isinf(om))
    assert np.abs(gm[np.isfinite(om)] - om[np.isfinite(om)]).max(initial=0.0) <= NEAR_TIE
    same = np.all(blocks.cpu().numpy() == ob, axis=-1)  # [B, H_kv]
    G = H_q // H_kv
    og = out.float().cpu().numpy()
    for b in range(B):
        for r in range(H_kv):
            if same[b, r]:
                check_attention(og[b, r * G:(r + 1) * G], oo[b, r * G:(r + 1) * G])


def test_results_are_deterministic():
    dm, od, x = mk("main_ragged", seed=3)
    g = to_dev(x)
    b1 = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"])
    o1, l1 = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], b1)
    b2 = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"])
    o2, l2 = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], b2)
    assert torch.equal(b1, b2) and torch.equal(o1, o2) and torch.equal(l1, l2)


def test_kl_loss_and_dq_idx_are_deterministic():
    """The loss and dQ_idx are reduced in a fixed order (per-slot partials, then rows): two calls on
    the same inputs give bit-identical values. dK_idx accumulates with atomics and is compared with
    a tolerance only."""
    dm, od, x = mk("main_two_seqs", seed=5)
    g = to_dev(x)
    blocks, lse_idx = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"], want_lse=True)
    _, lse = msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], blocks)
    r1 = msa.msa_kl_fwd_grad(dm, g["q"], g["k"], g["q_idx"], g["k_idx"], blocks, lse, lse_idx)
    r2 = msa.msa_kl_fwd_grad(dm, g["q"], g["k"], g["q_idx"], g["k_idx"], blocks, lse, lse_idx)
    torch.cuda.synchronize()
    assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])
    assert torch.allclose(r1[2], r2[2], rtol=0, atol=1e-9)


def test_invalid_block_ids_raise_device_check_not_a_fault():
    """An out-of-range or repeated block id in `blocks` is skipped by the kernels and reported
    through the status word (no out-of-bounds access, no trap)."""
    dm, od, x = mk("tiny_cfg", seed=4)
    g = to_dev(x)
    blocks = msa.msa_index_topk(dm, g["q_idx"], g["k_idx"])
    ws = msa.workspace(msa.MSA_OP_ATTN_FWD, dm, DEV)
    msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], blocks, ws=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    bad = blocks.clone()
    bad[0, 5, 0, 0] = 3  # row 5 lives in block 0: block 3 is in its future
    bad[0, 300, 1, 1] = bad[0, 300, 1, 0]  # repeated id
    msa.msa_sparse_attn_fwd(dm, g["q"], g["k"], g["v"], bad, ws=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_DEVICE_CHECK
