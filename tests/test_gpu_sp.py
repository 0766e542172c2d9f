"""Sequence-parallel index branch on one GPU, ranks emulated: the key ranges of P ranks (contiguous,
or zig-zag with two ranges per rank) are run one after the other through msa_index_topk_local /
msa_lse_idx_local on their own K_idx, the candidates stacked in rank order as the all-gather would,
then merged. The result must be the single-device msa_index_topk selection (bit-exact) and LSE_idx,
and the oracle's."""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
from block_sparse_attention_idx_b200 import sp
import oracle
from oracle import sp as osp
from msa_inputs import small_prefill
from parity import compare_blocks

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (N, H_q, H_kv, d, d_idx, block_k, topk, B, P)
CASES = [(1000, 64, 4, 128, 64, 128, 16, 1, 2), (1000, 64, 4, 128, 64, 128, 16, 1, 3),
         (777, 64, 4, 128, 64, 128, 4, 2, 4), (300, 16, 2, 128, 64, 64, 3, 1, 3), (260, 8, 4, 64, 32, 32, 5, 1, 8)]


@pytest.mark.parametrize("assign", ["zigzag", "contiguous"])
@pytest.mark.parametrize("case", CASES)
def test_sp_emulated_ranks_match_single_device(case, assign):
    N, H_q, H_kv, d, d_idx, bk, k, B, P = case
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=900 + N + P, B=B)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    qi, ki = x["q_idx"].to(DEV), x["k_idx"].to(DEV)
    ref_blocks, ref_lse = msa.msa_index_topk(dm, qi, ki, want_lse=True)
    ranges_of = sp.zigzag_ranges if assign == "zigzag" else sp.contiguous_ranges
    cs, ci, helds = [], [], []
    for p in range(P):
        held = ranges_of(N, bk, P, p)
        helds.append(held)
        s_, i_ = (msa.msa_index_topk_local(dm, qi, sp.local_keys(ki, held), held) if held
                  else sp.no_candidates(dm, qi.device))
        cs.append(s_)
        ci.append(i_)
    blocks = msa.msa_topk_merge(dm, torch.stack(cs), torch.stack(ci))
    ml = torch.stack([msa.msa_lse_idx_local(dm, qi, sp.local_keys(ki, h), h, blocks) if h
                      else sp.no_lse_pairs(dm, qi.device) for h in helds])
    lse = msa.msa_lse_combine(dm, ml)
    torch.cuda.synchronize()
    # identical to the single-device selection, ties included
    assert torch.equal(blocks, ref_blocks)
    # LSE_idx: the same quantity, summed in another order
    assert torch.allclose(lse, ref_lse, rtol=0, atol=2e-5 * max(1.0, float(ref_lse.abs().max())))
    # and the oracle: selection except near-ties, LSE_idx, and the candidates of one rank
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, k)
    ob, om, ol = oracle.index_topk(od, x["q_idx"], x["k_idx"], want_lse=True)
    bad, near = compare_blocks(blocks.cpu().numpy(), ob, om)
    assert bad == 0
    same = np.all(blocks.cpu().numpy().reshape(ob.shape) == ob, axis=-1)
    assert np.abs(lse.cpu().numpy().reshape(ol.shape) - ol)[same].max() <= 1e-3
    # one rank's candidates against the oracle's local Top-k of the same held blocks
    # (rows whose local list has a near-tie among its first k+1 scores may order those differently)
    pr = max(range(P), key=lambda p: len(helds[p]))
    hb = [(t0 // bk, -(-(t0 + n) // bk)) for t0, n in helds[pr]]
    os1, oi1 = osp.local_topk(oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, k + 1), x["q_idx"], x["k_idx"], hb)
    os_, oi_ = os1[..., :k], oi1[..., :k]
    with np.errstate(invalid="ignore"):
        gaps = np.abs(np.diff(os1, axis=-1))
    local_near = np.any(gaps < 1e-4, axis=-1)
    gi = ci[pr].cpu().numpy()
    rows_ok = np.all(gi == oi_, axis=-1) | local_near
    assert rows_ok.all()
    fin = gi >= 0
    scale_idx = 1.0 / np.sqrt(d_idx)
    np.testing.assert_allclose(cs[pr].cpu().numpy()[fin & (gi == oi_)] * scale_idx, os_[fin & (gi == oi_)], atol=1e-4)
