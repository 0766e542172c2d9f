"""Sequence-parallel index branch on one GPU, ranks emulated: the key ranges of P ranks are run one
after the other through msa_index_topk_local / msa_lse_idx_local on their own K_idx slices, the
candidates stacked in rank order as the all-gather would, then merged. The result must be the
single-device msa_index_topk selection (bit-exact) and LSE_idx, and the oracle's."""
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


@pytest.mark.parametrize("case", CASES)
def test_sp_emulated_ranks_match_single_device(case):
    N, H_q, H_kv, d, d_idx, bk, k, B, P = case
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=900 + N + P, B=B)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    qi, ki = x["q_idx"].to(DEV), x["k_idx"].to(DEV)
    ref_blocks, ref_lse = msa.msa_index_topk(dm, qi, ki, want_lse=True)
    cs, ci, ranges = [], [], []
    for p in range(P):
        tok0, ntok = sp.split_range(N, bk, P, p)
        ranges.append((tok0, ntok))
        s_, i_ = msa.msa_index_topk_local(dm, qi, ki[:, tok0:tok0 + ntok].contiguous(), tok0)
        cs.append(s_)
        ci.append(i_)
    blocks = msa.msa_topk_merge(dm, torch.stack(cs), torch.stack(ci))
    ml = torch.stack([msa.msa_lse_idx_local(dm, qi, ki[:, t0:t0 + n].contiguous(), t0, blocks) for t0, n in ranges])
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
    t0, n = ranges[-1]
    os_, oi_ = osp.local_topk(od, x["q_idx"], x["k_idx"], t0 // bk, -(-(t0 + n) // bk))
    gi = ci[-1].cpu().numpy()
    rows_ok = np.all(gi == oi_, axis=-1) | (om.reshape(B, N, H_kv) < 1e-4)
    assert rows_ok.all()
    fin = gi >= 0
    scale_idx = 1.0 / np.sqrt(d_idx)
    np.testing.assert_allclose(cs[-1].cpu().numpy()[fin & (gi == oi_)] * scale_idx, os_[fin & (gi == oi_)], atol=1e-4)
