"""Backward of the sparse attention on the GPU, through the C ABI, against the float64 oracle
(selection held fixed: the oracle's selection is fed to both the GPU forward and backward)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from msa_inputs import small_prefill
from parity import check_bwd

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (N, H_q, H_kv, d, d_idx, block_k, topk, B)
SHAPES = {
    "main_ragged": (1000, 64, 4, 128, 64, 128, 16, 1),
    "main_two_seqs": (777, 64, 4, 128, 64, 128, 4, 2),
    "main_short": (130, 64, 4, 128, 64, 128, 16, 1),
    "main_one_token": (1, 64, 4, 128, 64, 128, 16, 1),
    "g8_d64_bk64": (300, 16, 2, 64, 32, 64, 3, 1),
    "g32_d64_bk32": (200, 32, 1, 64, 32, 32, 4, 1),
    "g8_d128_bk32": (260, 8, 1, 128, 64, 32, 5, 1),
}


def run_case(name, seed=0):
    N, H_q, H_kv, d, d_idx, bk, k, B = SHAPES[name]
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=4321 + seed + N, B=B)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, k)
    ob, _, _ = oracle.index_topk(od, x["q_idx"], x["k_idx"])
    blocks = torch.from_numpy(np.ascontiguousarray(ob)).reshape(B, N, H_kv, k + 1)
    g = torch.Generator().manual_seed(77 + seed)
    dout = torch.randn(B, N, H_q, d, generator=g).to(torch.bfloat16)
    gd = {kk: vv.to(DEV) for kk, vv in x.items()}
    bl = blocks.to(DEV)
    out, lse = msa.msa_sparse_attn_fwd(dm, gd["q"], gd["k"], gd["v"], bl)
    ws = msa.workspace(msa.MSA_OP_ATTN_BWD, dm, DEV)
    dq, dk, dv = msa.msa_sparse_attn_bwd(dm, gd["q"], gd["k"], gd["v"], bl, out, lse, dout.to(DEV), ws=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    rq, rk, rv = oracle.sparse_attn_bwd(od, x["q"], x["k"], x["v"], blocks, dout)
    return (dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()), (rq, rk, rv), dout, blocks


@pytest.mark.parametrize("name", list(SHAPES))
def test_bwd_matches_oracle(name):
    (dq, dk, dv), (rq, rk, rv), _, _ = run_case(name)
    check_bwd(dq, rq, "dq")
    check_bwd(dk, rk, "dk")
    check_bwd(dv, rv, "dv")


def test_bwd_sums_over_tokens():
    """Closed forms that hold at any size: per (sequence, group), sum_j dv_j is the sum of the
    group's upstream gradients and sum_j dk_j = 0."""
    (dq, dk, dv), _, dout, _ = run_case("main_ragged", seed=1)
    N, H_q, H_kv, d, _, _, _, B = SHAPES["main_ragged"]
    G = H_q // H_kv
    do = dout.double().numpy()
    for b in range(B):
        for r in range(H_kv):
            want = do[b, :, r * G:(r + 1) * G].sum(axis=(0, 1))
            got = dv[b, :, r].astype(np.float64).sum(0)
            assert np.abs(got - want).max() <= 1e-3 * max(np.abs(want).max(), 1.0)
            ks = dk[b, :, r].astype(np.float64)
            assert np.abs(ks.sum(0)).max() <= 1e-3 * np.abs(ks).sum(0).max()
