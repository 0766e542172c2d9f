"""The training workload's KL alignment at full size (N = 65536, 64 query / 4 KV heads) against the
float64 oracle over EVERY row: the loss L_KL, dQ_idx of every (query, group) row and dK_idx of every
token ("MSA 中的 KL 对齐与局部知识蒸馏", section 3: the loss and its gradient P_idx - P).

The selection of all 262144 (query, group) rows is compared first (bit-exact except near-ties).
Both sides then run the KL on the oracle's selection, so every oracle input is independent of the
CUDA path: the library computes the main LSE (msa_sparse_attn_fwd), LSE_idx and the KL terms on
that selection exactly as the training step does. The oracle takes a few minutes on the host's
cores (it is the plain float64 definition)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from msa_inputs import WORKLOADS, prefill_inputs
from parity import GRAD_MAX, GRAD_REL, KL_REL, compare_blocks, report

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_train_64k_kl_loss_and_gradients_all_rows_match_oracle():
    w = WORKLOADS["train_64k"]
    x = prefill_inputs(w, device=DEV)
    dm = msa.MsaDims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    od = oracle.Dims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    xc = {k: v.cpu() for k, v in x.items()}
    # gradients of sum_{i,r} KL (the loss times N*H_kv): per-row gradients of order one, so the
    # absolute bound is a real check, not one the 1/(N*H_kv) factor meets by itself
    gs = float(w.N * w.H_kv)

    # selection of every row, GPU against the oracle
    ws_i = msa.workspace(msa.MSA_OP_INDEX_TOPK, dm, DEV)
    gb = msa.msa_index_topk(dm, x["q_idx"], x["k_idx"], ws=ws_i).cpu().numpy()
    ob, om, _ = oracle.index_topk(od, xc["q_idx"], xc["k_idx"])
    bad, near = compare_blocks(gb.reshape(ob.shape), ob, om)
    report(f"train_64k selection: {bad} rows differ outside near-ties, {near} near-tied of {om.size}")
    assert bad == 0

    # the training step's KL path on the oracle's selection
    blocks = torch.from_numpy(ob.reshape(gb.shape)).to(DEV)
    ws_a = msa.workspace(msa.MSA_OP_ATTN_FWD, dm, DEV)
    out, lse = msa.msa_sparse_attn_fwd(dm, x["q"], x["k"], x["v"], blocks, ws=ws_a)
    del out, ws_a
    ws_k = msa.workspace(msa.MSA_OP_KL, dm, DEV)
    loss, dq, dk = msa.msa_kl_fwd_grad(dm, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, lse, None,
                                       grad_scale=gs, ws=ws_k)
    assert msa.msa_get_device_status(ws_k) == msa.MSA_OK
    g_loss = float(loss.item())
    g_dq = dq.cpu().numpy().reshape(w.B * w.N, w.H_kv, w.d_idx).astype(np.float64)
    g_dk = dk.cpu().numpy().reshape(w.B, w.N, w.d_idx).astype(np.float64)
    del x, blocks, lse, loss, dq, dk, ws_k, ws_i
    torch.cuda.empty_cache()

    o_loss, _, o_dq, o_dk = oracle.kl(od, xc["q"], xc["k"], xc["q_idx"], xc["k_idx"], ob.reshape(gb.shape),
                                      grad_scale=gs)
    rel = abs(g_loss - o_loss) / abs(o_loss)
    e_dq = np.abs(g_dq - o_dq).max()
    e_dk = np.abs(g_dk - o_dk).max()
    report(f"train_64k KL: loss {g_loss:.9g} vs oracle {o_loss:.9g} (rel {rel:.2e}); "
          f"dq_idx max abs {e_dq:.2e} (largest {np.abs(o_dq).max():.2e}); "
          f"dk_idx max abs {e_dk:.2e} (largest {np.abs(o_dk).max():.2e})")
    assert rel <= KL_REL
    for name, e, ref in (("dq_idx", e_dq, o_dq), ("dk_idx", e_dk, o_dk)):
        assert e <= GRAD_MAX, f"{name} max abs error {e:.3e}"
        assert e <= GRAD_REL * np.abs(ref).max(), f"{name} max error {e:.3e} vs largest {np.abs(ref).max():.3e}"
