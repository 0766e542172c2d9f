"""The dense warm-up KL ("MSA 中的 KL 对齐与局部知识蒸馏", section 5: before sparse training the index
branch is aligned to a teacher over the whole causal context) against the float64 oracle's KL with
every causal block selected. The oracle's reading of that case is itself pinned against the dense
warm-up definition (whole-matrix masked softmaxes and autograd) in test_oracle_pins.

Small sizes compare everything: the loss, dQ_idx of every row, dK_idx of every token and the
teacher's LSE (the dense causal attention LSE). At N = 65536 (the training workload) the oracle
checks sampled rows (dQ_idx and the teacher LSE of each); the loss and dK_idx are checked through
properties that hold at any size."""
import numpy as np
import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from msa_inputs import WORKLOADS, prefill_inputs, small_prefill
from parity import GRAD_MAX, GRAD_REL, KL_REL, LSE_MAX, report

pytestmark = pytest.mark.gpu

DEV = "cuda"


def dense_blocks(B, N, H_kv, bk):
    """Every causal block of every row: ids 0 .. i // bk, ascending, -1 padded to ceil(N / bk)."""
    nb = -(-N // bk)
    ids = np.arange(nb, dtype=np.int32)[None, :].repeat(N, 0)
    last = (np.arange(N) // bk)[:, None]
    ids[ids > last] = -1
    return np.ascontiguousarray(np.broadcast_to(ids[None, :, None, :], (B, N, H_kv, nb)))


@pytest.mark.parametrize("shape", [(1, 1000, 64, 4, 128, 64, 128), (2, 300, 64, 4, 128, 64, 128),
                                   (1, 512, 4, 2, 64, 32, 32), (2, 333, 4, 2, 64, 32, 32)],
                         ids=["main_1000", "main_b2_300", "tiny_512", "tiny_b2_333"])
def test_dense_kl_matches_oracle_every_row(shape):
    B, N, H_q, H_kv, d, d_idx, bk = shape
    nb = -(-N // bk)
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, 4, seed=900 + N, B=B)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, 1)  # topk is not used by the dense path
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, nb - 1)
    gs = float(B * N * H_kv)  # gradients of the summed KL: order-one entries
    g = {kk: vv.to(DEV) for kk, vv in x.items()}
    ws = msa.workspace(msa.MSA_OP_KL_DENSE, dm, DEV)
    loss, dq, dk, lse = msa.msa_kl_dense_fwd_grad(dm, g["q"], g["k"], g["q_idx"], g["k_idx"], grad_scale=gs,
                                                  want_lse=True, ws=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    blocks = dense_blocks(B, N, H_kv, bk)
    ol, _, odq, odk = oracle.kl(od, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, grad_scale=gs)
    _, olse = oracle.sparse_attn(od, x["q"], x["k"], x["v"], blocks)
    rel = abs(float(loss.item()) - ol) / abs(ol)
    e_dq = np.abs(dq.cpu().numpy().reshape(odq.shape) - odq).max()
    e_dk = np.abs(dk.cpu().numpy() - odk).max()
    e_lse = np.abs(lse.cpu().numpy().reshape(olse.shape) - olse).max()
    report(f"dense KL {shape}: loss rel {rel:.2e}, dq_idx {e_dq:.2e} (largest {np.abs(odq).max():.2e}), "
           f"dk_idx {e_dk:.2e} (largest {np.abs(odk).max():.2e}), teacher LSE {e_lse:.2e}")
    assert rel <= KL_REL
    assert e_lse <= LSE_MAX
    for name, e, ref in (("dq_idx", e_dq, odq), ("dk_idx", e_dk, odk)):
        assert e <= GRAD_MAX, f"{name} max abs error {e:.3e}"
        assert e <= GRAD_REL * np.abs(ref).max(), f"{name} {e:.3e} vs largest {np.abs(ref).max():.3e}"


def test_dense_kl_equals_sparse_kl_when_k_covers_every_block():
    """With k at least the number of blocks, the sparse entry point selects every causal block: both
    entry points compute the same KL (different kernels, same definition)."""
    B, N, H_q, H_kv, d, d_idx, bk = 1, 1100, 64, 4, 128, 64, 128
    nb = -(-N // bk)
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, nb, seed=31, B=B, device=DEV)
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, nb)
    gs = float(N * H_kv)
    blocks, lse_idx = msa.msa_index_topk(dm, x["q_idx"], x["k_idx"], want_lse=True)
    _, lse = msa.msa_sparse_attn_fwd(dm, x["q"], x["k"], x["v"], blocks)
    ls, dqs, dks = msa.msa_kl_fwd_grad(dm, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, lse, lse_idx,
                                       grad_scale=gs)
    ld, dqd, dkd = msa.msa_kl_dense_fwd_grad(dm, x["q"], x["k"], x["q_idx"], x["k_idx"], grad_scale=gs)
    torch.cuda.synchronize()
    assert abs(ls.item() - ld.item()) <= KL_REL * abs(ls.item())
    assert (dqs - dqd).abs().max().item() <= GRAD_MAX
    assert (dks - dkd).abs().max().item() <= GRAD_MAX


def test_dense_kl_train_64k_sampled_rows_and_invariants():
    w = WORKLOADS["train_64k"]
    x = prefill_inputs(w, device=DEV)
    nb = -(-w.N // w.block_k)
    dm = msa.MsaDims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    od = oracle.Dims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, nb - 1)
    gs = float(w.N * w.H_kv)
    ws = msa.workspace(msa.MSA_OP_KL_DENSE, dm, DEV)
    loss, dq, dk, lse = msa.msa_kl_dense_fwd_grad(dm, x["q"], x["k"], x["q_idx"], x["k_idx"], grad_scale=gs,
                                                  want_lse=True, ws=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    del ws
    # a KL divergence is never negative; P and P_idx each sum to one over a row's token set, so the
    # contributions to dK_idx cancel when summed over the tokens
    assert float(loss.item()) > 0.0
    tot = dk.double().sum(dim=1).abs().max().item()
    scale = dk.double().abs().sum(dim=1).max().item()
    assert tot <= 1e-3 * scale
    rng = np.random.default_rng(64)
    rows = np.array(sorted({0, 1, 127, 128, w.N // 2, w.N - 1} | set(rng.choice(w.N, 14, replace=False).tolist())),
                    dtype=np.int64)
    xc = {kk: vv.cpu() for kk, vv in x.items()}
    blocks = dense_blocks(w.B, w.N, w.H_kv, w.block_k)
    _, _, odq, _ = oracle.kl(od, xc["q"], xc["k"], xc["q_idx"], xc["k_idx"], blocks, grad_scale=gs, rows=rows)
    _, olse = oracle.sparse_attn(od, xc["q"], xc["k"], xc["v"], blocks, rows=rows)
    gdq = dq.cpu().numpy().reshape(w.B * w.N, w.H_kv, w.d_idx)[rows]
    glse = lse.cpu().numpy().reshape(w.B * w.N, w.H_q)[rows]
    e_dq = np.abs(gdq - odq).max()
    e_lse = np.abs(glse - olse).max()
    report(f"dense KL train_64k sampled rows: dq_idx {e_dq:.2e} (largest {np.abs(odq).max():.2e}), "
           f"teacher LSE {e_lse:.2e}; loss {loss.item():.6f}")
    assert e_lse <= LSE_MAX
    assert e_dq <= GRAD_MAX and e_dq <= GRAD_REL * np.abs(odq).max()
