"""Failure detection on the device without any GPU fault.

Every wait inside the library's kernels is bounded; a wait that runs out sets MSA_ERR_TIMEOUT in the
call's status word and the kernel drains what it issued, frees its TMEM and returns, so the context
stays usable. The probe launch holds TMEM and a bulk copy in flight while its consumer waits on an
mbarrier that nothing arrives on: with the test hook's 20 us limit the wait gives up at once.
Device-side range checks (a cache length beyond the caches' capacity) are clamped and reported the
same way."""
import time

import pytest
import torch

import block_sparse_attention_idx_b200 as msa
import oracle
from msa_inputs import small_prefill

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _small_index_call():
    """An ordinary call on a fresh workspace: selection of a small random case (and its status)."""
    dm = msa.MsaDims(1, 300, 4, 2, 64, 32, 32, 4)
    x = small_prefill(300, 4, 2, 64, 32, 32, 4, seed=11, device=DEV)
    ws = msa.workspace(msa.MSA_OP_INDEX_TOPK, dm, DEV)
    blocks = msa.msa_index_topk(dm, x["q_idx"], x["k_idx"], ws=ws)
    return dm, x, blocks, msa.msa_get_device_status(ws)


def test_bounded_wait_runs_out_reports_timeout_and_the_context_stays_usable():
    ws = torch.zeros(256 + 4096, dtype=torch.uint8, device=DEV)
    torch.cuda.synchronize()
    msa.msa_debug_set_wait_ns(20_000)
    try:
        t0 = time.perf_counter()
        msa.msa_debug_wait_probe(ws)
        status = msa.msa_get_device_status(ws)
        dt = time.perf_counter() - t0
    finally:
        msa.msa_debug_set_wait_ns(0)
    assert status == msa.MSA_ERR_TIMEOUT
    # the probe gave up after the test limit, not after the 2 s default
    assert dt < 1.0, f"probe took {dt:.3f} s"
    # same device, same process: an ordinary call runs, reports no problem and is correct
    dm, x, blocks, st = _small_index_call()
    assert st == msa.MSA_OK
    od = oracle.Dims(1, 300, 4, 2, 64, 32, 32, 4)
    ob, om, _ = oracle.index_topk(od, x["q_idx"].cpu(), x["k_idx"].cpu())
    gb = blocks.cpu().numpy().reshape(ob.shape)
    assert ((gb != ob).any(axis=-1) & (om >= 1e-4)).sum() == 0


def test_default_limit_is_restored_after_the_test_hook():
    # with the hook back at 0 an ordinary call's status word carries the default limit: the call
    # succeeds (its waits are not cut short)
    _, _, _, st = _small_index_call()
    assert st == msa.MSA_OK


def _decode_case(B, L, seed, H_q=4, H_kv=2, d=64, d_idx=32, bk=32, k=4):
    g = torch.Generator(device=DEV).manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g, device=DEV).to(torch.bfloat16)
    x = dict(q=mk(B, H_q, d), q_idx=mk(B, H_kv, d_idx), k_cache=mk(B, L, H_kv, d), v_cache=mk(B, L, H_kv, d),
             k_idx_cache=mk(B, L, d_idx))
    return msa.MsaDims(B, L, H_q, H_kv, d, d_idx, bk, k), x


def test_decode_cache_len_outside_capacity_is_clamped_and_reported():
    dm, x = _decode_case(3, 1000, seed=21)
    ws = msa.workspace(msa.MSA_OP_DECODE, dm, DEV)
    bad = torch.tensor([1000 + 1, 0, 517], dtype=torch.int32, device=DEV)
    good = torch.tensor([1000, 1, 517], dtype=torch.int32, device=DEV)
    out_b, blk_b = msa.msa_sparse_attn_decode(dm, bad, x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                              x["k_idx_cache"], ws=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_DEVICE_CHECK
    out_g, blk_g = msa.msa_sparse_attn_decode(dm, good, x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                              x["k_idx_cache"], ws=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    # the out-of-range lengths were read as the nearest valid ones
    assert torch.equal(blk_b, blk_g)
    assert torch.equal(out_b, out_g)
