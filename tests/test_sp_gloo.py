"""Sequence-parallel index branch, the exchange between ranks, on two and three CPU ranks over
gloo: each rank computes its key range's candidates and (max, exp-sum) pairs with the oracle, the
library's gather (block_sparse_attention_idx_b200.sp) moves them, and the merge and eq (16) give
the single-device selection and LSE_idx on every rank."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import datetime
    import oracle
    from oracle import sp as osp
    from block_sparse_attention_idx_b200 import sp
    from msa_inputs import small_prefill
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world, timeout=datetime.timedelta(seconds=60))
    N, Bk, k, Hkv = 77, 8, 3, 2
    dims = oracle.Dims(B=1, N=N, H_q=2 * Hkv, H_kv=Hkv, d=8, d_idx=8, block_k=Bk, topk=k)
    x = small_prefill(N, 2 * Hkv, Hkv, 8, 8, Bk, k, seed=5)  # every rank draws the same inputs
    tok0, ntok = sp.split_range(N, Bk, world, rank)
    b0, b1 = tok0 // Bk, -(-(tok0 + ntok) // Bk)
    cs, ci = osp.local_topk(dims, x["q_idx"], x["k_idx"], b0, b1)
    S = sp.gather(torch.from_numpy(cs)).numpy()
    I = sp.gather(torch.from_numpy(ci)).numpy()
    blocks = osp.merge(dims, list(S), list(I))
    ml = osp.local_lse(dims, x["q_idx"], x["k_idx"], blocks, b0, b1)
    lse = osp.combine_lse(sp.gather(torch.from_numpy(ml)).numpy())
    ref_blocks, _, ref_lse = oracle.index_topk(dims, x["q_idx"], x["k_idx"], want_lse=True)
    res = {"blocks_equal": bool(np.array_equal(blocks.reshape(ref_blocks.shape), ref_blocks)),
           "lse_err": float(np.abs(lse.reshape(ref_lse.shape) - ref_lse).max()),
           "range": [tok0, ntok]}
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world", [2, 3])
def test_sp_exchange_on_gloo_ranks(tmp_path, world):
    port = _free_port()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        assert p.exitcode == 0
    res = [json.load(open(os.path.join(tmp_path, f"rank{r}.json"))) for r in range(world)]
    ranges = [r["range"] for r in res]
    assert ranges[0][0] == 0 and sum(n for _, n in ranges) == 77
    for r in res:
        assert r["blocks_equal"]
        assert r["lse_err"] <= 1e-12


def test_rank_without_keys_contributes_padding_only():
    """With more ranks than blocks a rank holds no key: its candidates are the padding the oracle
    gives for an empty range (-inf, -1), its (max, exp-sum) pairs are (-inf, 0), and adding such a
    rank changes neither the merged selection nor eq (16)."""
    sys.path.insert(0, ROOT)
    import oracle
    from oracle import sp as osp
    from block_sparse_attention_idx_b200 import sp
    from msa_inputs import small_prefill
    N, Bk, k, Hkv = 40, 8, 3, 2
    dims = oracle.Dims(B=1, N=N, H_q=2 * Hkv, H_kv=Hkv, d=8, d_idx=8, block_k=Bk, topk=k)
    x = small_prefill(N, 2 * Hkv, Hkv, 8, 8, Bk, k, seed=5)
    assert sp.split_range(N, Bk, 8, 0)[1] == 0  # 5 blocks over 8 ranks: rank 0 holds none
    cs, ci = sp.no_candidates(dims, torch.device("cpu"))
    ocs, oci = osp.local_topk(dims, x["q_idx"], x["k_idx"], 3, 3)
    np.testing.assert_array_equal(cs.double().numpy(), ocs)
    np.testing.assert_array_equal(ci.numpy(), oci)
    full_s, full_i = osp.local_topk(dims, x["q_idx"], x["k_idx"], 0, 5)
    np.testing.assert_array_equal(osp.merge(dims, [full_s, ocs], [full_i, oci]), osp.merge(dims, [full_s], [full_i]))
    ml = sp.no_lse_pairs(dims, torch.device("cpu")).double().numpy()
    blocks = osp.merge(dims, [full_s], [full_i])
    own = osp.local_lse(dims, x["q_idx"], x["k_idx"], blocks, 0, 5)
    np.testing.assert_array_equal(osp.combine_lse([own, ml]), osp.combine_lse([own]))
