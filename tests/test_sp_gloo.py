"""Sequence-parallel index branch, the exchange between ranks, on two and three CPU ranks over
gloo: each rank takes its key ranges from the library's assignment (contiguous or zig-zag,
block_sparse_attention_idx_b200.sp), computes their candidates and (max, exp-sum) pairs with the
oracle, the library's gather moves them, and the merge and eq (16) give the single-device selection
and LSE_idx on every rank. The same exchange with the library's kernels on the parts runs on a GPU
in test_gpu_sp_gloo."""
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


def _blocks_of(held, bk):
    """Token ranges -> half-open block ranges."""
    return [(t0 // bk, -(-(t0 + n) // bk)) for t0, n in held]


def _rank_main(rank, world, port, out_dir, assign):
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
    held = (sp.zigzag_ranges if assign == "zigzag" else sp.contiguous_ranges)(N, Bk, world, rank)
    hb = _blocks_of(held, Bk)
    cs, ci = osp.local_topk(dims, x["q_idx"], x["k_idx"], hb)
    S = sp.gather(torch.from_numpy(cs)).numpy()
    I = sp.gather(torch.from_numpy(ci)).numpy()
    blocks = osp.merge(dims, list(S), list(I))
    ml = osp.local_lse(dims, x["q_idx"], x["k_idx"], blocks, hb)
    lse = osp.combine_lse(sp.gather(torch.from_numpy(ml)).numpy())
    ref_blocks, _, ref_lse = oracle.index_topk(dims, x["q_idx"], x["k_idx"], want_lse=True)
    res = {"blocks_equal": bool(np.array_equal(blocks.reshape(ref_blocks.shape), ref_blocks)),
           "lse_err": float(np.abs(lse.reshape(ref_lse.shape) - ref_lse).max()),
           "held": held}
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("assign", ["zigzag", "contiguous"])
@pytest.mark.parametrize("world", [2, 3])
def test_sp_exchange_on_gloo_ranks(tmp_path, world, assign):
    port = _free_port()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), assign)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        assert p.exitcode == 0
    res = [json.load(open(os.path.join(tmp_path, f"rank{r}.json"))) for r in range(world)]
    # the ranks' ranges tile [0, 77) without overlap
    toks = sorted(t for r in res for t0, n in r["held"] for t in range(t0, t0 + n))
    assert toks == list(range(77))
    if assign == "zigzag":
        assert all(len(r["held"]) == 2 for r in res)
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
    assert sp.contiguous_ranges(N, Bk, 8, 0) == []  # 5 blocks over 8 ranks: rank 0 holds none
    assert [] in [sp.zigzag_ranges(N, Bk, 8, r) for r in range(8)]  # 5 blocks in 16 chunks: some rank holds none
    cs, ci = sp.no_candidates(dims, torch.device("cpu"))
    ocs, oci = osp.local_topk(dims, x["q_idx"], x["k_idx"], [])
    np.testing.assert_array_equal(cs.double().numpy(), ocs)
    np.testing.assert_array_equal(ci.numpy(), oci)
    full_s, full_i = osp.local_topk(dims, x["q_idx"], x["k_idx"], [(0, 5)])
    np.testing.assert_array_equal(osp.merge(dims, [full_s, ocs], [full_i, oci]), osp.merge(dims, [full_s], [full_i]))
    ml = sp.no_lse_pairs(dims, torch.device("cpu")).double().numpy()
    blocks = osp.merge(dims, [full_s], [full_i])
    own = osp.local_lse(dims, x["q_idx"], x["k_idx"], blocks, [(0, 5)])
    np.testing.assert_array_equal(osp.combine_lse([own, ml]), osp.combine_lse([own]))


@pytest.mark.parametrize("N,bk", [(32768, 128), (8192, 128), (77, 8), (1000, 32)])
@pytest.mark.parametrize("world", [2, 3, 4, 8])
def test_zigzag_assignment_tiles_the_keys_and_balances_the_causal_work(N, bk, world):
    """The zig-zag ranges of the ranks tile [0, N) in whole blocks, each rank's ranges are ordered
    and at most two, and the causal work of the local Top-k (pairs of a query and a complete past
    block it holds) is within 1.3x between ranks where every rank holds at least two chunks' worth
    of blocks; the contiguous assignment's first rank carries far more."""
    from block_sparse_attention_idx_b200 import sp
    nb = -(-N // bk)

    def work(held):
        # sum over queries i of the held blocks c < i // bk
        tot = 0
        for t0, n in held:
            for c in range(t0 // bk, -(-(t0 + n) // bk)):
                tot += max(0, N - (c + 1) * bk)
        return tot

    zz = [sp.zigzag_ranges(N, bk, world, r) for r in range(world)]
    toks = []
    for h in zz:
        assert len(h) <= 2
        for x, (t0, n) in enumerate(h):
            assert t0 % bk == 0 and n > 0 and (n % bk == 0 or t0 + n == N)
            if x == 1:
                assert t0 >= h[0][0] + h[0][1]
        toks += [(t0, n) for t0, n in h]
    toks.sort()
    assert toks[0][0] == 0 and toks[-1][0] + toks[-1][1] == N
    assert all(a0 + an == b0 for (a0, an), (b0, _) in zip(toks, toks[1:]))
    if nb >= 8 * world:
        w = [work(h) for h in zz]
        assert max(w) <= 1.3 * min(w), w
        c = [work(sp.contiguous_ranges(N, bk, world, r)) for r in range(world)]
        assert max(c) > 1.5 * min(c) or world == 1
