"""Sequence-parallel index branch end to end in separate processes: two and three ranks, each its own
process on the same GPU with a gloo process group on 127.0.0.1, call the library's
sp.sp_index_topk on their zig-zag (or contiguous) key ranges: the local Top-k kernel, the gather
(staged through the host, as gloo moves host memory), the merge kernel, the local LSE_idx kernel,
the second gather and the eq (16) kernel ("4.1.1 · 监督与联合训练", section 3). Every rank must end
with the single-device selection (bit-exact) and LSE_idx.

A second pass feeds the oracle's local parts (host-side, float64 candidates of each rank's held
blocks) through the same gather into the library's merge and combine kernels, so the exchange is
also checked on parts that do not come from the CUDA path.

The ranks' kernels never wait on one another: the only waits are the host-side gathers."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, assign, shape):
    sys.path.insert(0, ROOT)
    import datetime

    import numpy as np

    import block_sparse_attention_idx_b200 as msa
    import oracle
    from block_sparse_attention_idx_b200 import sp
    from msa_inputs import small_prefill
    from oracle import sp as osp
    torch.cuda.set_device(0)
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world, timeout=datetime.timedelta(seconds=120))
    B, N, H_q, H_kv, d, d_idx, bk, k = shape
    dm = msa.MsaDims(B, N, H_q, H_kv, d, d_idx, bk, k)
    x = small_prefill(N, H_q, H_kv, d, d_idx, bk, k, seed=77 + N, B=B)  # every rank draws the same inputs
    qi, ki = x["q_idx"].cuda(), x["k_idx"].cuda()
    held = (sp.zigzag_ranges if assign == "zigzag" else sp.contiguous_ranges)(N, bk, world, rank)
    k_local = sp.local_keys(ki, held) if held else ki[:, :0]
    blocks, lse = sp.sp_index_topk(dm, qi, k_local, held, want_lse=True)
    ref_blocks, ref_lse = msa.msa_index_topk(dm, qi, ki, want_lse=True)
    torch.cuda.synchronize()
    res = {"held": held, "blocks_equal": bool(torch.equal(blocks, ref_blocks)),
           "lse_err": float((lse - ref_lse).abs().max()), "lse_scale": float(ref_lse.abs().max())}

    # the oracle's parts of this rank through the library's gather, merge and combine
    od = oracle.Dims(B, N, H_q, H_kv, d, d_idx, bk, k)
    hb = [(t0 // bk, -(-(t0 + n) // bk)) for t0, n in held]
    os_, oi_ = osp.local_topk(od, x["q_idx"], x["k_idx"], hb)
    # candidate scores as the kernels exchange them: raw block maxima, without scale_idx
    raw = torch.from_numpy(os_ * np.sqrt(d_idx)).float().cuda()
    ob = msa.msa_topk_merge(dm, sp.gather(raw), sp.gather(torch.from_numpy(oi_).cuda()))
    ob_ref, om, ol = oracle.index_topk(od, x["q_idx"], x["k_idx"], want_lse=True)
    ob_np = ob.cpu().numpy().reshape(ob_ref.shape)
    ml = osp.local_lse(od, x["q_idx"], x["k_idx"], ob_ref.reshape(B, N, H_kv, k + 1), hb)
    olse = msa.msa_lse_combine(dm, sp.gather(torch.from_numpy(ml).float().cuda()))
    res["oracle_parts_blocks_equal"] = bool(np.array_equal(ob_np, ob_ref))
    res["oracle_parts_near_ties"] = int((om < 1e-4).sum())
    res["oracle_parts_blocks_bad"] = int(((ob_np != ob_ref).any(axis=-1) & (om >= 1e-4)).sum())
    res["oracle_parts_lse_err"] = float(np.abs(olse.cpu().numpy().reshape(ol.shape) - ol).max())
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


SHAPES = {"main_1000": (1, 1000, 64, 4, 128, 64, 128, 4), "b2_ragged_777": (2, 777, 16, 2, 64, 64, 64, 3),
          "tiny_bk32_300": (1, 300, 8, 4, 64, 32, 32, 5)}


CASES = [("main_1000", 2, "zigzag"), ("main_1000", 3, "zigzag"), ("b2_ragged_777", 3, "zigzag"),
         ("tiny_bk32_300", 2, "zigzag"), ("main_1000", 2, "contiguous")]


@pytest.mark.parametrize("shape,world,assign", CASES, ids=[f"{a}-P{b}-{c}" for a, b, c in CASES])
def test_sp_index_topk_end_to_end_on_gloo_ranks(tmp_path, shape, world, assign):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), assign, SHAPES[shape]))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.exitcode is None:
            p.kill()
        assert p.exitcode == 0
    res = [json.load(open(os.path.join(tmp_path, f"rank{r}.json"))) for r in range(world)]
    N = SHAPES[shape][1]
    toks = sorted(t for r in res for t0, n in r["held"] for t in range(t0, t0 + n))
    assert toks == list(range(N))
    for r in res:
        assert r["blocks_equal"]
        assert r["lse_err"] <= 2e-5 * max(1.0, r["lse_scale"])
        assert r["oracle_parts_blocks_bad"] == 0
        assert r["oracle_parts_lse_err"] <= 1e-4
