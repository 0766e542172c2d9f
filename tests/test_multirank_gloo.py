"""The benchmark's multi-rank host logic on two CPU ranks over gloo: the max over ranks that times a
step, per-rank independent inputs (weak scaling, no data-path collective), the whole-job
throughput, and the reference arm that only rank 0 runs."""
import json
import os
import socket
import sys

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
    import bench
    from msa_inputs import WORKLOADS, prefill_inputs
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world, timeout=datetime.timedelta(seconds=60))
    res = {}
    # step time: each rank reports its own; everyone gets the slowest
    res["max"] = bench.max_over_ranks(1.5 + rank, world, device="cpu")
    # independent per-rank inputs for the same workload shape
    w = WORKLOADS["prefill_8k"]
    x = prefill_inputs(w, device="cpu", seed=bench.rank_seed(w, rank), N=256)
    res["seed"] = bench.rank_seed(w, rank)
    res["q_sum"] = float(x["q"].float().sum())
    res["shape"] = list(x["q"].shape)
    res["value"] = bench.job_throughput(w.N * w.B, world, res["max"])

    class A:
        ref_rows, steps, warmup, gpus, workload = 4, 1, 0, world, "prefill_32k_needles"
    if rank != 0:
        res["reference"] = bench.run_reference(A, world, rank)  # only rank 0 runs the oracle
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_host_logic(tmp_path):
    world = 2
    port = _free_port()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    # every rank sees the slowest rank's time
    assert res[0]["max"] == res[1]["max"] == 2.5
    # weak scaling: same shapes, different seeded data on each rank
    assert res[0]["shape"] == res[1]["shape"]
    assert res[0]["seed"] != res[1]["seed"] and res[0]["q_sum"] != res[1]["q_sum"]
    # whole-job throughput = all ranks' tokens over the slowest step
    assert res[0]["value"] == pytest.approx(8192 * 2 / 2.5e-3)
    assert res[1]["reference"] is None
