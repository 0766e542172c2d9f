"""The reference arm of bench.py (the oracle on the host cores) prints one JSON line with the
benchmark contract's keys; runs on CPU on a small row sample."""
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--ref-rows", "16"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["unit"] == "query-tokens/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "prefill_32k_needles"
    # the same config object as our arm's line
    for key in ("N", "H_q", "H_kv", "d", "d_idx", "block_k", "topk", "batch_per_gpu", "global_batch",
                "parallelism", "l2", "step"):
        assert key in d["config"], key
    # ms_per_step is the measured time of a (sampled) step: the timed steps fit in the run
    assert d["steps"] * d["ms_per_step"] / 1e3 <= wall
    assert d["full_step_ms_extrapolated"] > d["ms_per_step"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
