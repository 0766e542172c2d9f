#!/usr/bin/env python
"""Benchmark of the MSA layer hot path on B200 through the libmsa C ABI; prints one JSON line.

Headline step (one pass of the prefill hot path over one batch): msa_index_topk (index scoring,
causal block max-pool, Top-k + local block) then msa_sparse_attn_fwd (exact sparse attention) on the
N=32768, 64-query / 4-KV-head needle workload. value = query tokens per second over all ranks.
Secondary measurements in the same line: the decode step (16 x 262144 cached tokens, us per step =
us per generated token of each sequence) and the training KL alignment (N=65536).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Ranks run independent sequences (weak scaling, no data-path collective); timing is on the device
with CUDA events, the max over ranks. The L2 cache is flushed (a 256 MiB read) before every
timed step. --impl reference times the float64 CPU oracle on a bounded sample of the same rows.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from msa_inputs import WORKLOADS, prefill_inputs, decode_inputs  # noqa: E402

METRIC = "MSA prefill query-tokens/s (N=32K, 64q/4kv heads); decode µs/token; % roofline"
HEADLINE = "prefill_32k_needles"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """SM clock and clock-event (throttle) reasons read through NVML every 2 ms in a background
    thread while the timed region runs (read-only queries; no setting is changed). Entering waits
    until the first sample is in, so sampling covers the whole timed region."""
    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu, self.period = gpu_index, period_s
        self.samples, self.max_mhz, self.err = [], None, None
        self._stop = None

    def _run(self):
        import pynvml as nv
        try:
            nv.nvmlInit()
            uuid = torch.cuda.get_device_properties(self.gpu).uuid
            h = None
            for x in range(nv.nvmlDeviceGetCount()):
                hx = nv.nvmlDeviceGetHandleByIndex(x)
                u = nv.nvmlDeviceGetUUID(hx)
                u = u.decode() if isinstance(u, bytes) else u
                if str(uuid) in u:
                    h = hx
            if h is None:
                h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            bits = {k: getattr(nv, v) for k, v in self.REASONS.items()}
            while not self._stop.is_set():
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((mhz, [k for k, b in bits.items() if rs & b]))
                time.sleep(self.period)
            nv.nvmlShutdown()
        except Exception as e:  # sampling must never break the benchmark
            self.err = f"{type(e).__name__}: {e}"

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        t0 = time.time()
        while not self.samples and self.err is None and time.time() - t0 < 5.0:
            time.sleep(0.005)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join(timeout=5)

    def summary(self) -> dict:
        if len(self.samples) > 2:
            self.samples = self.samples[1:]  # the first one is taken before the timed region starts
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0,
                    "error": self.err}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml, 2 ms"}


def selected_tokens(blocks: torch.Tensor, block_k: int) -> int:
    """Sum over (b, i, r) of |J|: causal tokens of the selected blocks (the algorithmic work)."""
    B, N, H_kv, K1 = blocks.shape
    i = torch.arange(N, device=blocks.device).view(1, N, 1, 1)
    c = blocks.long()
    n = torch.clamp(i - c * block_k + 1, max=block_k)
    return int(torch.where(c >= 0, n, torch.zeros_like(n)).sum().item())


def valid_slots(blocks: torch.Tensor, block_k: int) -> int:
    """Number of (b, i, r, slot) selections that name a causal block (each yields one partial)."""
    B, N, H_kv, K1 = blocks.shape
    i = torch.arange(N, device=blocks.device).view(1, N, 1, 1)
    c = blocks.long()
    return int(((c >= 0) & (c <= i // block_k)).sum().item())


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch, per unit of work, from an
# ncu capture of the kernel; it holds only for the kernel source it was measured on (sha256 of the
# file), and reads null once that file changes.
MEASURED_TRAFFIC = {
    # prefill_8k capture (dram read 206,667,520 B + write 1,967,239,936 B per launch over 60,309,504
    # selected tokens), scaled by the selected tokens of the timed launch
    "attn_kv_outer": {"file": "block_sparse_attention_idx_b200/csrc/msa_attn.cu",
                      "sha256": "11bf6bf43a5ec6c71421ad4d730aa2ad534fab2788f3cb4cb682f2627595f9c0",
                      "bytes_per_unit": (206667520 + 1967239936) / 60309504, "unit": "selected token",
                      "capture": "profiles/attn_kv_outer_prefill_8k.md"},
    # training capture at N=8192 (dram read 993,972,992 B + write 132,998,656 B per launch over
    # 60,309,504 selected tokens), scaled by the selected tokens of the timed launch
    "kl_kv_outer": {"file": "block_sparse_attention_idx_b200/csrc/msa_kl.cu",
                    "sha256": "5bdbc48d446823c16a19b6fb37cd93766e699a6ebb9553cb0633fa63e61a978d",
                    "bytes_per_unit": (993972992 + 132998656) / 60309504, "unit": "selected token",
                    "capture": "profiles/kl_kv_outer_train_8k.md"},
    # attention backward at N=8192 (dram read 6,612,550,485 B + write 3,289,236,480 B per launch over
    # 60,309,504 selected tokens; most of it is the read-modify-write of dQ by the per-item reductions)
    "attn_bwd": {"file": "block_sparse_attention_idx_b200/csrc/msa_bwd.cu",
                 "sha256": "a4643c88591d2bddd8e05910abc956258cb6b52d27530488526b1f18be7f5e2e",
                 "bytes_per_unit": (6612550485 + 3289236480) / 60309504, "unit": "selected token",
                 "capture": "profiles/attn_bwd_train_8k.md"},
    # decode scans at 16 x 131,072 (read + write per launch over 16 x 130,944 scanned tokens), scaled
    # by the scanned tokens of the timed launch
    "dec_scan": {"file": "block_sparse_attention_idx_b200/csrc/msa_decode.cu",
                 "sha256": "f603b9d207e2f59c5d3e090b6bded69c342452ba2fb824cc0959092b10450bfd",
                 "bytes_per_unit": (268227744 + 606608) / (16 * 130944), "unit": "scanned token",
                 "capture": "profiles/decode_16x256k.md"},
    "dec_scan_e4m3": {"file": "block_sparse_attention_idx_b200/csrc/msa_decode.cu",
                      "sha256": "f603b9d207e2f59c5d3e090b6bded69c342452ba2fb824cc0959092b10450bfd",
                      "bytes_per_unit": (142531008 + 148864) / (16 * 130944), "unit": "scanned token",
                      "capture": "profiles/decode_16x256k.md"},
}


def measured_traffic(kernel: str, units: float):
    m = MEASURED_TRAFFIC.get(kernel)
    if not m or not m["sha256"]:
        return None
    import hashlib
    with open(os.path.join(ROOT, m["file"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != m["sha256"]:
            return None
    return m["bytes_per_unit"] * units


def flush_l2(flush: torch.Tensor) -> None:
    """Evicts the previous step's lines from the 126 MB L2 by READING a 256 MiB buffer. A write
    would also evict them, but would leave the L2 full of dirty lines whose write-back then lands
    inside the timed step and competes with its reads."""
    torch.amax(flush.view(torch.int32))


def timed_steps(fn, steps: int, flush: torch.Tensor):
    """Per-step device times (ms) with CUDA events on the current stream; L2 flushed before each."""
    st = torch.cuda.current_stream()
    times = []
    for _ in range(steps):
        flush_l2(flush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        fn()
        b.record(st)
        times.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in times]


def streamed_steps(xs, host, out_host, dims, ws_i, ws_a, msa, n_steps: int) -> float:
    """n_steps prefill steps through the public API, pipelined over three streams: step s uploads
    its inputs into device buffer s % 2 (once step s - 2 has finished reading it), computes on the
    compute stream, and downloads its output into pinned host buffer s % 2. Each step's own copies
    are inside the region; the overlap is between different steps. Returns the device time (ms)
    from before the first upload to after the last download."""
    cur = torch.cuda.current_stream()
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(cur)
    for st in (s_in, s_cmp, s_out):
        st.wait_stream(cur)
    done = [None, None]
    for s in range(n_steps):
        j = s % 2
        with torch.cuda.stream(s_in):
            if done[j] is not None:
                s_in.wait_event(done[j])
            for k in host:
                xs[j][k].copy_(host[k], non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ready)
            blocks = msa.msa_index_topk(dims, xs[j]["q_idx"], xs[j]["k_idx"], ws=ws_i)
            out, _ = msa.msa_sparse_attn_fwd(dims, xs[j]["q"], xs[j]["k"], xs[j]["v"], blocks, ws=ws_a,
                                             out_dtype=torch.bfloat16)
            done[j] = torch.cuda.Event()
            done[j].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[j])
            out_host[j].copy_(out, non_blocking=True)
            out.record_stream(s_out)
    for st in (s_in, s_cmp, s_out):
        cur.wait_stream(st)
    b.record(cur)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def roofline_entry(bound, achieved, peak, unit, traffic=None):
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": (achieved / peak) if (achieved is not None and peak) else None, "traffic": traffic}


def profile_avg(prof: dict) -> dict:
    return {k: {"avg_ms": v[0] / max(v[1], 1), "launches": v[1], "total_ms": v[0]} for k, v in prof.items()}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest of the ranks' values (every rank takes part and gets the answer)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w, rank: int) -> int:
    """Seed of a rank's synthetic inputs: every rank runs its own independent sequences."""
    return 1000 + w.cid + 7919 * rank


def workload_config(w, world: int) -> dict:
    """The `config` object of the JSON line (the same in both arms)."""
    return {"workload": w.name, "N": w.N, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d, "d_idx": w.d_idx,
            "block_k": w.block_k, "topk": w.topk, "batch_per_gpu": w.B, "global_batch": w.B * world,
            "parallelism": f"dp{world} (independent sequences)",
            "l2": "flushed (256 MiB read) before every timed step; inputs also larger than L2; the pipelined "
                  "e2e steps are not flushed (625 MB uploaded per step)",
            "step": "msa_index_topk + msa_sparse_attn_fwd_bf16 (O stored as bf16, rounded from the fp32 result)"}


def rnd(x, sig: int = 4):
    """Floats rounded to `sig` significant digits, recursively (keeps the JSON line short)."""
    if isinstance(x, float):
        return float(f"{x:.{sig}g}") if math.isfinite(x) else x
    if isinstance(x, dict):
        return {k: rnd(v, sig) for k, v in x.items()}
    if isinstance(x, (list, tuple)):
        return [rnd(v, sig) for v in x]
    return x


def job_throughput(units_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's step time."""
    return units_per_rank * world / (slowest_ms * 1e-3)


# ============================================================================ reference arm
def run_reference(args, world, rank):
    """The float64 CPU oracle on a bounded row sample of the headline workload per step."""
    if rank != 0:
        return None
    import numpy as np
    import oracle
    w = WORKLOADS[HEADLINE]
    x = prefill_inputs(w, device="cpu")
    od = oracle.Dims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    rows_per_step = args.ref_rows
    rng = np.random.default_rng(0)
    full_blocks = np.full((w.B, w.N, w.H_kv, w.topk + 1), -1, dtype=np.int32)

    def step():
        rows = np.sort(rng.choice(w.N, size=rows_per_step, replace=False))
        b, _, _ = oracle.index_topk(od, x["q_idx"], x["k_idx"], rows=rows)
        full_blocks[0, rows] = b
        oracle.sparse_attn(od, x["q"], x["k"], x["v"], full_blocks, rows=rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = rows_per_step * args.steps / dt
    sample = (f"{rows_per_step} uniformly drawn query rows of {HEADLINE} per step (index Top-k + sparse "
              f"attention); a step is one such sample, timed")
    return {"metric": METRIC, "value": value, "unit": "query-tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            # not a measurement: the time a whole N-row step would take at the sampled rate
            "full_step_ms_extrapolated": 1e3 * dt / args.steps * (w.N / rows_per_step),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": "query-tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "query-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ============================================================================ our arm
def cpu_baseline(x, w, rows_n: int, blocks=None, out=None):
    """The oracle as it stands on a bounded row sample of the same workload (rank 0, N=1). With the
    GPU's selection and output of the same inputs, also their parity on that sample: selection
    (bit-exact except near-ties: cutoff margin < 1e-4, counted) and attention error on the rows
    where both selected the same blocks."""
    import numpy as np
    import oracle
    od = oracle.Dims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    xc = {k: x[k].cpu() for k in ("q", "k", "v", "q_idx", "k_idx")}
    rows = np.sort(np.random.default_rng(1).choice(w.N, size=rows_n, replace=False))
    full = np.full((w.B, w.N, w.H_kv, w.topk + 1), -1, dtype=np.int32)
    t0 = time.perf_counter()
    b, margin, _ = oracle.index_topk(od, xc["q_idx"], xc["k_idx"], rows=rows)
    full[0, rows] = b
    oo, _ = oracle.sparse_attn(od, xc["q"], xc["k"], xc["v"], full, rows=rows)
    dt = time.perf_counter() - t0
    res = {"value": rows_n / dt, "unit": "query-tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
           "sample": f"{rows_n} uniformly drawn query rows of {w.name} (index Top-k + sparse attention), "
                     f"{dt:.1f} s"}
    par = None
    if blocks is not None and out is not None:
        rt = torch.from_numpy(rows).to(blocks.device)
        gb = blocks.reshape(w.B * w.N, w.H_kv, w.topk + 1)[rt].cpu().numpy()
        og = out.reshape(w.B * w.N, w.H_q, w.d)[rt].double().cpu().numpy()
        near = margin < 1e-4
        differ = (gb != b).any(axis=-1)
        same = ~differ.any(axis=-1)
        err = np.abs(og[same] - oo[same])
        # the output is bf16: the fp32 bound plus half a bf16 unit (at most 2^-8 |o|)
        within = bool((err <= 1e-2 + 2.0 ** -8 * np.abs(oo[same])).all())
        par = {"sample": f"the cpu_baseline rows ({rows_n} query rows x {w.H_kv} groups)",
               "selection_pairs": int(gb.shape[0] * w.H_kv), "near_ties": int(near.sum()),
               "near_ties_selected_differently": int((differ & near).sum()),
               "mismatches_outside_near_ties": int((differ & ~near).sum()),
               "attn_rows_compared": int(same.sum()),
               "attn_max_abs_err": float(err.max()) if err.size else None,
               "attn_mean_abs_err": float(err.mean()) if err.size else None,
               "attn_within_bound": within,
               "tolerance": "selection bit-exact outside near-ties; attention (bf16 output) max abs "
                            "1e-2 + 2^-8 |o| elementwise"}
    return res, par


def bench_prefill(args, world, rank, msa, pk):
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    x = prefill_inputs(w, device=dev, seed=rank_seed(w, rank))
    dims = msa.MsaDims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    ws_i = msa.workspace(msa.MSA_OP_INDEX_TOPK, dims, dev)
    ws_a = msa.workspace(msa.MSA_OP_ATTN_FWD, dims, dev)
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        blocks = msa.msa_index_topk(dims, x["q_idx"], x["k_idx"], ws=ws_i)
        return blocks, msa.msa_sparse_attn_fwd(dims, x["q"], x["k"], x["v"], blocks, ws=ws_a, out_dtype=torch.bfloat16)

    for _ in range(args.warmup):
        blocks, _ = step()
    torch.cuda.synchronize()
    sel_tok = selected_tokens(blocks, w.block_k)  # sum_{i,r} |J|
    G = w.H_q // w.H_kv
    # merge: read every valid partial (fp16 o + fp32 lse) and the selection, write bf16 out + fp32 lse
    merge_bytes = (valid_slots(blocks, w.block_k) * G * (2 * w.d + 4) + w.B * w.N * w.H_q * (2 * w.d + 4)
                   + blocks.numel() * 4)
    attn_flops = 4.0 * w.d * G * sel_tok
    index_flops = 2.0 * w.d_idx * w.H_kv * w.N * (w.N + 1) / 2
    msa.msa_profile_read()
    barrier(world)
    msa.msa_profile_enable(True)
    with ClockSampler(dev.index) as cs:
        t = timed_steps(step, args.steps, flush)
    msa.msa_profile_enable(False)
    prof = profile_avg(msa.msa_profile_read())
    barrier(world)
    step_ms = max_over_ranks(sum(t) / len(t), world)
    value = job_throughput(w.N * w.B, world, step_ms)
    # roofline of the dominant kernel (live CUDA-event durations of its launches)
    dom = max(prof, key=lambda k: prof[k]["total_ms"])
    per_kernel = {}
    for k, v in prof.items():
        fl = attn_flops if k == "attn_kv_outer" else index_flops if k == "index_topk" else None
        tf = fl / (v["avg_ms"] * 1e-3) / 1e12 if fl else None
        per_kernel[k] = {"avg_ms": round(v["avg_ms"], 4), "launches": v["launches"],
                         "share": round(v["total_ms"] / sum(u["total_ms"] for u in prof.values()), 4),
                         **({"tflops": round(tf, 1), "frac_of_measured_bf16": round(tf / pk["bf16_tflops"], 4)}
                            if tf else {})}
        if k == "attn_merge":
            gbs = merge_bytes / (v["avg_ms"] * 1e-3) / 1e9
            per_kernel[k].update({"bytes": merge_bytes, "gbs": round(gbs, 1),
                                  "frac_of_measured_hbm": round(gbs / pk["hbm_gbs"], 4)})
    dfl = attn_flops if dom == "attn_kv_outer" else index_flops if dom == "index_topk" else None
    roof = roofline_entry("tensor", dfl / (prof[dom]["avg_ms"] * 1e-3) / 1e12 if dfl else None,
                          pk["bf16_tflops"], "TFLOP/s", measured_traffic(dom, sel_tok))
    roof["kernel"] = dom
    roof["flops_per_launch"] = dfl
    roof["peak_source"] = f"{pk['source']} bf16 burst"
    # e2e through the public API with pinned host buffers (H2D inputs, D2H output inside the region)
    host = {k: x[k].cpu().pin_memory() for k in ("q", "k", "v", "q_idx", "k_idx")}
    out_host = [torch.empty(x["q"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()

    def e2e_step():
        for k in host:
            x[k].copy_(host[k], non_blocking=True)
        _, (out, _) = step()
        out_host[0].copy_(out, non_blocking=True)

    e2e_ms = e2e_serial_ms = float("nan")
    if not args.no_e2e:
        e2e_steps = max(1, min(args.steps, 10))
        for _ in range(2):
            e2e_step()
        barrier(world)
        te = timed_steps(e2e_step, min(e2e_steps, 5), flush)
        e2e_serial_ms = max_over_ranks(sum(te) / len(te), world)
        xs = [x, {k: torch.empty_like(x[k]) for k in host}]
        streamed_steps(xs, host, out_host, dims, ws_i, ws_a, msa, 2)  # warm-up of the pipelined form
        barrier(world)
        e2e_ms = max_over_ranks(streamed_steps(xs, host, out_host, dims, ws_i, ws_a, msa, e2e_steps) / e2e_steps,
                                world)
        del xs
    res = {"value": value, "ms_per_step": step_ms, "roofline": roof, "kernels": per_kernel, "clocks": cs.summary(),
           "e2e": {"value": job_throughput(w.N * w.B, world, e2e_ms), "unit": "query-tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                   "pipelined": "consecutive steps overlap: step s+1 uploads while step s computes and downloads",
                   "serial_ms_per_step": e2e_serial_ms},
           # index Top-k, the six inverse-list kernels, attention and merge (memsets are not counted)
           "gpu_launches": 9 * args.steps,
           "work": {"selected_tokens": sel_tok, "mean_J": sel_tok / (w.N * w.H_kv), "attn_flops": attn_flops,
                    "index_flops": index_flops}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        blocks, (out, _) = step()
        res["cpu_baseline"], res["parity"] = cpu_baseline(x, w, args.cpu_rows, blocks, out)
        del blocks, out
    del ws_a, x
    torch.cuda.empty_cache()
    return res


def measure_decode(args, world, step, scan_kernel, scan_bytes, step_bytes, pk, msa, scanned_tokens=None):
    """Eager and graph-replayed µs per decode step, and a profiled pass for the kernel split."""
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    # (1) eager API calls, no profiler events in the stream
    barrier(world)
    t = timed_steps(step, args.decode_steps, flush)
    us = max_over_ranks(1e3 * sum(t) / len(t), world)
    # (2) the same call captured once in a CUDA graph and replayed, as a serving loop runs decode
    us_graph, graph_note = None, None
    try:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step()
        torch.cuda.current_stream().wait_stream(s)
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        tg = timed_steps(g.replay, args.decode_steps, flush)
        us_graph = 1e3 * sum(tg) / len(tg)
        del g
    except Exception as ex:  # noqa: BLE001 -- reported, the eager number stands
        graph_note = f"graph capture failed: {type(ex).__name__}"
    us_graph = max_over_ranks(us_graph if us_graph is not None else float("nan"), world)
    # (3) a profiled pass for the per-kernel breakdown (CUDA events around every launch)
    msa.msa_profile_read()
    msa.msa_profile_enable(True)
    timed_steps(step, args.decode_steps, flush)
    msa.msa_profile_enable(False)
    prof = profile_avg(msa.msa_profile_read())
    # the batch may be cut into parts (one scan launch each): time per step = total / steps
    scan_ms = prof[scan_kernel]["total_ms"] / args.decode_steps
    res = {"us_per_step": us, "us_per_step_graph": us_graph, "bytes_per_step": step_bytes,
           "step_roofline": roofline_entry("hbm", step_bytes / (us * 1e-6) / 1e9, pk["hbm_gbs"], "GB/s"),
           "step_roofline_graph": roofline_entry("hbm", step_bytes / (us_graph * 1e-6) / 1e9, pk["hbm_gbs"], "GB/s")
           if us_graph == us_graph else None,
           "roofline": {**roofline_entry("hbm", scan_bytes / (scan_ms * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s",
                                         measured_traffic(scan_kernel, scanned_tokens or 0) if scanned_tokens else None),
                        "kernel": scan_kernel, "bytes_per_step": scan_bytes,
                        "launches_per_step": prof[scan_kernel]["launches"] // args.decode_steps},
           "kernels": {k: {"ms_per_step": round(v["total_ms"] / args.decode_steps, 4),
                           "launches_per_step": v["launches"] // args.decode_steps} for k, v in prof.items()}}
    if graph_note:
        res["graph_note"] = graph_note
    return res


def bench_decode(args, world, rank, msa, pk):
    """The bf16 decode step, and the same step with FP8 (e4m3) index keys plus the report of the
    rows whose selection differs between the two scorings (with their bf16 cutoff margins)."""
    w = WORKLOADS["decode_16x256k"]
    dev = torch.device("cuda", torch.cuda.current_device())
    L = args.decode_len or w.N
    x = decode_inputs(w, device=dev, seed=rank_seed(w, rank), L=L)
    dims = msa.MsaDims(w.B, L, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    ws = msa.workspace(msa.MSA_OP_DECODE, dims, dev)

    def step():
        return msa.msa_sparse_attn_decode(dims, x["cache_len"], x["q"], x["q_idx"], x["k_cache"], x["v_cache"],
                                          x["k_idx_cache"], ws=ws)

    for _ in range(max(3, args.warmup)):
        out, blocks = step()
    torch.cuda.synchronize()
    nscored = ((L - 1) // w.block_k) * w.block_k
    scan_bytes = w.B * nscored * w.d_idx * 2
    sel_blocks = int((blocks >= 0).sum().item())
    kv_bytes = sel_blocks * w.block_k * w.d * 2 * 2
    small_bytes = w.B * (w.H_q * w.d * 2 * 2 + w.H_kv * w.d_idx * 2)
    m = measure_decode(args, world, step, "dec_scan", scan_bytes, scan_bytes + kv_bytes + small_bytes, pk, msa,
                       scanned_tokens=w.B * nscored)
    res = {"workload": "decode_16x256k" if L == w.N else f"decode_16x{L}", "us_per_token": m["us_per_step"],
           "tokens_per_s": w.B * world / (m["us_per_step"] * 1e-6), **m}

    # FP8 index keys: the cache's K_idx quantised once (as a serving cache stores it), then the
    # same step scoring from e4m3 codes + per-token scales
    codes, kscale = msa.msa_quantize_e4m3_rows(x["k_idx_cache"])

    def step8():
        return msa.msa_sparse_attn_decode_fp8idx(dims, x["cache_len"], x["q"], x["q_idx"], x["k_cache"],
                                                 x["v_cache"], codes, kscale, ws=ws)

    for _ in range(max(3, args.warmup)):
        out8, blocks8 = step8()
    torch.cuda.synchronize()
    scan8 = w.B * nscored * (w.d_idx + 4)
    sel8 = int((blocks8 >= 0).sum().item())
    m8 = measure_decode(args, world, step8, "dec_scan_e4m3", scan8,
                        scan8 + sel8 * w.block_k * w.d * 2 * 2 + small_bytes, pk, msa, scanned_tokens=w.B * nscored)
    # flip report: bf16 vs FP8 selection, bf16 margins of the rows that flip, planted-block recall
    _, b16, mg16 = msa.msa_sparse_attn_decode(dims, x["cache_len"], x["q"], x["q_idx"], x["k_cache"],
                                              x["v_cache"], x["k_idx_cache"], ws=ws, want_margin=True)
    _, b8, mg8 = msa.msa_sparse_attn_decode_fp8idx(dims, x["cache_len"], x["q"], x["q_idx"], x["k_cache"],
                                                   x["v_cache"], codes, kscale, ws=ws, want_margin=True)
    torch.cuda.synchronize()
    flipped = (b16 != b8).any(dim=-1)
    planted = x["planted_blocks"]

    def planted_recall(sel):
        hit = (sel[:, :, :, None] == planted[:, None, None, :]).any(dim=2)  # [B, H_kv, n_planted]
        return float(hit.float().mean().item())

    fin16 = mg16[torch.isfinite(mg16)]
    m8["flip_report"] = {
        "rows": int(flipped.numel()), "rows_flipped": int(flipped.sum().item()),
        "slots_changed": int(sum(len(set(b16[i, r].tolist()) ^ set(b8[i, r].tolist())) // 2
                                 for i in range(w.B) for r in range(w.H_kv))),
        "bf16_margin_median": float(fin16.median().item()) if fin16.numel() else None,
        "bf16_margin_max_of_flipped": float(mg16[flipped].max().item()) if flipped.any() else None,
        "fp8_margin_median": float(mg8[torch.isfinite(mg8)].median().item()) if torch.isfinite(mg8).any() else None,
        "planted_recall_bf16": planted_recall(b16), "planted_recall_fp8": planted_recall(b8)}
    m8["cache_bytes"] = {"k_idx_bf16": w.B * L * w.d_idx * 2, "k_idx_e4m3_codes_and_scales": w.B * L * (w.d_idx + 4)}
    res["fp8_index"] = m8
    del x, ws, codes, kscale
    torch.cuda.empty_cache()
    return res


def bench_sp(args, world, rank, msa, pk):
    """Sequence-parallel index branch on the headline workload with P ranks emulated on this GPU:
    each rank's local Top-k and local (max, exp-sum) on its own K_idx timed separately (on P GPUs
    they run side by side, so the step's compute is the slowest rank), plus the merge and the
    eq (16) combine that every rank runs after the all-gather. Both key assignments are measured:
    contiguous ranges, and the zig-zag one (chunks p and 2P-1-p of 2P) that the library's
    sp_index_topk callers use. The all-gather itself is not timed here (one GPU); its bytes per
    rank are reported."""
    from block_sparse_attention_idx_b200 import sp
    w = WORKLOADS[HEADLINE]
    dev = torch.device("cuda", torch.cuda.current_device())
    x = prefill_inputs(w, device=dev, seed=rank_seed(w, rank))
    dims = msa.MsaDims(w.B, w.N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    ref_blocks, ref_lse = msa.msa_index_topk(dims, x["q_idx"], x["k_idx"], want_lse=True)
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    res = {"workload": HEADLINE, "note": "ranks emulated on one GPU; the all-gather is not timed"}
    ws = msa.workspace(msa.MSA_OP_INDEX_TOPK, dims, dev)
    ws_l = msa.workspace(msa.MSA_OP_LSE_IDX_LOCAL, dims, dev)
    for P in (2, 8):
        for assign, ranges_of in (("zigzag", sp.zigzag_ranges), ("contiguous", sp.contiguous_ranges)):
            helds = [ranges_of(w.N, w.block_k, P, p) for p in range(P)]
            keys = [sp.local_keys(x["k_idx"], h) for h in helds]
            local_ms, cands = [], []
            for h, kl in zip(helds, keys):
                for _ in range(max(3, args.warmup)):
                    c = msa.msa_index_topk_local(dims, x["q_idx"], kl, h, ws=ws)
                t = timed_steps(lambda: msa.msa_index_topk_local(dims, x["q_idx"], kl, h, ws=ws), 5, flush)
                local_ms.append(sorted(t)[len(t) // 2])
                cands.append(c)
            cs = torch.stack([c[0] for c in cands])
            ci = torch.stack([c[1] for c in cands])
            for _ in range(3):
                blocks = msa.msa_topk_merge(dims, cs, ci)
            tm = timed_steps(lambda: msa.msa_topk_merge(dims, cs, ci), 5, flush)
            lse_ms, mls = [], []
            for h, kl in zip(helds, keys):
                ml = msa.msa_lse_idx_local(dims, x["q_idx"], kl, h, blocks, ws=ws_l).clone()
                t = timed_steps(lambda: msa.msa_lse_idx_local(dims, x["q_idx"], kl, h, blocks, ws=ws_l), 3, flush)
                lse_ms.append(sorted(t)[len(t) // 2])
                mls.append(ml)
            ml_all = torch.stack(mls)
            lse = msa.msa_lse_combine(dims, ml_all)
            tc = timed_steps(lambda: msa.msa_lse_combine(dims, ml_all), 5, flush)
            torch.cuda.synchronize()
            rows = w.B * w.N * w.H_kv
            res[f"P{P}_{assign}"] = {
                "held_tokens": [[list(r) for r in h] for h in helds] if P <= 2 else None,
                "local_topk_ms_max_rank": max(local_ms), "local_topk_ms_per_rank": [round(v, 4) for v in local_ms],
                "local_topk_max_over_min": max(local_ms) / min(local_ms),
                "merge_ms": sorted(tm)[len(tm) // 2], "local_lse_ms_max_rank": max(lse_ms),
                "local_lse_max_over_min": max(lse_ms) / min(lse_ms),
                "lse_combine_ms": sorted(tc)[len(tc) // 2],
                "gather_bytes_per_rank": rows * w.topk * 8 + rows * 8,
                "blocks_equal_single_device": bool(torch.equal(blocks, ref_blocks)),
                "lse_max_abs_diff": float((lse - ref_lse).abs().max())}
            del keys, cands, cs, ci, mls, ml_all
    del x, flush, ws, ws_l
    torch.cuda.empty_cache()
    return res


def bench_train(args, world, rank, msa, pk):
    w = WORKLOADS["train_64k"]
    dev = torch.device("cuda", torch.cuda.current_device())
    N = args.train_n or w.N
    x = prefill_inputs(w, device=dev, seed=rank_seed(w, rank), N=N)
    dims = msa.MsaDims(w.B, N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    ws_i = msa.workspace(msa.MSA_OP_INDEX_TOPK_LSE, dims, dev)
    ws_a = msa.workspace(msa.MSA_OP_ATTN_FWD, dims, dev)
    ws_k = msa.workspace(msa.MSA_OP_KL, dims, dev)
    ws_b = msa.workspace(msa.MSA_OP_ATTN_BWD, dims, dev)
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    # upstream gradient of the layer output: synthetic N(0,1), drawn once
    gen = torch.Generator(device=dev)
    gen.manual_seed(rank_seed(w, rank) + 17)
    dout = torch.randn(w.B, N, w.H_q, w.d, generator=gen, device=dev).to(torch.bfloat16)

    def step():
        # index branch (selection, LSE_idx), main forward, main backward, KL of the index branch
        blocks, lse_idx = msa.msa_index_topk(dims, x["q_idx"], x["k_idx"], want_lse=True, ws=ws_i)
        out, lse = msa.msa_sparse_attn_fwd(dims, x["q"], x["k"], x["v"], blocks, ws=ws_a)
        gq, gk, gv = msa.msa_sparse_attn_bwd(dims, x["q"], x["k"], x["v"], blocks, out, lse, dout, ws=ws_b)
        loss, dq, dk = msa.msa_kl_fwd_grad(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], blocks, lse, lse_idx,
                                           ws=ws_k)
        return blocks, loss

    for _ in range(2):
        blocks, loss = step()
    torch.cuda.synchronize()
    sel_tok = selected_tokens(blocks, w.block_k)
    G = w.H_q // w.H_kv
    kl_flops = (2.0 * w.d * G + 6.0 * w.d_idx) * sel_tok
    bwd_flops = 10.0 * w.d * G * sel_tok  # S, dP, dV, dK, dQ: 2 d FLOPs each per selected (head, token) pair
    msa.msa_profile_read()
    msa.msa_profile_enable(True)
    t = timed_steps(step, args.train_steps, flush)
    msa.msa_profile_enable(False)
    prof = profile_avg(msa.msa_profile_read())
    ms = max_over_ranks(sum(t) / len(t), world)
    kl_ms = prof["kl_kv_outer"]["avg_ms"]
    bwd_ms = prof["attn_bwd"]["avg_ms"]
    res = {"workload": "train_64k" if N == w.N else f"train_{N}", "ms_per_step": ms, "loss": float(loss.item()),
           "roofline": {**roofline_entry("tensor", kl_flops / (kl_ms * 1e-3) / 1e12, pk["bf16_tflops"], "TFLOP/s",
                                         measured_traffic("kl_kv_outer", sel_tok)),
                        "kernel": "kl_kv_outer", "flops_per_launch": kl_flops},
           "roofline_attn_bwd": {**roofline_entry("tensor", bwd_flops / (bwd_ms * 1e-3) / 1e12, pk["bf16_tflops"],
                                                  "TFLOP/s", measured_traffic("attn_bwd", sel_tok)),
                                 "kernel": "attn_bwd", "flops_per_launch": bwd_flops},
           "work": {"selected_tokens": sel_tok, "kl_flops": kl_flops, "attn_bwd_flops": bwd_flops},
           "kernels": {k: {"avg_ms": round(v["avg_ms"], 4), "launches": v["launches"]} for k, v in prof.items()}}
    del ws_a, ws_k, ws_b, dout
    torch.cuda.empty_cache()
    res["dense_warmup"] = bench_dense_warmup(args, world, x, w, N, msa, pk, flush)
    del x
    torch.cuda.empty_cache()
    return res


def bench_dense_warmup(args, world, x, w, N, msa, pk, flush):
    """The dense warm-up KL (every causal block selected: teacher LSE over all keys, LSE_idx, KL and
    index gradients) on the training workload's inputs, with its tensor roofline."""
    dims = msa.MsaDims(w.B, N, w.H_q, w.H_kv, w.d, w.d_idx, w.block_k, w.topk)
    dev = x["q"].device
    ws = msa.workspace(msa.MSA_OP_KL_DENSE, dims, dev)

    def step():
        return msa.msa_kl_dense_fwd_grad(dims, x["q"], x["k"], x["q_idx"], x["k_idx"], ws=ws)

    loss, _, _ = step()
    torch.cuda.synchronize()
    G = w.H_q // w.H_kv
    pairs = w.B * w.H_kv * N * (N + 1) / 2  # causal (row, group, token) triples
    fl = {"teacher_lse": 2.0 * w.d * G * pairs, "lse_idx": 2.0 * w.d_idx * pairs,
          "kl": (2.0 * w.d * G + 6.0 * w.d_idx) * pairs}
    msa.msa_profile_read()
    msa.msa_profile_enable(True)
    t = timed_steps(step, 2, flush)
    msa.msa_profile_enable(False)
    prof = profile_avg(msa.msa_profile_read())
    ms = max_over_ranks(sum(t) / len(t), world)
    total = sum(fl.values())
    tf = total / (ms * 1e-3) / 1e12
    kern = {k: {"avg_ms": v["avg_ms"], "launches": v["launches"]} for k, v in prof.items()}
    for k, f in (("dense_lse", fl["teacher_lse"]), ("lse_idx", fl["lse_idx"]), ("kl_kv_outer", fl["kl"])):
        if k in kern:
            kern[k]["tflops"] = f / (kern[k]["avg_ms"] * 1e-3) / 1e12
    del ws
    torch.cuda.empty_cache()
    return {"workload": "train_64k" if N == w.N else f"train_{N}", "ms_per_step": ms, "loss": float(loss.item()),
            "flops": fl,
            "roofline": {**roofline_entry("tensor", tf, pk["bf16_tflops_sustained"], "TFLOP/s"),
                         "peak_source": f"{pk['source']} bf16 sustained (a step of this length runs under the "
                                        f"power cap)", "frac_of_burst": tf / pk["bf16_tflops"]},
            "kernels": kern}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=30)
    ap.add_argument("--train-steps", type=int, default=3)
    ap.add_argument("--cpu-rows", type=int, default=4096)
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workload", default=HEADLINE, choices=["prefill_8k", "prefill_32k_needles", "train_64k"],
                    help="prefill workload of the headline step (smaller ones serve profiler captures)")
    ap.add_argument("--only", choices=["decode", "train", "sp"], default=None,
                    help="profiler captures: run only this secondary measurement and print its object")
    ap.add_argument("--decode-len", type=int, default=0, help="profiler captures: decode cache length")
    ap.add_argument("--train-n", type=int, default=0, help="profiler captures: training sequence length")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        world, rank = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    world, rank, local = dist_setup(args.gpus)
    import block_sparse_attention_idx_b200 as msa
    pk = peaks()
    if args.only:
        res = {"decode": bench_decode, "train": bench_train, "sp": bench_sp}[args.only](args, world, rank, msa, pk)
        if world > 1:
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps({"only": args.only, args.only: res}), flush=True)
        return
    pre = bench_prefill(args, world, rank, msa, pk)
    w = WORKLOADS[args.workload]
    line = {"metric": METRIC, "value": pre["value"], "unit": "query-tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(w, world),
            "roofline": pre["roofline"], "e2e": pre["e2e"], "gpu_launches": pre["gpu_launches"],
            "clocks": pre["clocks"], "kernels": rnd(pre["kernels"]), "work": rnd(pre["work"]),
            "peaks": pk}
    if "cpu_baseline" in pre:
        line["cpu_baseline"] = pre["cpu_baseline"]
        line["parity"] = rnd(pre["parity"])
    if not args.no_secondary:
        # the decode object goes last: the end of the line is what a truncated log keeps
        dec = bench_decode(args, world, rank, msa, pk)
        line["train"] = rnd(bench_train(args, world, rank, msa, pk))
        line["sp_index"] = rnd(bench_sp(args, world, rank, msa, pk))
        line["decode"] = rnd(dec)
        # the decode step's figures once more, compactly, as the line's last key
        f8 = dec["fp8_index"]
        line["decode_summary"] = rnd({
            "bf16_us_per_step": dec["us_per_step"], "bf16_us_per_step_graph": dec["us_per_step_graph"],
            "bf16_step_frac_hbm": dec["step_roofline"]["frac"], "bf16_scan_frac_hbm": dec["roofline"]["frac"],
            "fp8_us_per_step": f8["us_per_step"], "fp8_us_per_step_graph": f8["us_per_step_graph"],
            "fp8_step_frac_hbm": f8["step_roofline"]["frac"], "fp8_scan_frac_hbm": f8["roofline"]["frac"]})
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
