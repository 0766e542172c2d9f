"""MSA oracle: plain float64 CPU definitions of the MiniMax Sparse Attention hot path.

TEST INFRASTRUCTURE ONLY. The product package never imports this module. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``
may import or call it.

The arithmetic lives in ``msa_oracle.c`` (float64, OpenMP over rows); this module builds it with
gcc and marshals arrays. Inputs may be bfloat16 (read bit-exactly and widened to float64) or
float64 (used by the finite-difference pins). ``metrics.py`` holds the host-side selection
metrics (recall@k, probability-mass coverage, output error).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")

F64, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, -O2, OpenMP, no fast-math) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("H_q", ctypes.c_int), ("H_kv", ctypes.c_int),
                ("d", ctypes.c_int), ("d_idx", ctypes.c_int), ("block_k", ctypes.c_int),
                ("topk", ctypes.c_int), ("local_mode", ctypes.c_int), ("scale", ctypes.c_double),
                ("scale_idx", ctypes.c_double)]


@dataclass
class Dims:
    """Problem sizes. scale / scale_idx of 0 mean 1/sqrt(d) and 1/sqrt(d_idx).

    local_mode selects the reading of the forced local block: 0 = Top-k over the complete past
    blocks plus the local block on top (the library's reading), 1 = the local block takes one of
    the k slots, 2 = Top-k over all blocks including the local one, then the local block added.
    """
    B: int
    N: int
    H_q: int
    H_kv: int
    d: int
    d_idx: int
    block_k: int
    topk: int
    local_mode: int = 0
    scale: float = 0.0
    scale_idx: float = 0.0

    def c(self) -> _Dims:
        return _Dims(self.B, self.N, self.H_q, self.H_kv, self.d, self.d_idx, self.block_k, self.topk,
                     self.local_mode, self.scale, self.scale_idx)


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        D = ctypes.POINTER(_Dims)
        i64 = ctypes.c_int64
        _lib.orc_index_scores_row.argtypes = [D, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        _lib.orc_block_max_row.argtypes = [D, P, ctypes.c_int, P]
        _lib.orc_select_from_max.argtypes = [D, P, ctypes.c_int, P, P]
        _lib.orc_index_topk.argtypes = [D, P, P, ctypes.c_int, P, i64, P, P, P]
        _lib.orc_sparse_attn.argtypes = [D, P, P, P, ctypes.c_int, P, P, i64, P, P]
        _lib.orc_attend_tokens.argtypes = [ctypes.c_int, ctypes.c_double, P, P, P, P, ctypes.c_int, P, P]
        _lib.orc_kl.argtypes = [D, P, P, P, P, ctypes.c_int, P, ctypes.c_double, P, i64, P, P, P, P]
        _lib.orc_decode.argtypes = [D, P, P, P, P, P, P, ctypes.c_int, P, P, P, P]
        _lib.orc_sparse_attn_bwd.argtypes = [D, P, P, P, P, ctypes.c_int, P, P, P, P]
        _lib.orc_sparse_attn_bwd_dq_rows.argtypes = [D, P, P, P, P, ctypes.c_int, P, P, i64, P]
        _lib.orc_e4m3_values.argtypes = [P, i64, P]
        _lib.orc_e4m3_round_many.argtypes = [P, i64, P]
        _lib.orc_quantize_e4m3_rows.argtypes = [P, i64, ctypes.c_int, P, P]
        _lib.orc_num_threads.restype = ctypes.c_int
    return _lib


def num_threads() -> int:
    return lib().orc_num_threads()


def e4m3_values(codes) -> np.ndarray:
    """float64 values of e4m3 codes (uint8 bit patterns), from the format's definition."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(c.shape, dtype=np.float64)
    lib().orc_e4m3_values(c.ctypes.data, c.size, out.ctypes.data)
    return out


def e4m3_round(y) -> np.ndarray:
    """e4m3 codes of float32 values: nearest value, ties to even, saturated to +-448."""
    f = np.ascontiguousarray(np.asarray(y, dtype=np.float32))
    out = np.empty(f.shape, dtype=np.uint8)
    lib().orc_e4m3_round_many(f.ctypes.data, f.size, out.ctypes.data)
    return out


def quantize_e4m3_rows(x):
    """Row-wise e4m3 quantisation of a bf16 tensor [..., n]: (codes uint8 [..., n], scale float32
    [...]) with scale = max|row| / 448 and codes = e4m3(x / scale), quotients in float32."""
    t = torch.as_tensor(x).detach().to("cpu").contiguous()
    if t.dtype != torch.bfloat16:
        raise TypeError("quantize_e4m3_rows takes bfloat16")
    n = t.shape[-1]
    rows = t.numel() // n
    codes = np.empty(tuple(t.shape), dtype=np.uint8)
    scale = np.empty(tuple(t.shape[:-1]), dtype=np.float32)
    lib().orc_quantize_e4m3_rows(_ptr(t.view(torch.int16)), rows, n, codes.ctypes.data, scale.ctypes.data)
    return codes, scale


def dequantize_e4m3_rows(codes, scale) -> torch.Tensor:
    """float64 values scale[r] * e4m3(codes[r, c])."""
    v = e4m3_values(codes) * np.asarray(scale, dtype=np.float64)[..., None]
    return torch.from_numpy(v)


def _inp(*ts):
    """Contiguous CPU views of the inputs and their common element-type code."""
    outs, ty = [], None
    for t in ts:
        if isinstance(t, np.ndarray):
            t = torch.from_numpy(t)
        t = t.detach().to("cpu").contiguous()
        if t.dtype == torch.bfloat16:
            code, t = BF16, t.view(torch.int16)
        elif t.dtype == torch.float64:
            code = F64
        else:
            raise TypeError(f"oracle inputs must be bfloat16 or float64, got {t.dtype}")
        if ty is None:
            ty = code
        elif ty != code:
            raise TypeError("all oracle inputs of one call must share a dtype")
        outs.append(t)
    return outs, ty


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


def _rows(rows):
    if rows is None:
        return None, 0
    r = torch.as_tensor(rows, dtype=torch.int64).contiguous()
    return r, r.numel()


def index_scores_row(dims: Dims, q_idx, k_idx, b: int, i: int, r: int) -> np.ndarray:
    (q, k), ty = _inp(q_idx, k_idx)
    s = np.zeros(i + 1, dtype=np.float64)
    lib().orc_index_scores_row(ctypes.byref(dims.c()), _ptr(q), _ptr(k), ty, b, i, r, s.ctypes.data)
    return s


def block_max_row(dims: Dims, s: np.ndarray, i: int) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float64)
    M = np.zeros(i // dims.block_k + 1, dtype=np.float64)
    lib().orc_block_max_row(ctypes.byref(dims.c()), s.ctypes.data, i, M.ctypes.data)
    return M


def select_from_max(dims: Dims, M: np.ndarray, i: int):
    M = np.ascontiguousarray(M, dtype=np.float64)
    sel = np.zeros(dims.topk + 1, dtype=np.int32)
    margin = np.zeros(1, dtype=np.float64)
    n = lib().orc_select_from_max(ctypes.byref(dims.c()), M.ctypes.data, i, sel.ctypes.data, margin.ctypes.data)
    return sel, float(margin[0]), n


def index_topk(dims: Dims, q_idx, k_idx, rows=None, want_lse: bool = False):
    """Selected blocks [nrows, H_kv, topk+1] (ascending, -1 padded), cutoff margins [nrows, H_kv],
    and optionally LSE_idx [nrows, H_kv] over the selected causal token set."""
    (q, k), ty = _inp(q_idx, k_idx)
    rt, nrows = _rows(rows)
    if rt is None:
        nrows = dims.B * dims.N
    blocks = np.zeros((nrows, dims.H_kv, dims.topk + 1), dtype=np.int32)
    margin = np.zeros((nrows, dims.H_kv), dtype=np.float64)
    lse = np.zeros((nrows, dims.H_kv), dtype=np.float64) if want_lse else None
    lib().orc_index_topk(ctypes.byref(dims.c()), _ptr(q), _ptr(k), ty, _ptr(rt) if rt is not None else None,
                         nrows, blocks.ctypes.data, margin.ctypes.data, lse.ctypes.data if want_lse else None)
    return blocks, margin, lse


def _full_blocks(dims: Dims, blocks) -> torch.Tensor:
    b = torch.as_tensor(blocks, dtype=torch.int32).contiguous()
    if b.numel() != dims.B * dims.N * dims.H_kv * (dims.topk + 1):
        raise ValueError("blocks must cover every (b, i, group): [B, N, H_kv, topk+1]")
    return b


def sparse_attn(dims: Dims, q, k, v, blocks, rows=None):
    """Output [nrows, H_q, d] and LSE [nrows, H_q] of exact attention over the selected tokens."""
    (qt, kt, vt), ty = _inp(q, k, v)
    bt = _full_blocks(dims, blocks)
    rt, nrows = _rows(rows)
    if rt is None:
        nrows = dims.B * dims.N
    out = np.zeros((nrows, dims.H_q, dims.d), dtype=np.float64)
    lse = np.zeros((nrows, dims.H_q), dtype=np.float64)
    lib().orc_sparse_attn(ctypes.byref(dims.c()), _ptr(qt), _ptr(kt), _ptr(vt), ty, _ptr(bt),
                          _ptr(rt) if rt is not None else None, nrows, out.ctypes.data, lse.ctypes.data)
    return out, lse


def sparse_attn_bwd(dims: Dims, q, k, v, blocks, dout):
    """Gradients of sum(dout * o) of the sparse attention with the selection fixed: (dq [B,N,H_q,d],
    dk [B,N,H_kv,d], dv [B,N,H_kv,d]) in float64."""
    (qt, kt, vt, gt), ty = _inp(q, k, v, dout)
    bl = _full_blocks(dims, blocks)
    dq = np.zeros((dims.B, dims.N, dims.H_q, dims.d), dtype=np.float64)
    dk = np.zeros((dims.B, dims.N, dims.H_kv, dims.d), dtype=np.float64)
    dv = np.zeros((dims.B, dims.N, dims.H_kv, dims.d), dtype=np.float64)
    lib().orc_sparse_attn_bwd(ctypes.byref(dims.c()), _ptr(qt), _ptr(kt), _ptr(vt), _ptr(gt), ty, _ptr(bl),
                              dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
    return dq, dk, dv


def sparse_attn_bwd_dq_rows(dims: Dims, q, k, v, blocks, dout, rows):
    """dq [nrows, H_q, d] of the given rows (flat b*N + i) only; same definition as sparse_attn_bwd."""
    (qt, kt, vt, gt), ty = _inp(q, k, v, dout)
    bl = _full_blocks(dims, blocks)
    rt, nrows = _rows(rows)
    dq = np.zeros((nrows, dims.H_q, dims.d), dtype=np.float64)
    lib().orc_sparse_attn_bwd_dq_rows(ctypes.byref(dims.c()), _ptr(qt), _ptr(kt), _ptr(vt), _ptr(gt), ty, _ptr(bl),
                                      _ptr(rt), nrows, dq.ctypes.data)
    return dq


def attend_tokens(q: np.ndarray, k: np.ndarray, v: np.ndarray, J, scale: float):
    """Attention of one query vector over the listed rows of k / v (all float64)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    J = np.ascontiguousarray(J, dtype=np.int32)
    d = q.shape[-1]
    o = np.zeros(d, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    lib().orc_attend_tokens(d, scale, q.ctypes.data, k.ctypes.data, v.ctypes.data, J.ctypes.data, len(J),
                            o.ctypes.data, lse.ctypes.data)
    return o, float(lse[0])


def kl(dims: Dims, q, k, q_idx, k_idx, blocks, grad_scale: float = 1.0, rows=None):
    """KL alignment: (loss, kl_rows [nrows,H_kv], dq_idx [nrows,H_kv,d_idx], dk_idx [B,N,d_idx]).
    With rows=None the loss and dk_idx are the full-layer values."""
    (qt, kt, qit, kit), ty = _inp(q, k, q_idx, k_idx)
    bt = _full_blocks(dims, blocks)
    rt, nrows = _rows(rows)
    if rt is None:
        nrows = dims.B * dims.N
    kl_rows = np.zeros((nrows, dims.H_kv), dtype=np.float64)
    dq = np.zeros((nrows, dims.H_kv, dims.d_idx), dtype=np.float64)
    dk = np.zeros((dims.B, dims.N, dims.d_idx), dtype=np.float64)
    loss = np.zeros(1, dtype=np.float64)
    lib().orc_kl(ctypes.byref(dims.c()), _ptr(qt), _ptr(kt), _ptr(qit), _ptr(kit), ty, _ptr(bt), grad_scale,
                 _ptr(rt) if rt is not None else None, nrows, kl_rows.ctypes.data, dq.ctypes.data,
                 dk.ctypes.data, loss.ctypes.data)
    return float(loss[0]), kl_rows, dq, dk


def decode(dims: Dims, cache_len, q, q_idx, k_cache, v_cache, k_idx_cache):
    """One decode step over caches of capacity dims.N: (blocks [B,H_kv,topk+1], margin [B,H_kv],
    out [B,H_q,d], lse [B,H_q])."""
    (qt, qit, kc, vc, kic), ty = _inp(q, q_idx, k_cache, v_cache, k_idx_cache)
    cl = torch.as_tensor(cache_len, dtype=torch.int32).contiguous()
    blocks = np.full((dims.B, dims.H_kv, dims.topk + 1), -1, dtype=np.int32)
    margin = np.zeros((dims.B, dims.H_kv), dtype=np.float64)
    out = np.zeros((dims.B, dims.H_q, dims.d), dtype=np.float64)
    lse = np.zeros((dims.B, dims.H_q), dtype=np.float64)
    lib().orc_decode(ctypes.byref(dims.c()), _ptr(cl), _ptr(qt), _ptr(qit), _ptr(kc), _ptr(vc), _ptr(kic), ty,
                     blocks.ctypes.data, margin.ctypes.data, out.ctypes.data, lse.ctypes.data)
    return blocks, margin, out, lse


def decode_fp8idx(dims: Dims, cache_len, q, q_idx, k_cache, v_cache, k_idx_codes, k_idx_scale):
    """One decode step with FP8 index scoring: the K_idx cache given as e4m3 codes [B,N,d_idx] and
    per-token scales [B,N]; Q_idx (bf16) rounded to e4m3 per (sequence, group) row by the same rule.
    The step is ``decode`` on the dequantised index vectors scale * e4m3(code) (exact in float64),
    so the index score is scale_idx * sq * sk * sum_c q8[c] k8[c]. Same returns as ``decode``."""
    qc, qs = quantize_e4m3_rows(q_idx)
    qd = dequantize_e4m3_rows(qc, qs)
    kd = dequantize_e4m3_rows(k_idx_codes, k_idx_scale)
    f64 = lambda t: torch.as_tensor(t).detach().to("cpu").to(torch.float64)
    return decode(dims, cache_len, f64(q), qd, f64(k_cache), f64(v_cache), kd)
