"""Python binding of libmsa, the B200 (sm_100a) MiniMax Sparse Attention hot path.

Thin ctypes marshalling over the C ABI in include/msa.h: every function here only checks shapes,
allocates outputs / workspace through PyTorch and calls the same-named C entry point on the
current CUDA stream. All arithmetic runs in the library's CUDA kernels; there is no other path.
Importing works without a GPU (the library loads without one); calling needs a CUDA device.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmsa.so")

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_WORKSPACE, MSA_ERR_CUDA, MSA_ERR_TIMEOUT, \
    MSA_ERR_DEVICE_CHECK = range(7)
(MSA_OP_INDEX_TOPK, MSA_OP_INDEX_TOPK_LSE, MSA_OP_ATTN_FWD, MSA_OP_DECODE, MSA_OP_KL, MSA_OP_ATTN_BWD,
 MSA_OP_LSE_IDX_LOCAL, MSA_OP_KL_DENSE) = range(8)


class MsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {msa_status_string(code)} ({code})")
        self.code = code


class _Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("H_q", ctypes.c_int), ("H_kv", ctypes.c_int),
                ("d", ctypes.c_int), ("d_idx", ctypes.c_int), ("block_k", ctypes.c_int), ("topk", ctypes.c_int),
                ("scale", ctypes.c_float), ("scale_idx", ctypes.c_float)]


class _KeyRanges(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("tok0", ctypes.c_int32 * 2), ("ntok", ctypes.c_int32 * 2)]


def _held(held, k_idx_local) -> _KeyRanges:
    """msa_key_ranges from a list of one or two (tok0, ntok) ranges, or from a single first token
    (one range spanning k_idx_local); the tokens must add up to k_idx_local's length."""
    rng = [(int(held), int(k_idx_local.shape[1]))] if isinstance(held, int) else [(int(a), int(n)) for a, n in held]
    if not 1 <= len(rng) <= 2 or sum(n for _, n in rng) != k_idx_local.shape[1]:
        raise ValueError(f"held ranges {rng} do not describe k_idx_local of {k_idx_local.shape[1]} tokens")
    h = _KeyRanges()
    h.n = len(rng)
    for x, (a, n) in enumerate(rng):
        h.tok0[x], h.ntok[x] = a, n
    return h


@dataclass
class MsaDims:
    """msa_dims: B sequences of N tokens (cache capacity for decode), H_q / H_kv heads, head dim d,
    index dim d_idx, KV block size block_k, topk past blocks per (query, group).
    scale / scale_idx of 0 mean 1/sqrt(d) and 1/sqrt(d_idx)."""
    B: int
    N: int
    H_q: int
    H_kv: int
    d: int
    d_idx: int
    block_k: int
    topk: int
    scale: float = 0.0
    scale_idx: float = 0.0

    def c(self) -> _Dims:
        return _Dims(self.B, self.N, self.H_q, self.H_kv, self.d, self.d_idx, self.block_k, self.topk,
                     self.scale, self.scale_idx)


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmsa.so; raises if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmsa.so not found at {LIB_PATH}; build it with "
                               "`python -m block_sparse_attention_idx_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, D, S = ctypes.c_void_p, ctypes.POINTER(_Dims), ctypes.c_size_t
        L.msa_workspace_size.argtypes = [ctypes.c_int, D, ctypes.POINTER(ctypes.c_size_t)]
        L.msa_index_topk.argtypes = [D, P, P, P, P, P, S, P]
        L.msa_sparse_attn_fwd.argtypes = [D, P, P, P, P, P, P, P, S, P]
        L.msa_sparse_attn_fwd_bf16.argtypes = [D, P, P, P, P, P, P, P, S, P]
        L.msa_sparse_attn_decode.argtypes = [D, P, P, P, P, P, P, P, P, P, P, S, P]
        L.msa_sparse_attn_decode_fp8idx.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, S, P]
        L.msa_quantize_e4m3_rows.argtypes = [P, ctypes.c_int64, ctypes.c_int, P, P, P]
        L.msa_kl_fwd_grad.argtypes = [D, P, P, P, P, P, P, P, ctypes.c_float, P, P, P, P, S, P]
        L.msa_kl_dense_fwd_grad.argtypes = [D, P, P, P, P, ctypes.c_float, P, P, P, P, P, S, P]
        L.msa_sparse_attn_bwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, S, P]
        I = ctypes.c_int
        H = ctypes.POINTER(_KeyRanges)
        L.msa_index_topk_local.argtypes = [D, P, P, H, P, P, P, S, P]
        L.msa_topk_merge.argtypes = [D, I, P, P, P, P]
        L.msa_lse_idx_local.argtypes = [D, P, P, H, P, P, P, S, P]
        L.msa_lse_combine.argtypes = [D, I, P, P, P]
        L.msa_sparse_attn_decode_noalloc.argtypes = [D, P, P, P, P, P, P, P, P, P]
        L.msa_sparse_attn_decode_noalloc.restype = ctypes.c_int
        L.msa_get_device_status.argtypes = [P, P]
        L.msa_decode_noalloc_status.argtypes = [P]
        L.msa_decode_noalloc_status.restype = ctypes.c_int
        L.msa_debug_set_wait_ns.argtypes = [ctypes.c_ulonglong]
        L.msa_debug_set_wait_ns.restype = None
        L.msa_debug_wait_probe.argtypes = [P, S, P]
        L.msa_debug_wait_probe.restype = ctypes.c_int
        L.msa_debug_exp2_fma.argtypes = [P, P, ctypes.c_int64, P]
        L.msa_debug_exp2_fma.restype = ctypes.c_int
        L.msa_profile_enable.argtypes = [ctypes.c_int]
        L.msa_profile_enable.restype = None
        L.msa_profile_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int), ctypes.c_int]
        L.msa_profile_read.restype = ctypes.c_int
        L.msa_status_string.argtypes = [ctypes.c_int]
        L.msa_status_string.restype = ctypes.c_char_p
        L.msa_version.restype = ctypes.c_char_p
        for fn in ("msa_workspace_size", "msa_index_topk", "msa_sparse_attn_fwd", "msa_sparse_attn_fwd_bf16",
                   "msa_sparse_attn_decode",
                   "msa_sparse_attn_decode_fp8idx", "msa_quantize_e4m3_rows", "msa_kl_fwd_grad",
                   "msa_sparse_attn_bwd", "msa_index_topk_local", "msa_topk_merge", "msa_lse_idx_local",
                   "msa_lse_combine", "msa_get_device_status", "msa_kl_dense_fwd_grad"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def msa_status_string(code: int) -> str:
    return lib().msa_status_string(code).decode()


def msa_version() -> str:
    return lib().msa_version().decode()


def _check(fn: str, code: int):
    if code != MSA_OK:
        raise MsaError(fn, code)


def msa_workspace_size(op: int, dims: MsaDims) -> int:
    n = ctypes.c_size_t(0)
    _check("msa_workspace_size", lib().msa_workspace_size(op, ctypes.byref(dims.c()), ctypes.byref(n)))
    return n.value


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, dev: torch.device):
    """The stream to launch on. The library launches on the current CUDA device, so the tensors'
    device must be the current one (and an explicit stream must belong to it)."""
    cur = torch.cuda.current_device()
    if dev.type != "cuda" or (dev.index is not None and dev.index != cur):
        raise ValueError(f"tensors are on {dev}, but the current CUDA device is cuda:{cur}; "
                         "call under torch.cuda.device(...)")
    s = torch.cuda.current_stream() if stream is None else stream
    if s.device.index != cur:
        raise ValueError(f"stream belongs to {s.device}, not to the current device cuda:{cur}")
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, shape, dtype, device):
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (the library takes device pointers), got {t.device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")


def workspace(op: int, dims: MsaDims, device) -> torch.Tensor:
    """A device workspace buffer of the size `op` needs (256-byte aligned by the allocator)."""
    return torch.empty(max(msa_workspace_size(op, dims), 256), dtype=torch.uint8, device=device)


def _ws(ws, op: int, dims: MsaDims, dev) -> torch.Tensor:
    """The caller's workspace, checked (a contiguous uint8 CUDA tensor on the inputs' device; the
    library checks its size and alignment), or a new one for `op`."""
    if ws is None:
        return workspace(op, dims, dev)
    if ws.dtype != torch.uint8 or not ws.is_contiguous() or ws.device != dev:
        raise ValueError(f"ws must be a contiguous uint8 tensor on {dev}")
    return ws


def msa_index_topk(dims: MsaDims, q_idx, k_idx, want_lse: bool = False, ws=None, stream=None):
    """Block selection. Returns blocks int32 [B,N,H_kv,topk+1] (and LSE_idx fp32 [B,N,H_kv])."""
    dev = q_idx.device
    _need(q_idx, "q_idx", (dims.B, dims.N, dims.H_kv, dims.d_idx), torch.bfloat16, dev)
    _need(k_idx, "k_idx", (dims.B, dims.N, dims.d_idx), torch.bfloat16, dev)
    blocks = torch.empty(dims.B, dims.N, dims.H_kv, dims.topk + 1, dtype=torch.int32, device=dev)
    lse = torch.empty(dims.B, dims.N, dims.H_kv, dtype=torch.float32, device=dev) if want_lse else None
    ws = _ws(ws, MSA_OP_INDEX_TOPK_LSE if want_lse else MSA_OP_INDEX_TOPK, dims, dev)
    _check("msa_index_topk", lib().msa_index_topk(ctypes.byref(dims.c()), _p(q_idx), _p(k_idx), _p(blocks), _p(lse),
                                                  _p(ws), ws.numel(), _stream(stream, dev)))
    return (blocks, lse) if want_lse else blocks


def msa_sparse_attn_fwd(dims: MsaDims, q, k, v, blocks, want_lse: bool = True, ws=None, stream=None,
                        out_dtype=torch.float32, out=None):
    """Sparse attention forward. Returns out [B,N,H_q,d] (fp32, or with out_dtype=torch.bfloat16 the
    same values rounded to bf16 by msa_sparse_attn_fwd_bf16) and LSE fp32 [B,N,H_q] (or None).
    `out` may be given (contiguous, of out_dtype) to be written in place."""
    dev = q.device
    _need(q, "q", (dims.B, dims.N, dims.H_q, dims.d), torch.bfloat16, dev)
    _need(k, "k", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(v, "v", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(blocks, "blocks", (dims.B, dims.N, dims.H_kv, dims.topk + 1), torch.int32, dev)
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError(f"out_dtype must be torch.float32 or torch.bfloat16, not {out_dtype}")
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=dev)
    _need(out, "out", tuple(q.shape), out_dtype, dev)
    lse = torch.empty(dims.B, dims.N, dims.H_q, dtype=torch.float32, device=dev) if want_lse else None
    ws = _ws(ws, MSA_OP_ATTN_FWD, dims, dev)
    fn = "msa_sparse_attn_fwd" if out_dtype == torch.float32 else "msa_sparse_attn_fwd_bf16"
    _check(fn, getattr(lib(), fn)(ctypes.byref(dims.c()), _p(q), _p(k), _p(v), _p(blocks), _p(out), _p(lse), _p(ws),
                                  ws.numel(), _stream(stream, dev)))
    return out, lse


def _decode_io(dims: MsaDims, cache_len, q, q_idx, k_cache, v_cache, want_blocks, want_margin):
    dev = q.device
    _need(cache_len, "cache_len", (dims.B,), torch.int32, dev)
    _need(q, "q", (dims.B, dims.H_q, dims.d), torch.bfloat16, dev)
    _need(q_idx, "q_idx", (dims.B, dims.H_kv, dims.d_idx), torch.bfloat16, dev)
    _need(k_cache, "k_cache", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(v_cache, "v_cache", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    blocks = torch.empty(dims.B, dims.H_kv, dims.topk + 1, dtype=torch.int32, device=dev) if want_blocks else None
    margin = torch.empty(dims.B, dims.H_kv, dtype=torch.float32, device=dev) if want_margin else None
    return out, blocks, margin


def msa_sparse_attn_decode(dims: MsaDims, cache_len, q, q_idx, k_cache, v_cache, k_idx_cache, want_blocks=True,
                           ws=None, stream=None, want_margin=False):
    """One decode step. dims.N is the cache capacity. Returns out fp32 [B,H_q,d] and the selected
    blocks int32 [B,H_kv,topk+1] (or None); with want_margin, also the cutoff margins fp32 [B,H_kv]."""
    out, blocks, margin = _decode_io(dims, cache_len, q, q_idx, k_cache, v_cache, want_blocks, want_margin)
    _need(k_idx_cache, "k_idx_cache", (dims.B, dims.N, dims.d_idx), torch.bfloat16, q.device)
    ws = _ws(ws, MSA_OP_DECODE, dims, q.device)
    _check("msa_sparse_attn_decode",
           lib().msa_sparse_attn_decode(ctypes.byref(dims.c()), _p(cache_len), _p(q), _p(q_idx), _p(k_cache),
                                        _p(v_cache), _p(k_idx_cache), _p(out), _p(blocks), _p(margin), _p(ws),
                                        ws.numel(), _stream(stream, q.device)))
    return (out, blocks, margin) if want_margin else (out, blocks)


def msa_quantize_e4m3_rows(x, codes=None, scale=None, stream=None):
    """Row-wise e4m3 quantisation of a bf16 tensor [..., n]: codes uint8 [..., n] (e4m3 bit
    patterns) and scales fp32 [...], scale = max|row| / 448."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    n = x.shape[-1]
    rows = x.numel() // n if n else 0
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _need(codes, "codes", tuple(x.shape), torch.uint8, x.device)
    _need(scale, "scale", tuple(x.shape[:-1]), torch.float32, x.device)
    _check("msa_quantize_e4m3_rows",
           lib().msa_quantize_e4m3_rows(_p(x), rows, n, _p(codes), _p(scale), _stream(stream, x.device)))
    return codes, scale


def msa_sparse_attn_decode_fp8idx(dims: MsaDims, cache_len, q, q_idx, k_cache, v_cache, k_idx_codes, k_idx_scale,
                                  want_blocks=True, ws=None, stream=None, want_margin=False):
    """Decode step with FP8 index scoring: the K_idx cache as e4m3 codes uint8 [B,N,d_idx] plus
    per-token scales fp32 [B,N] (msa_quantize_e4m3_rows). Returns as msa_sparse_attn_decode."""
    out, blocks, margin = _decode_io(dims, cache_len, q, q_idx, k_cache, v_cache, want_blocks, want_margin)
    _need(k_idx_codes, "k_idx_codes", (dims.B, dims.N, dims.d_idx), torch.uint8, q.device)
    _need(k_idx_scale, "k_idx_scale", (dims.B, dims.N), torch.float32, q.device)
    ws = _ws(ws, MSA_OP_DECODE, dims, q.device)
    _check("msa_sparse_attn_decode_fp8idx",
           lib().msa_sparse_attn_decode_fp8idx(ctypes.byref(dims.c()), _p(cache_len), _p(q), _p(q_idx),
                                               _p(k_cache), _p(v_cache), _p(k_idx_codes), _p(k_idx_scale),
                                               _p(out), _p(blocks), _p(margin), _p(ws), ws.numel(),
                                               _stream(stream, q.device)))
    return (out, blocks, margin) if want_margin else (out, blocks)


def msa_sparse_attn_decode_noalloc(dims: MsaDims, cache_len, q, q_idx, k_cache, v_cache, k_idx_cache, out=None,
                                   blocks=None, stream=None):
    """Decode step through the allocation-free entry point (the library's static 16 MiB device scratch
    instead of a workspace). For callers that cannot allocate device memory while decoding; outputs may
    be passed in preallocated. Calls on one device share the scratch and must not overlap on the GPU."""
    dev = q.device
    _need(cache_len, "cache_len", (dims.B,), torch.int32, dev)
    _need(q, "q", (dims.B, dims.H_q, dims.d), torch.bfloat16, dev)
    _need(q_idx, "q_idx", (dims.B, dims.H_kv, dims.d_idx), torch.bfloat16, dev)
    _need(k_cache, "k_cache", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(v_cache, "v_cache", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(k_idx_cache, "k_idx_cache", (dims.B, dims.N, dims.d_idx), torch.bfloat16, dev)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    _need(out, "out", (dims.B, dims.H_q, dims.d), torch.float32, dev)
    if blocks is not None:
        _need(blocks, "blocks", (dims.B, dims.H_kv, dims.topk + 1), torch.int32, dev)
    _check("msa_sparse_attn_decode_noalloc",
           lib().msa_sparse_attn_decode_noalloc(ctypes.byref(dims.c()), _p(cache_len), _p(q), _p(q_idx),
                                                _p(k_cache), _p(v_cache), _p(k_idx_cache), _p(out), _p(blocks),
                                                _stream(stream, dev)))
    return out, blocks


def msa_sparse_attn_bwd(dims: MsaDims, q, k, v, blocks, out, lse, dout, ws=None, stream=None):
    """Backward of the sparse attention with the selection fixed. out / lse are the forward's
    (fp32), dout bf16 [B,N,H_q,d]. Returns dq fp32 [B,N,H_q,d], dk and dv fp32 [B,N,H_kv,d]."""
    dev = q.device
    _need(q, "q", (dims.B, dims.N, dims.H_q, dims.d), torch.bfloat16, dev)
    _need(k, "k", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(v, "v", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(blocks, "blocks", (dims.B, dims.N, dims.H_kv, dims.topk + 1), torch.int32, dev)
    _need(out, "out", (dims.B, dims.N, dims.H_q, dims.d), torch.float32, dev)
    _need(lse, "lse", (dims.B, dims.N, dims.H_q), torch.float32, dev)
    _need(dout, "dout", (dims.B, dims.N, dims.H_q, dims.d), torch.bfloat16, dev)
    dq = torch.empty(dims.B, dims.N, dims.H_q, dims.d, dtype=torch.float32, device=dev)
    dk = torch.empty(dims.B, dims.N, dims.H_kv, dims.d, dtype=torch.float32, device=dev)
    dv = torch.empty(dims.B, dims.N, dims.H_kv, dims.d, dtype=torch.float32, device=dev)
    ws = _ws(ws, MSA_OP_ATTN_BWD, dims, dev)
    _check("msa_sparse_attn_bwd",
           lib().msa_sparse_attn_bwd(ctypes.byref(dims.c()), _p(q), _p(k), _p(v), _p(blocks), _p(out), _p(lse),
                                     _p(dout), _p(dq), _p(dk), _p(dv), _p(ws), ws.numel(), _stream(stream, dev)))
    return dq, dk, dv


def msa_index_topk_local(dims: MsaDims, q_idx, k_idx_local, held, ws=None, stream=None):
    """This rank's candidates for the sequence-parallel selection: k_idx_local bf16 [B, ntok, d_idx]
    holds the tokens of `held`, one or two (tok0, ntok) ranges in order (or a single tok0: one range
    of ntok tokens). Returns (raw block maxima fp32, block ids int32), each [B, N, H_kv, topk], best
    first, -inf / -1 padded."""
    dev = q_idx.device
    _need(q_idx, "q_idx", (dims.B, dims.N, dims.H_kv, dims.d_idx), torch.bfloat16, dev)
    ntok = k_idx_local.shape[1]
    _need(k_idx_local, "k_idx_local", (dims.B, ntok, dims.d_idx), torch.bfloat16, dev)
    h = _held(held, k_idx_local)
    cs = torch.empty(dims.B, dims.N, dims.H_kv, dims.topk, dtype=torch.float32, device=dev)
    ci = torch.empty(dims.B, dims.N, dims.H_kv, dims.topk, dtype=torch.int32, device=dev)
    ws = _ws(ws, MSA_OP_INDEX_TOPK, dims, dev)
    _check("msa_index_topk_local",
           lib().msa_index_topk_local(ctypes.byref(dims.c()), _p(q_idx), _p(k_idx_local), ctypes.byref(h), _p(cs),
                                      _p(ci), _p(ws), ws.numel(), _stream(stream, dev)))
    return cs, ci


def msa_topk_merge(dims: MsaDims, cand_scores, cand_ids, stream=None):
    """Merge of P ranks' candidates [P, B, N, H_kv, topk] into blocks int32 [B, N, H_kv, topk+1]."""
    P = cand_scores.shape[0]
    dev = cand_scores.device
    _need(cand_scores, "cand_scores", (P, dims.B, dims.N, dims.H_kv, dims.topk), torch.float32, dev)
    _need(cand_ids, "cand_ids", (P, dims.B, dims.N, dims.H_kv, dims.topk), torch.int32, dev)
    blocks = torch.empty(dims.B, dims.N, dims.H_kv, dims.topk + 1, dtype=torch.int32, device=dev)
    _check("msa_topk_merge", lib().msa_topk_merge(ctypes.byref(dims.c()), P, _p(cand_scores), _p(cand_ids), _p(blocks),
                                                  _stream(stream, dev)))
    return blocks


def msa_lse_idx_local(dims: MsaDims, q_idx, k_idx_local, held, blocks, ws=None, stream=None):
    """This rank's (max, exp-sum) of the index scores over the selected tokens it holds (`held` as in
    msa_index_topk_local): fp32 [B, N, H_kv, 2]."""
    dev = q_idx.device
    ntok = k_idx_local.shape[1]
    _need(q_idx, "q_idx", (dims.B, dims.N, dims.H_kv, dims.d_idx), torch.bfloat16, dev)
    _need(k_idx_local, "k_idx_local", (dims.B, ntok, dims.d_idx), torch.bfloat16, dev)
    _need(blocks, "blocks", (dims.B, dims.N, dims.H_kv, dims.topk + 1), torch.int32, dev)
    h = _held(held, k_idx_local)
    ml = torch.empty(dims.B, dims.N, dims.H_kv, 2, dtype=torch.float32, device=dev)
    ws = _ws(ws, MSA_OP_LSE_IDX_LOCAL, dims, dev)
    _check("msa_lse_idx_local",
           lib().msa_lse_idx_local(ctypes.byref(dims.c()), _p(q_idx), _p(k_idx_local), ctypes.byref(h), _p(blocks),
                                   _p(ml), _p(ws), ws.numel(), _stream(stream, dev)))
    return ml


def msa_lse_combine(dims: MsaDims, ml, stream=None):
    """Eq (16) over the P ranks' pairs ml [P, B, N, H_kv, 2]: LSE_idx fp32 [B, N, H_kv]."""
    P = ml.shape[0]
    _need(ml, "ml", (P, dims.B, dims.N, dims.H_kv, 2), torch.float32, ml.device)
    lse = torch.empty(dims.B, dims.N, dims.H_kv, dtype=torch.float32, device=ml.device)
    _check("msa_lse_combine", lib().msa_lse_combine(ctypes.byref(dims.c()), P, _p(ml), _p(lse), _stream(stream, ml.device)))
    return lse


def msa_kl_fwd_grad(dims: MsaDims, q, k, q_idx, k_idx, blocks, lse, lse_idx=None, grad_scale: float = 1.0, ws=None,
                    stream=None):
    """KL alignment. Returns loss fp32 [1], dq_idx fp32 [B,N,H_kv,d_idx], dk_idx fp32 [B,N,d_idx]."""
    dev = q.device
    _need(q, "q", (dims.B, dims.N, dims.H_q, dims.d), torch.bfloat16, dev)
    _need(k, "k", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(q_idx, "q_idx", (dims.B, dims.N, dims.H_kv, dims.d_idx), torch.bfloat16, dev)
    _need(k_idx, "k_idx", (dims.B, dims.N, dims.d_idx), torch.bfloat16, dev)
    _need(blocks, "blocks", (dims.B, dims.N, dims.H_kv, dims.topk + 1), torch.int32, dev)
    _need(lse, "lse", (dims.B, dims.N, dims.H_q), torch.float32, dev)
    if lse_idx is not None:
        _need(lse_idx, "lse_idx", (dims.B, dims.N, dims.H_kv), torch.float32, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dq = torch.empty(dims.B, dims.N, dims.H_kv, dims.d_idx, dtype=torch.float32, device=dev)
    dk = torch.empty(dims.B, dims.N, dims.d_idx, dtype=torch.float32, device=dev)
    ws = _ws(ws, MSA_OP_KL, dims, dev)
    _check("msa_kl_fwd_grad",
           lib().msa_kl_fwd_grad(ctypes.byref(dims.c()), _p(q), _p(k), _p(q_idx), _p(k_idx), _p(blocks), _p(lse),
                                 _p(lse_idx), ctypes.c_float(grad_scale), _p(loss), _p(dq), _p(dk), _p(ws),
                                 ws.numel(), _stream(stream, dev)))
    return loss, dq, dk


def msa_kl_dense_fwd_grad(dims: MsaDims, q, k, q_idx, k_idx, grad_scale: float = 1.0, want_lse: bool = False,
                          ws=None, stream=None):
    """Dense warm-up KL (every causal block selected). Returns (loss fp32 [1], dq_idx [B,N,H_kv,d_idx],
    dk_idx [B,N,d_idx]) and, with want_lse, the teacher LSE fp32 [B,N,H_q]."""
    dev = q.device
    _need(q, "q", (dims.B, dims.N, dims.H_q, dims.d), torch.bfloat16, dev)
    _need(k, "k", (dims.B, dims.N, dims.H_kv, dims.d), torch.bfloat16, dev)
    _need(q_idx, "q_idx", (dims.B, dims.N, dims.H_kv, dims.d_idx), torch.bfloat16, dev)
    _need(k_idx, "k_idx", (dims.B, dims.N, dims.d_idx), torch.bfloat16, dev)
    ws = _ws(ws, MSA_OP_KL_DENSE, dims, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dq = torch.empty(dims.B, dims.N, dims.H_kv, dims.d_idx, dtype=torch.float32, device=dev)
    dk = torch.empty(dims.B, dims.N, dims.d_idx, dtype=torch.float32, device=dev)
    lse = torch.empty(dims.B, dims.N, dims.H_q, dtype=torch.float32, device=dev) if want_lse else None
    _check("msa_kl_dense_fwd_grad",
           lib().msa_kl_dense_fwd_grad(ctypes.byref(dims.c()), _p(q), _p(k), _p(q_idx), _p(k_idx),
                                       ctypes.c_float(grad_scale), _p(loss), _p(dq), _p(dk), _p(lse), _p(ws),
                                       ws.numel(), _stream(stream, dev)))
    return (loss, dq, dk, lse) if want_lse else (loss, dq, dk)


def msa_profile_enable(on: bool = True) -> None:
    """Record CUDA events around every kernel the library launches (on the launching stream)."""
    lib().msa_profile_enable(1 if on else 0)


def msa_profile_read() -> dict:
    """{kernel name: (total ms, launches)} since the last read; synchronises on the events."""
    cap = 64
    names = (ctypes.c_char_p * cap)()
    ms = (ctypes.c_double * cap)()
    n = (ctypes.c_int * cap)()
    k = lib().msa_profile_read(names, ms, n, cap)
    if k < 0:
        raise MsaError("msa_profile_read", MSA_ERR_CUDA)
    return {names[x].decode(): (ms[x], n[x]) for x in range(k)}


def msa_get_device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return the status code recorded by the last call using `ws`."""
    return lib().msa_get_device_status(_p(ws), _stream(stream, ws.device))


def msa_decode_noalloc_status(stream=None) -> int:
    """Synchronise the stream and return the status code of the last allocation-free decode call on
    the current device (its status word lives in the library's static scratch array)."""
    return lib().msa_decode_noalloc_status(_stream(stream, torch.device("cuda", torch.cuda.current_device())))


def msa_debug_set_wait_ns(ns: int) -> None:
    """Test hook: time limit (ns) of every bounded device wait of later calls (0: the 2 s default)."""
    lib().msa_debug_set_wait_ns(int(ns))


def msa_debug_exp2_fma(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x by the library's FMA-pipe exponential (fp32 device tensor in, same shape out)."""
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("msa_debug_exp2_fma: x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    _check("msa_debug_exp2_fma", lib().msa_debug_exp2_fma(_p(x), _p(y), x.numel(), _stream(stream, x.device)))
    return y


def msa_debug_wait_probe(ws: torch.Tensor, stream=None) -> None:
    """Test hook: enqueue the launch whose bounded wait can only run out (status MSA_ERR_TIMEOUT).
    ws: a uint8 CUDA tensor of at least 256 + 4096 bytes."""
    if ws.dtype != torch.uint8 or not ws.is_contiguous() or ws.device.type != "cuda":
        raise ValueError("ws must be a contiguous uint8 CUDA tensor")
    _check("msa_debug_wait_probe", lib().msa_debug_wait_probe(_p(ws), ws.numel(), _stream(stream, ws.device)))


__all__ = ["MsaDims", "MsaError", "msa_workspace_size", "msa_index_topk", "msa_sparse_attn_fwd",
           "msa_sparse_attn_decode", "msa_sparse_attn_decode_noalloc", "msa_sparse_attn_decode_fp8idx",
           "msa_quantize_e4m3_rows", "msa_kl_fwd_grad", "msa_sparse_attn_bwd", "msa_index_topk_local",
           "msa_topk_merge", "msa_lse_idx_local", "msa_lse_combine", "msa_get_device_status", "msa_status_string",
           "msa_version", "msa_profile_enable", "msa_profile_read", "msa_decode_noalloc_status",
           "msa_debug_set_wait_ns", "msa_debug_wait_probe", "msa_debug_exp2_fma", "msa_kl_dense_fwd_grad", "workspace", "lib",
           "LIB_PATH"]
