"""The allocation-free decode entry point (msa_sparse_attn_decode_noalloc).

It exists for callers that cannot allocate device memory where they decode (a plugin inside a host
application that owns every device allocation, a serving loop with a fixed memory budget, a path
that must not call cudaMalloc because it can synchronise the device): its scratch is a static
device array inside the library. These tests call it through the C ABI and check, on two calls in a
row, that it returns exactly what the workspace entry point returns (the same kernels run on the
same inputs), that its device status can be read back without allocating, and that sizes beyond its
fixed maximum are refused with a clear status. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import block_sparse_attention_idx_b200 as msa

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _decode_case(B, L, lens, seed, H_q=64, H_kv=4, d=128, d_idx=64, bk=128, k=16):
    g = torch.Generator(device=DEV).manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g, device=DEV).to(torch.bfloat16)
    x = dict(q=mk(B, H_q, d), q_idx=mk(B, H_kv, d_idx), k_cache=mk(B, L, H_kv, d), v_cache=mk(B, L, H_kv, d),
             k_idx_cache=mk(B, L, d_idx), cache_len=torch.tensor(lens, dtype=torch.int32, device=DEV))
    return msa.MsaDims(B, L, H_q, H_kv, d, d_idx, bk, k), x


def _noalloc_c(dims, x, out, blocks):
    """Direct C-ABI call of the allocation-free entry point on the current stream."""
    L = msa.lib()
    fn = L.msa_sparse_attn_decode_noalloc
    fn.argtypes = [ctypes.POINTER(type(dims.c()))] + [ctypes.c_void_p] * 9
    fn.restype = ctypes.c_int
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return fn(ctypes.byref(dims.c()), p(x["cache_len"]), p(x["q"]), p(x["q_idx"]), p(x["k_cache"]),
              p(x["v_cache"]), p(x["k_idx_cache"]), p(out), p(blocks),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    # a larger call first, then a smaller one that runs over the previous call's scratch contents
    cases = [_decode_case(4, 3000, [3000, 2999, 1537, 129], seed=5),
             _decode_case(2, 1500, [700, 1500], seed=6)]
    for dims, x in cases:
        ref_out, ref_blocks = msa.msa_sparse_attn_decode(dims, x["cache_len"], x["q"], x["q_idx"], x["k_cache"],
                                                         x["v_cache"], x["k_idx_cache"])
        out = torch.full_like(ref_out, float("nan"))
        blocks = torch.full_like(ref_blocks, -7)
        assert _noalloc_c(dims, x, out, blocks) == msa.MSA_OK
        # the call's device status, read from the static array without allocating
        assert msa.msa_decode_noalloc_status() == msa.MSA_OK
        # the same kernels on the same inputs: identical results, not merely close ones
        assert torch.equal(blocks, ref_blocks)
        assert torch.equal(out, ref_out)


def test_noalloc_refuses_sizes_beyond_its_static_scratch():
    dims = msa.MsaDims(32, 262144, 64, 4, 128, 64, 128, 16)  # valid sizes that need ~19 MiB of scratch
    assert msa.msa_workspace_size(msa.MSA_OP_DECODE, dims) > (16 << 20)
    t = torch.empty(16, dtype=torch.bfloat16, device=DEV)
    x = dict(cache_len=t, q=t, q_idx=t, k_cache=t, v_cache=t, k_idx_cache=t)
    assert _noalloc_c(dims, x, t, t) == msa.MSA_ERR_WORKSPACE
