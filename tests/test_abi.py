"""C-ABI checks that need no GPU: the library loads, exports every symbol include/msa.h declares,
sizes workspaces and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_idx_b200 as msa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "msa.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 8
    L = msa.lib()
    for s in syms:
        assert hasattr(L, s), s


def test_status_strings_and_version():
    assert msa.msa_status_string(0) == "MSA_OK"
    assert msa.msa_status_string(6) == "MSA_ERR_DEVICE_CHECK"
    assert msa.msa_version().startswith("msa-b200")


def dims(**kw):
    d = dict(B=1, N=512, H_q=4, H_kv=2, d=64, d_idx=32, block_k=32, topk=4)
    d.update(kw)
    return msa.MsaDims(**d)


def test_workspace_sizes():
    d = dims()
    assert msa.msa_workspace_size(msa.MSA_OP_INDEX_TOPK, d) == 256
    for op in (msa.MSA_OP_INDEX_TOPK_LSE, msa.MSA_OP_ATTN_FWD, msa.MSA_OP_DECODE, msa.MSA_OP_KL):
        assert msa.msa_workspace_size(op, d) > 256
    big = dims(N=32768, H_q=64, H_kv=4, d=128, d_idx=64, block_k=128, topk=16)
    # partials of every (query, head, slot): fp16 o (d values) and an fp32 lse dominate
    assert msa.msa_workspace_size(msa.MSA_OP_ATTN_FWD, big) >= 32768 * 64 * 17 * (128 * 2 + 4)


@pytest.mark.parametrize("bad,code", [
    (dict(H_q=5), msa.MSA_ERR_INVALID_ARG),
    (dict(topk=0), msa.MSA_ERR_INVALID_ARG),
    (dict(N=0), msa.MSA_ERR_INVALID_ARG),
    (dict(d=96), msa.MSA_ERR_UNSUPPORTED),
    (dict(d_idx=48), msa.MSA_ERR_UNSUPPORTED),
    (dict(block_k=16), msa.MSA_ERR_UNSUPPORTED),
    (dict(topk=17), msa.MSA_ERR_UNSUPPORTED),
    (dict(H_q=6, H_kv=2), msa.MSA_ERR_UNSUPPORTED),
])
def test_host_validation_codes(bad, code):
    d = dims(**bad)
    n = ctypes.c_size_t(0)
    assert msa.lib().msa_workspace_size(msa.MSA_OP_ATTN_FWD, ctypes.byref(d.c()), ctypes.byref(n)) == code


def test_null_and_misaligned_pointers_are_rejected_on_the_host():
    L = msa.lib()
    d = dims()
    c = d.c()
    P = ctypes.c_void_p
    # null inputs
    assert L.msa_index_topk(ctypes.byref(c), None, None, None, None, None, 0, None) == msa.MSA_ERR_INVALID_ARG
    # misaligned pointers (never dereferenced: rejected before any launch)
    assert L.msa_sparse_attn_fwd(ctypes.byref(c), P(0x1001), P(0x2000), P(0x3000), P(0x4000), P(0x5000), None,
                                 P(0x10000), 1 << 30, None) == msa.MSA_ERR_INVALID_ARG
    assert L.msa_sparse_attn_fwd_bf16(ctypes.byref(c), P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5008),
                                      None, P(0x10000), 1 << 30, None) == msa.MSA_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert L.msa_sparse_attn_fwd(ctypes.byref(c), P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), None,
                                 P(0x10000), 16, None) == msa.MSA_ERR_WORKSPACE
    assert L.msa_sparse_attn_fwd_bf16(ctypes.byref(c), P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000),
                                      None, P(0x10000), 16, None) == msa.MSA_ERR_WORKSPACE
    assert L.msa_sparse_attn_fwd(ctypes.byref(c), P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), None,
                                 P(0x10010), 1 << 30, None) == msa.MSA_ERR_WORKSPACE
    # KL: unsupported group size for the KL kernel family
    d2 = dims(H_q=8, H_kv=2)
    assert L.msa_kl_fwd_grad(ctypes.byref(d2.c()), *([P(0x1000)] * 7), ctypes.c_float(1.0), P(0x1000), P(0x1000),
                             P(0x1000), P(0x10000), 1 << 30, None) == msa.MSA_ERR_UNSUPPORTED
    assert L.msa_get_device_status(None, None) == msa.MSA_ERR_INVALID_ARG


def test_bindings_reject_host_tensors():
    """The library takes device pointers: every binding refuses host tensors before any call into
    it (a host pointer handed to a kernel would be an illegal address on the GPU)."""
    import torch
    d = dims()
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    blocks = torch.zeros(1, 512, 2, 5, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        msa.msa_index_topk(d, bf(1, 512, 2, 32), bf(1, 512, 32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        msa.msa_sparse_attn_fwd(d, bf(1, 512, 4, 64), bf(1, 512, 2, 64), bf(1, 512, 2, 64), blocks)
    with pytest.raises(ValueError, match="CUDA tensor"):
        msa.msa_sparse_attn_decode(d, torch.ones(1, dtype=torch.int32), bf(1, 4, 64), bf(1, 2, 32),
                                   bf(1, 512, 2, 64), bf(1, 512, 2, 64), bf(1, 512, 32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        msa.msa_quantize_e4m3_rows(bf(8, 64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        msa.msa_topk_merge(d, torch.zeros(2, 1, 512, 2, 4), torch.zeros(2, 1, 512, 2, 4, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        msa.msa_lse_combine(d, torch.zeros(2, 1, 512, 2, 2))


def test_stream_device_and_workspace_checks(monkeypatch):
    """Launches go to the current CUDA device: tensors or a stream of another device are refused,
    and a caller's workspace must be a contiguous uint8 tensor on the inputs' device (host logic,
    checked with a stand-in for the current device and stream)."""
    import torch

    class FakeStream:
        def __init__(self, idx):
            self.device = torch.device("cuda", idx)
            self.cuda_stream = 0x1234

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: FakeStream(0))
    assert msa._stream(None, torch.device("cuda", 0)).value == 0x1234
    assert msa._stream(FakeStream(0), torch.device("cuda", 0)).value == 0x1234
    with pytest.raises(ValueError, match="current CUDA device"):
        msa._stream(None, torch.device("cuda", 1))
    with pytest.raises(ValueError, match="current CUDA device"):
        msa._stream(None, torch.device("cpu"))
    with pytest.raises(ValueError, match="stream belongs"):
        msa._stream(FakeStream(1), torch.device("cuda", 0))
    with pytest.raises(ValueError, match="ws must be"):
        msa._ws(torch.zeros(64, dtype=torch.int32), msa.MSA_OP_DECODE, dims(), torch.device("cpu"))
    with pytest.raises(ValueError, match="ws must be"):
        msa._ws(torch.zeros(64, 4, dtype=torch.uint8)[:, 0], msa.MSA_OP_DECODE, dims(), torch.device("cpu"))
    ws = torch.zeros(256, dtype=torch.uint8)
    assert msa._ws(ws, msa.MSA_OP_DECODE, dims(), torch.device("cpu")) is ws
