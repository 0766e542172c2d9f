"""The FMA-pipe exponential exp2_fma_x2 (msa_common.cuh), checked without a GPU: its constants are
the ones the Remez generator beside it produces, their fp32 Horner error is within the stated bound,
and an fp32 emulation of the whole method (Cody-Waite reduction by the 1.5 * 2^23 addition, the
polynomial, the exponent-field addition) matches 2^x within 3e-7 relative on [-125, 1/2]."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_idx_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_constants():
    txt = open(os.path.join(CSRC, "msa_common.cuh")).read()
    body = re.search(r"constexpr uint32_t kC\[6\] = \{([^}]*)\}", txt).group(1)
    return [int(v.strip().rstrip("u"), 16) for v in body.split(",")]


def test_kernel_constants_are_the_generators():
    g = _gen()
    c = g.fp32_coefficients()
    assert [int(v.view(np.uint32)) for v in c] == _kernel_constants()
    assert g.horner_fp32_rel_error(c) <= 2.5e-7


def _emulate(x):
    """The helper's arithmetic in fp32, element by element as the kernel does it."""
    c = [np.uint32(v).view(np.float32) for v in _kernel_constants()]
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)  # the kernel's fma(j, -1, x): exact either way
    p = np.full_like(f, c[5])
    for k in (4, 3, 2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_emulated_method_error_bound():
    x = np.concatenate([np.linspace(-125.0, 0.5, 400001), np.array([0.0, -0.5, 0.5, -1.0, -124.5, -125.0])]).astype(np.float32)
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.abs((y - ref) / ref).max() <= 3e-7
    assert _emulate(np.array([0.0], dtype=np.float32))[0] == np.float32(1.0000001192092896)


def test_emulated_method_below_range_gives_tiny_positive():
    y = _emulate(np.array([-np.inf, -1000.0, -126.0, -125.5], dtype=np.float32)).astype(np.float64)
    assert np.all(y > 0) and np.all(y <= 2.0 ** -124)
