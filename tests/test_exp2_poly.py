"""The fused forward kernel evaluates part of its softmax exponentials with a
Cody-Waite range reduction and a degree-3 polynomial (FMA pipe) instead of the
MUFU ex2. This test emulates those exact fp32 steps with the constants read
from the kernel source and checks the error bound against 2^y: the relative
error must stay far below the bf16 rounding of P (2^-9)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_cov_b200", "csrc", "forward.cu")


def _consts():
    text = open(SRC).read()
    return [np.float32(float(re.search(rf"kPolyC{i} = ([0-9.eE+-]+)f", text).group(1))) for i in range(4)]


def _exp2_emulated(y):
    c0, c1, c2, c3 = _consts()
    f32 = np.float32
    x = np.maximum(y.astype(f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t + f32(-12582912.0)).astype(f32)
    f = (n * f32(-1.0) + x).astype(f32)  # exact: |f| <= 1/2 and n is an integer
    q = (c3 * f + c2).astype(f32)
    q = (q * f + c1).astype(f32)
    q = (q * f + c0).astype(f32)
    bits = (t.view(np.uint32).astype(np.uint64) * 8388608 + q.view(np.uint32).astype(np.uint64)) % (1 << 32)
    return bits.astype(np.uint32).view(np.float32)


def test_polynomial_exp2_error_bound():
    y = np.concatenate([np.linspace(-125.0, 9.0, 2_000_001), np.array([-0.5, 0.5, 0.0, 1.0, -1.0, 8.0])])
    y = y.astype(np.float32)
    got = _exp2_emulated(y).astype(np.float64)
    want = np.exp2(y.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1e-4, rel.max()


def test_polynomial_exp2_clamps_masked_keys():
    y = np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32)
    got = _exp2_emulated(y)
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got <= 2.0 ** -124)


def test_fit_script_reproduces_the_kernel_constants():
    import importlib.util

    path = os.path.join(os.path.dirname(SRC), "fit_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    np.testing.assert_allclose(mod.fit(), np.array(_consts(), np.float32), rtol=1e-6)
