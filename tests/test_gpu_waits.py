"""Failure detection on the GPU without a fault: every wait in the fused kernel
is bounded; when one runs out the kernel records SOLATTN_ERR_TIMEOUT with the
wait site and unit in the caller's workspace, the CTA stops, and the context
stays usable.

The test uses the test-hook build of the library (libsolattn_testhooks.so: the
product library has no hook): CTA 0 never requests its first K tile, so its
QK issuer's wait on that tile runs out after a short budget (a flag that
nothing sets). The next launch, hook cleared, must succeed and match the oracle.
"""
import ctypes
import math
import time

import numpy as np
import pytest
import torch

from block_sparse_attention_cov_b200 import _lib
from block_sparse_attention_cov_b200.inputs import WORKLOADS, make_qkv
from hooklib import hooks_lib
from oracle import solattn_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return hooks_lib()


def _run(L, q, k, v, beta):
    B, Hh, N, d = q.shape
    n = ctypes.c_size_t(0)
    assert L.solattn_pooled_layout(B, Hh, N, d, None, None, ctypes.byref(n)) == 0
    buf = torch.empty(n.value, dtype=torch.uint8, device="cuda")
    st = _lib.PooledStruct()
    assert L.solattn_pooled_layout(B, Hh, N, d, ctypes.c_void_p(buf.data_ptr()), ctypes.byref(st), None) == 0
    out = torch.empty_like(q)
    lse = torch.empty((B, Hh, N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert L.solattn_pool(p(q), p(k), p(v), B, Hh, N, d, ctypes.byref(st), None) == 0
    rc = L.solattn_forward(p(q), p(k), p(v), B, Hh, N, d, ctypes.byref(st), beta, p(out), p(lse), None, p(ws), 256,
                           None)
    assert rc == 0
    status = L.solattn_status(p(ws), None)
    words = ws[:16].view(torch.int32).cpu().tolist()  # tile counter, error, wait site, unit
    return status, words, out, lse


def test_expired_wait_reports_timeout_and_next_launch_succeeds(H):
    wl = WORKLOADS["tiny"]
    q, k, v = make_qkv(wl, seed=7)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    assert H.solattn_test_set_hook(0, 20_000_000) == 0  # CTA 0 skips its first K tile; 20 ms budget
    t0 = time.monotonic()
    status, words, _, _ = _run(H, qd, kd, vd, 0.5)
    elapsed = time.monotonic() - t0
    assert status == _lib.ERR_TIMEOUT, (status, words)
    assert words[1] == _lib.ERR_TIMEOUT and words[2] > 0  # the failing wait site is recorded
    assert elapsed < 30.0
    assert H.solattn_test_set_hook(-1, 2_000_000_000) == 0
    status, words, out, lse = _run(H, qd, kd, vd, 0.5)
    assert status == 0 and words[1] == 0
    out_o, lse_o, _ = orc.forward(q, k, v, 0.5)
    og = out.float().cpu().numpy().astype(np.float64)
    err = og - out_o
    assert np.linalg.norm(err) / np.linalg.norm(out_o) <= 1e-2 and np.abs(err).max() <= 2e-2
    assert np.abs(lse.cpu().numpy() - lse_o).max() <= 1e-3


def test_noalloc_status_reports_an_expired_wait(H):
    """solattn_forward_noalloc keeps its status block in the static array;
    solattn_noalloc_status reads it back (no allocation) and reports the
    timeout that the call's own return code cannot."""
    wl = WORKLOADS["tiny"]
    q, k, v = (x.cuda() for x in make_qkv(wl, seed=8))
    B, Hh, N, d = q.shape
    out = torch.empty_like(q)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert H.solattn_test_set_hook(0, 20_000_000) == 0
    try:
        assert H.solattn_forward_noalloc(p(q), p(k), p(v), B, Hh, N, d, 0.5, p(out), None, None, None) == 0
        assert H.solattn_noalloc_status(None) == _lib.ERR_TIMEOUT
    finally:
        assert H.solattn_test_set_hook(-1, 2_000_000_000) == 0
    assert H.solattn_forward_noalloc(p(q), p(k), p(v), B, Hh, N, d, 0.5, p(out), None, None, None) == 0
    assert H.solattn_noalloc_status(None) == _lib.OK
    out_o, _, _ = orc.forward(q.cpu(), k.cpu(), v.cpu(), 0.5)
    err = out.float().cpu().numpy().astype(np.float64) - out_o
    assert np.linalg.norm(err) / np.linalg.norm(out_o) <= 1e-2 and np.abs(err).max() <= 2e-2
