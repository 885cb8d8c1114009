"""Access to the test-hook build of the library (libsolattn_testhooks.so) for
the GPU tests: the same C ABI as the product library plus test-only calls that
(a) make one CTA skip its first K tile and shorten the bounded-wait budget, and
(b) copy every unit's kept bitmaps and row statistics (mu_i, sigma_i, tau_i)
out of the routing warps, so that the kept sets can be compared with the
oracle's element by element. The product library has neither."""
from __future__ import annotations

import ctypes
import math

import numpy as np
import torch

from block_sparse_attention_cov_b200 import _lib
from block_sparse_attention_cov_b200.build import build

_hooks = None


def hooks_lib() -> ctypes.CDLL:
    global _hooks
    if _hooks is None:
        L = _lib.declare(ctypes.CDLL(build(hooks=True)))
        L.solattn_test_set_hook.argtypes = [ctypes.c_int, ctypes.c_ulonglong]
        L.solattn_test_set_hook.restype = ctypes.c_int
        L.solattn_test_set_route_dump.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        L.solattn_test_set_route_dump.restype = ctypes.c_int
        _hooks = L
    return _hooks


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def pooled(L, q, k, v):
    """solattn_pool of the hook build into a fresh buffer: (buffer, struct)."""
    B, H, N, d = q.shape
    n = ctypes.c_size_t(0)
    assert L.solattn_pooled_layout(B, H, N, d, None, None, ctypes.byref(n)) == 0
    buf = torch.empty(n.value, dtype=torch.uint8, device=q.device)
    st = _lib.PooledStruct()
    assert L.solattn_pooled_layout(B, H, N, d, _p(buf), ctypes.byref(st), None) == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.solattn_pool(_p(q), _p(k), _p(v), B, H, N, d, ctypes.byref(st), stream) == 0
    return buf, st


def forward_with_routing(q, k, v, beta=0.0, rule="threshold", topk=0, topp=0.0, n_forced=0, correction="block"):
    """One forward through the hook build with the routing copy switched on.

    Returns (out, lse, density, mask, stats): mask [B, H, N_b, N_b] bool (the
    kept sets the kernel used), stats [B, H, N_b, 3] float (mu, sigma, tau)."""
    L = hooks_lib()
    B, H, N, d = q.shape
    nb = math.ceil(N / 64)
    words = math.ceil(nb / 32)
    buf, st = pooled(L, q, k, v)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dens = torch.empty((B, H, nb), dtype=torch.int32, device=q.device)
    mask_words = torch.zeros((B * H, nb, words), dtype=torch.int32, device=q.device)
    stats = torch.full((B * H, nb, 3), float("nan"), dtype=torch.float32, device=q.device)
    ws = torch.zeros(_lib.WORKSPACE_BYTES, dtype=torch.uint8, device=q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.solattn_test_set_route_dump(_p(mask_words), _p(stats)) == 0
    try:
        rules = {"threshold": _lib.RULE_THRESHOLD, "topk": _lib.RULE_TOPK, "topp": _lib.RULE_TOPP}
        opts = _lib.OptionsStruct(rules[rule], float(beta), int(topk), float(topp), int(n_forced),
                                  _lib.StridesStruct(0, 0, 0), 1 if correction == "token" else 0)
        rc = L.solattn_forward_ex(_p(q), _p(k), _p(v), B, H, N, d, ctypes.byref(st), ctypes.byref(opts), _p(out),
                                  _p(lse), _p(dens), _p(ws), ws.numel(), stream)
        assert rc == 0, _lib.strerror(rc)
        assert L.solattn_status(_p(ws), stream) == 0
    finally:
        assert L.solattn_test_set_route_dump(None, None) == 0
    w = mask_words.cpu().numpy().view(np.uint32)
    bits = (w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1  # [BH, nb, words, 32]
    mask = bits.reshape(B * H, nb, words * 32)[..., :nb].astype(bool).reshape(B, H, nb, nb)
    return out, lse, dens, mask, stats.cpu().numpy().reshape(B, H, nb, 3)
