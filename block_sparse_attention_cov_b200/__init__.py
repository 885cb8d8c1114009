"""Sol-Attn block-sparse attention forward for B200 (sm_100a).

Python binding of the C ABI in include/solattn.h: argument marshalling only
(torch tensors -> device pointers, the current CUDA stream, output allocation).
Every step of the computation runs in the library's CUDA kernels; there is no
CPU path. The names mirror the C calls:

    stats = pool(q, k, v)                          # solattn_pool
    out, lse, density = forward(q, k, v, stats, beta)   # solattn_forward
    out, lse = dense(q, k, v)                      # solattn_dense
    forward_host(q_h, k_h, v_h, beta, out_h, ...)  # solattn_forward_host (host tensors)

q, k, v: CUDA bf16 tensors [B, H, N, d], contiguous, d in {64, 128}.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _lib

__all__ = ["SolAttnError", "PooledStats", "pool", "forward", "dense", "status", "workspace", "pooled_bytes",
           "host_scratch", "forward_host"]


class SolAttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = int(code)
        super().__init__(f"{what}: {_lib.strerror(code)} (code {code})")


def _check(rc: int, what: str):
    if rc != _lib.OK:
        raise SolAttnError(rc, what)


def _shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _check_inputs(*ts):
    """q, k, v (and out): CUDA bf16 [B, H, N, d] with contiguous d and one common
    set of strides (contiguous, [B, N, H, d] seen through a permute, padded
    rows, ...)."""
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.stride(-1) == 1):
            raise ValueError("q, k, v must be CUDA bf16 [B, H, N, d] tensors with contiguous d")
    if not all(t.shape == ts[0].shape for t in ts):
        raise ValueError("q, k, v must have the same shape")
    if not all(t.stride() == ts[0].stride() for t in ts):
        raise ValueError("q, k, v must share their strides")


def _strides(t):
    """solattn_strides_t of a [B, H, N, d] tensor (all zero when contiguous)."""
    if t.is_contiguous():
        return _lib.StridesStruct(0, 0, 0)
    sb, sh, sn, _ = t.stride()
    return _lib.StridesStruct(sb, sh, sn)


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def pooled_bytes(B: int, H: int, N: int, d: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.lib().solattn_pooled_layout(B, H, N, d, None, None, ctypes.byref(n)), "solattn_pooled_layout")
    return int(n.value)


@dataclass
class PooledStats:
    """solattn_pool's outputs: one device buffer and fp32 views into it."""

    buffer: torch.Tensor
    struct: _lib.PooledStruct
    shape: tuple

    def view(self, name: str) -> torch.Tensor:
        B, H, N, d = self.shape
        nb = (N + _lib.BLOCK - 1) // _lib.BLOCK
        dims = {
            "qbar": (B, H, nb, d), "kbar": (B, H, nb, d), "vbar": (B, H, nb, d),
            "kmean": (B, H, d), "kcov": (B, H, d, d), "kbar16": (B, H, nb, d), "vbar16": (B, H, nb, d),
        }[name]
        dt, size = (torch.bfloat16, 2) if name.endswith("16") else (torch.float32, 4)
        off = getattr(self.struct, name) - self.buffer.data_ptr()
        n = math.prod(dims)
        return self.buffer[off:off + size * n].view(dt).view(dims)


def pool(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stats: PooledStats | None = None) -> PooledStats:
    """Block means of q, k, v and the mean and covariance of the pooled keys (solattn_pool)."""
    _check_inputs(q, k, v)
    B, H, N, d = _shape(q)
    if stats is None:
        nbytes = pooled_bytes(B, H, N, d)
        buf = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
        st = _lib.PooledStruct()
        _check(_lib.lib().solattn_pooled_layout(B, H, N, d, _ptr(buf), ctypes.byref(st), None),
               "solattn_pooled_layout")
        stats = PooledStats(buf, st, (B, H, N, d))
    elif stats.shape != (B, H, N, d):
        raise ValueError("PooledStats shape does not match the inputs")
    if q.is_contiguous():
        _check(_lib.lib().solattn_pool(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, ctypes.byref(stats.struct),
                                       _stream()), "solattn_pool")
    else:
        strides = _strides(q)
        _check(_lib.lib().solattn_pool_ex(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, ctypes.byref(strides),
                                          ctypes.byref(stats.struct), _stream()), "solattn_pool_ex")
    return stats


def workspace(device=None) -> torch.Tensor:
    """A device workspace for forward/dense (scheduler counter and status word)."""
    return torch.empty(_lib.WORKSPACE_BYTES, dtype=torch.uint8, device=device or "cuda")


RULES = {"threshold": _lib.RULE_THRESHOLD, "topk": _lib.RULE_TOPK, "topp": _lib.RULE_TOPP}


def forward(q, k, v, stats: PooledStats, beta: float = 0.0, out=None, lse=None, density=None, ws=None,
            want_lse: bool = True, want_density: bool = True, rule: str = "threshold", topk: int = 0,
            topp: float = 0.0, n_forced: int = 0, correction: str = "block"):
    """Sol-Attn forward. Returns (out, lse, density).

    rule "threshold" (the method: tau_i = mu_i + beta sigma_i) on contiguous
    tensors calls solattn_forward; "topk" / "topp" (ablation rules),
    n_forced > 0, strided tensors or correction="token" (skipped blocks scored
    per query token against their mean key) call solattn_forward_ex. out is
    allocated with q's strides (torch.empty_like) and must share them."""
    _check_inputs(q, k, v)
    B, H, N, d = _shape(q)
    nb = (N + _lib.BLOCK - 1) // _lib.BLOCK
    out = torch.empty_like(q) if out is None else out
    if out.stride() != q.stride() or out.dtype != torch.bfloat16:
        raise ValueError("out must be a bf16 tensor with q's strides")
    if lse is None and want_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if density is None and want_density:
        density = torch.empty((B, H, nb), dtype=torch.int32, device=q.device)
    ws = workspace(q.device) if ws is None else ws
    if correction not in ("block", "token"):
        raise ValueError(f"unknown correction {correction!r}")
    if rule == "threshold" and n_forced == 0 and q.is_contiguous() and correction == "block":
        rc = _lib.lib().solattn_forward(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, ctypes.byref(stats.struct),
                                        ctypes.c_float(beta), _ptr(out), _ptr(lse), _ptr(density), _ptr(ws),
                                        ws.numel(), _stream())
        _check(rc, "solattn_forward")
    else:
        if rule not in RULES:
            raise ValueError(f"unknown rule {rule!r}")
        opts = _lib.OptionsStruct(RULES[rule], float(beta), int(topk), float(topp), int(n_forced), _strides(q),
                                  1 if correction == "token" else 0)
        rc = _lib.lib().solattn_forward_ex(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, ctypes.byref(stats.struct),
                                           ctypes.byref(opts), _ptr(out), _ptr(lse), _ptr(density), _ptr(ws),
                                           ws.numel(), _stream())
        _check(rc, "solattn_forward_ex")
    return out, lse, density


def dense(q, k, v, out=None, lse=None, ws=None, want_lse: bool = True):
    """Dense attention through the same kernel with routing off (solattn_dense).
    solattn_dense takes no strides: q, k, v and out must be contiguous
    [B, H, N, d] (a permuted, sliced or expanded view is rejected, since the
    kernel would read it as contiguous memory)."""
    for t in (q, k, v) + (() if out is None else (out,)):
        if not t.is_contiguous():
            raise ValueError("dense() needs contiguous [B, H, N, d] q, k, v and out")
    _check_inputs(q, k, v)
    B, H, N, d = _shape(q)
    out = torch.empty_like(q) if out is None else out
    if out.shape != q.shape or out.dtype != torch.bfloat16:
        raise ValueError("out must be a bf16 tensor of q's shape")
    if lse is None and want_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    ws = workspace(q.device) if ws is None else ws
    rc = _lib.lib().solattn_dense(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(out), _ptr(lse), _ptr(ws),
                                  ws.numel(), _stream())
    _check(rc, "solattn_dense")
    return out, lse


def host_scratch(B: int, H: int, N: int, d: int, chunk_heads: int = 0, device=None) -> torch.Tensor:
    """Device scratch for forward_host (solattn_host_scratch_bytes bytes)."""
    n = ctypes.c_size_t(0)
    _check(_lib.lib().solattn_host_scratch_bytes(B, H, N, d, int(chunk_heads), ctypes.byref(n)),
           "solattn_host_scratch_bytes")
    return torch.empty(n.value, dtype=torch.uint8, device=device or "cuda")


def forward_host(q, k, v, beta: float, out, lse=None, density=None, scratch=None, chunk_heads: int = 0):
    """solattn_forward_host: the threshold-rule forward on HOST tensors (CPU,
    contiguous bf16 [B, H, N, d]; page-locked for the copies to overlap the
    computation). out (bf16, q's shape), lse (float32 [B, H, N]) and density
    (int32 [B, H, N_b]) are host tensors written once the current stream has
    completed; the call only enqueues. scratch: a device tensor from
    host_scratch() (allocated here when None). Returns the scratch, whose first
    bytes hold the device status (status(scratch))."""
    for t in (q, k, v, out):
        if t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise ValueError("q, k, v, out must be contiguous host bf16 [B, H, N, d] tensors")
    if not (q.shape == k.shape == v.shape == out.shape):
        raise ValueError("q, k, v and out must have the same shape")
    B, H, N, d = _shape(q)
    nb = (N + _lib.BLOCK - 1) // _lib.BLOCK
    if lse is not None and (lse.is_cuda or lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N)
                            or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous host float32 [B, H, N] tensor")
    if density is not None and (density.is_cuda or density.dtype != torch.int32 or tuple(density.shape) != (B, H, nb)
                                or not density.is_contiguous()):
        raise ValueError("density must be a contiguous host int32 [B, H, N_b] tensor")
    scratch = host_scratch(B, H, N, d, chunk_heads) if scratch is None else scratch
    rc = _lib.lib().solattn_forward_host(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, ctypes.c_float(beta), _ptr(out),
                                         _ptr(lse), _ptr(density), int(chunk_heads), _ptr(scratch), scratch.numel(),
                                         _stream())
    _check(rc, "solattn_forward_host")
    return scratch


def status(ws: torch.Tensor) -> int:
    """Synchronises the current stream and returns the device status of the last
    call that used `ws` (0 = ok, 5 = a bounded wait expired)."""
    return int(_lib.lib().solattn_status(_ptr(ws), _stream()))
