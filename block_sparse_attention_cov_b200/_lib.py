"""ctypes loader for libsolattn.so (the C ABI of include/solattn.h)."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsolattn.so")

# Every symbol declared in include/solattn.h.
EXPORTS = (
    "solattn_pooled_layout",
    "solattn_pool",
    "solattn_forward",
    "solattn_dense",
    "solattn_status",
    "solattn_strerror",
    "solattn_version",
    "solattn_forward_noalloc",
    "solattn_forward_ex",
    "solattn_pool_ex",
    "solattn_noalloc_status",
    "solattn_host_scratch_bytes",
    "solattn_forward_host",
)

OK = 0
ERR_ARG = 1
ERR_UNSUPPORTED = 2
ERR_ALIGN = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_DEVICE = 6
ERR_WORKSPACE = 7
ERR_SCRATCH = 8
WORKSPACE_BYTES = 256
NOALLOC_SCRATCH_BYTES = 16 << 20
BLOCK = 64
MAX_TOKENS = 262144
RULE_THRESHOLD, RULE_TOPK, RULE_TOPP = 0, 1, 2


class PooledStruct(ctypes.Structure):
    """Mirror of solattn_pooled_t."""

    _fields_ = [(name, ctypes.c_void_p) for name in ("qbar", "kbar", "vbar", "kmean", "kcov", "kbar16", "vbar16")]


class StridesStruct(ctypes.Structure):
    """Mirror of solattn_strides_t."""

    _fields_ = [("batch", ctypes.c_longlong), ("head", ctypes.c_longlong), ("token", ctypes.c_longlong)]


class OptionsStruct(ctypes.Structure):
    """Mirror of solattn_options_t."""

    _fields_ = [("rule", ctypes.c_int), ("beta", ctypes.c_float), ("topk", ctypes.c_int), ("topp", ctypes.c_float),
                ("n_forced", ctypes.c_int), ("strides", StridesStruct), ("correction", ctypes.c_int)]


_lib = None


def declare(L: ctypes.CDLL) -> ctypes.CDLL:
    """Sets the argument and result types of every exported call on a loaded
    copy of the library (the product build or its test-hook variant)."""
    i, vp, f, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
    L.solattn_pooled_layout.argtypes = [i, i, i, i, vp, ctypes.POINTER(PooledStruct), ctypes.POINTER(sz)]
    L.solattn_pooled_layout.restype = i
    L.solattn_pool.argtypes = [vp, vp, vp, i, i, i, i, ctypes.POINTER(PooledStruct), vp]
    L.solattn_pool.restype = i
    L.solattn_forward.argtypes = [vp, vp, vp, i, i, i, i, ctypes.POINTER(PooledStruct), f, vp, vp, vp, vp, sz, vp]
    L.solattn_forward.restype = i
    L.solattn_dense.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, sz, vp]
    L.solattn_dense.restype = i
    L.solattn_status.argtypes = [vp, vp]
    L.solattn_status.restype = i
    L.solattn_strerror.argtypes = [i]
    L.solattn_strerror.restype = ctypes.c_char_p
    L.solattn_forward_noalloc.argtypes = [vp, vp, vp, i, i, i, i, f, vp, vp, vp, vp]
    L.solattn_forward_noalloc.restype = i
    L.solattn_noalloc_status.argtypes = [vp]
    L.solattn_noalloc_status.restype = i
    L.solattn_forward_ex.argtypes = [vp, vp, vp, i, i, i, i, ctypes.POINTER(PooledStruct),
                                     ctypes.POINTER(OptionsStruct), vp, vp, vp, vp, sz, vp]
    L.solattn_forward_ex.restype = i
    L.solattn_pool_ex.argtypes = [vp, vp, vp, i, i, i, i, ctypes.POINTER(StridesStruct), ctypes.POINTER(PooledStruct),
                                  vp]
    L.solattn_pool_ex.restype = i
    L.solattn_host_scratch_bytes.argtypes = [i, i, i, i, i, ctypes.POINTER(sz)]
    L.solattn_host_scratch_bytes.restype = i
    L.solattn_forward_host.argtypes = [vp, vp, vp, i, i, i, i, f, vp, vp, vp, i, vp, sz, vp]
    L.solattn_forward_host.restype = i
    L.solattn_version.argtypes = []
    L.solattn_version.restype = i
    return L


def lib() -> ctypes.CDLL:
    """The loaded library. Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing; build it with `python -m block_sparse_attention_cov_b200.build`"
        )
    _lib = declare(ctypes.CDLL(LIB_PATH))
    return _lib


def strerror(code: int) -> str:
    return lib().solattn_strerror(int(code)).decode()
