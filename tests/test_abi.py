"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/solattn.h declares, and rejects bad arguments before it
touches the device."""
import ctypes
import math
import os
import re

import pytest

from block_sparse_attention_cov_b200 import _lib
from block_sparse_attention_cov_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "solattn.h")


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(solattn_[a-z_]+)\s*\(", text)))


def test_header_declares_the_python_export_list():
    assert _declared() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_version_and_strerror(L):
    assert L.solattn_version() == 10000
    for code in range(0, 9):
        assert _lib.strerror(code) and "unknown" not in _lib.strerror(code)
    assert "unknown" in _lib.strerror(99)


def _pooled_struct(addr=0x100000):
    st = _lib.PooledStruct()
    for i, (name, _) in enumerate(_lib.PooledStruct._fields_):
        setattr(st, name, addr + i * 0x10000)
    return st


FAKE = ctypes.c_void_p(0x7F0000000000)  # never dereferenced: every call below fails validation first


def _fwd(L, q=FAKE, k=FAKE, v=FAKE, B=1, H=1, N=128, d=64, pooled=None, beta=0.5, out=FAKE, lse=None,
         dens=None, ws=FAKE, wsb=256):
    pooled = _pooled_struct() if pooled is None else pooled
    return L.solattn_forward(q, k, v, B, H, N, d, ctypes.byref(pooled), ctypes.c_float(beta), out, lse, dens,
                             ws, wsb, None)


def test_forward_argument_errors(L):
    assert _fwd(L, q=None) == _lib.ERR_ARG
    assert _fwd(L, out=None) == _lib.ERR_ARG
    assert _fwd(L, N=0) == _lib.ERR_ARG
    assert _fwd(L, B=-1) == _lib.ERR_ARG
    assert _fwd(L, d=96) == _lib.ERR_UNSUPPORTED
    assert _fwd(L, N=_lib.MAX_TOKENS + 1) == _lib.ERR_UNSUPPORTED
    assert _fwd(L, beta=math.nan) == _lib.ERR_ARG
    assert _fwd(L, k=ctypes.c_void_p(0x7F0000000008)) == _lib.ERR_ALIGN
    assert _fwd(L, lse=ctypes.c_void_p(0x7F0000000002)) == _lib.ERR_ALIGN
    bad = _pooled_struct()
    bad.kmean = None
    assert _fwd(L, pooled=bad) == _lib.ERR_ARG
    bad = _pooled_struct()
    bad.kcov = 0x100004
    assert _fwd(L, pooled=bad) == _lib.ERR_ALIGN
    assert _fwd(L, ws=None) == _lib.ERR_WORKSPACE
    assert _fwd(L, wsb=255) == _lib.ERR_WORKSPACE


def test_forward_ex_argument_errors(L):
    def call(opts, **kw):
        return L.solattn_forward_ex(FAKE, FAKE, FAKE, 1, 1, 128, 64, ctypes.byref(_pooled_struct()),
                                    None if opts is None else ctypes.byref(opts), FAKE, None, None, FAKE, 256, None)
    O = _lib.OptionsStruct
    assert call(None) == _lib.ERR_ARG
    assert call(O(7, 0.5, 0, 0.0, 0)) == _lib.ERR_ARG                      # unknown rule
    assert call(O(_lib.RULE_THRESHOLD, math.nan, 0, 0.0, 0)) == _lib.ERR_ARG
    assert call(O(_lib.RULE_TOPP, 0.0, 0, math.nan, 0)) == _lib.ERR_ARG
    assert call(O(_lib.RULE_TOPK, 0.0, 3, 0.0, -1)) == _lib.ERR_ARG        # negative forced count
    assert call(O(_lib.RULE_THRESHOLD, 0.5, 0, 0.0, 0, _lib.StridesStruct(0, 0, 0), 2)) == _lib.ERR_ARG
    bad = _pooled_struct()
    bad.kcov = None
    assert L.solattn_forward_ex(FAKE, FAKE, FAKE, 1, 1, 128, 64, ctypes.byref(bad),
                                ctypes.byref(O(_lib.RULE_TOPK, 0.0, 3, 0.0, 0)), FAKE, None, None, FAKE, 256,
                                None) == _lib.ERR_ARG


def test_strides_validation(L):
    S = _lib.StridesStruct
    st = _pooled_struct()

    def pool(strides):
        return L.solattn_pool_ex(FAKE, FAKE, FAKE, 1, 2, 128, 64, ctypes.byref(strides), ctypes.byref(st), None)

    def fwd(strides):
        o = _lib.OptionsStruct(_lib.RULE_THRESHOLD, 0.5, 0, 0.0, 0, strides)
        return L.solattn_forward_ex(FAKE, FAKE, FAKE, 1, 2, 128, 64, ctypes.byref(st), ctypes.byref(o), FAKE, None,
                                    None, FAKE, 256, None)
    for bad in (S(128 * 64 * 2, 64, 60), S(-8, 64, 128), S(128 * 128, 64 + 4, 128), S(0, 64 * 128, 32)):
        assert pool(bad) == _lib.ERR_ARG
        assert fwd(bad) == _lib.ERR_ARG


def test_dense_and_pool_argument_errors(L):
    assert L.solattn_dense(FAKE, FAKE, None, 1, 1, 64, 128, FAKE, None, FAKE, 256, None) == _lib.ERR_ARG
    assert L.solattn_dense(FAKE, FAKE, FAKE, 1, 1, 64, 32, FAKE, None, FAKE, 256, None) == _lib.ERR_UNSUPPORTED
    assert L.solattn_dense(FAKE, FAKE, FAKE, 1, 1, 64, 128, FAKE, None, None, 256, None) == _lib.ERR_WORKSPACE
    st = _pooled_struct()
    assert L.solattn_pool(FAKE, FAKE, FAKE, 1, 1, 0, 64, ctypes.byref(st), None) == _lib.ERR_ARG
    assert L.solattn_pool(FAKE, FAKE, FAKE, 1, 1, 64, 64, None, None) == _lib.ERR_ARG
    assert L.solattn_status(None, None) == _lib.ERR_WORKSPACE


def test_pooled_layout_sizes_and_alignment(L):
    n = ctypes.c_size_t(0)
    B, H, N, d = 1, 40, 75600, 128
    assert L.solattn_pooled_layout(B, H, N, d, None, None, ctypes.byref(n)) == 0
    nb = math.ceil(N / 64)
    r = lambda x: (x + 255) // 256 * 256
    want = 3 * r(B * H * nb * d * 4) + r(B * H * d * 4) + r(B * H * d * d * 4) + 2 * r(B * H * nb * d * 2)
    assert n.value == want
    st = _lib.PooledStruct()
    base = 0x10000000
    assert L.solattn_pooled_layout(B, H, N, d, ctypes.c_void_p(base), ctypes.byref(st), None) == 0
    ptrs = [getattr(st, f) for f, _ in _lib.PooledStruct._fields_]
    assert ptrs[0] == base and all(p % 256 == 0 for p in ptrs) and ptrs == sorted(ptrs)
    assert ptrs[-1] + r(B * H * nb * d * 2) == base + want
    assert L.solattn_pooled_layout(B, H, N, d, ctypes.c_void_p(base + 8), ctypes.byref(st), None) == _lib.ERR_ALIGN
    assert L.solattn_pooled_layout(B, H, N, 80, None, None, ctypes.byref(n)) == _lib.ERR_UNSUPPORTED


def test_noalloc_path_names_no_allocating_call():
    """The allocation-free entry point and its helpers call no device
    allocator (checked on the source of the noalloc section of api.cu)."""
    src = open(os.path.join(ROOT, "block_sparse_attention_cov_b200", "csrc", "api.cu")).read()
    section = src[src.index("Allocation-free forward"):src.index("End-to-end forward on host buffers")]
    code = re.sub(r"//[^\n]*", "", section)
    for name in ("cudaMalloc", "cudaMallocAsync", "cudaMallocManaged", "cudaFree", "malloc(", "new ", "torch"):
        assert name not in code, name


def test_strides_reject_aliasing_heads_and_batches(L):
    """out shares q's strides: a zero head (batch) stride with several heads
    (batches) would make them write the same rows."""
    def call(B, H, strides):
        opts = _lib.OptionsStruct(_lib.RULE_THRESHOLD, 0.5, 0, 0.0, 0, _lib.StridesStruct(*strides), 0)
        return L.solattn_forward_ex(FAKE, FAKE, FAKE, B, H, 128, 64, ctypes.byref(_pooled_struct()),
                                    ctypes.byref(opts), FAKE, None, None, None, 0, None)

    assert call(1, 2, (0, 0, 64)) == _lib.ERR_ARG
    assert call(2, 1, (0, 64, 64)) == _lib.ERR_ARG
    # one head and one batch: a zero stride there is harmless; the call then
    # fails later, on the missing workspace
    assert call(1, 1, (0, 0, 64)) == _lib.ERR_WORKSPACE


def test_dense_rejects_non_contiguous_views():
    import torch

    import block_sparse_attention_cov_b200 as sa

    x = torch.zeros((1, 4, 2, 64), dtype=torch.bfloat16).permute(0, 2, 1, 3)  # [B, N, H, d] seen as [B, H, N, d]
    with pytest.raises(ValueError, match="contiguous"):
        sa.dense(x, x, x)


def test_host_scratch_sizes(L):
    """Two chunk buffers (q, k, v, out, lse, density and the chunk's pooled
    statistics, each 256-byte aligned) after the workspace."""
    B, H, N, d = 1, 40, 75600, 128
    nb = math.ceil(N / 64)
    r = lambda x: (x + 255) // 256 * 256
    for chunk, C in ((0, 3), (5, 5), (100, 40)):
        n, p = ctypes.c_size_t(0), ctypes.c_size_t(0)
        assert L.solattn_host_scratch_bytes(B, H, N, d, chunk, ctypes.byref(n)) == 0
        assert L.solattn_pooled_layout(1, C, N, d, None, None, ctypes.byref(p)) == 0
        buf = 4 * r(C * N * d * 2) + r(C * N * 4) + r(C * nb * 4) + r(p.value)
        assert n.value == _lib.WORKSPACE_BYTES + 2 * buf, chunk
    assert L.solattn_host_scratch_bytes(B, H, N, d, -1, ctypes.byref(n)) == _lib.ERR_ARG
    assert L.solattn_host_scratch_bytes(B, H, N, 80, 0, ctypes.byref(n)) == _lib.ERR_UNSUPPORTED
    assert L.solattn_host_scratch_bytes(B, H, N, d, 0, None) == _lib.ERR_ARG


def test_forward_host_argument_errors(L):
    h = ctypes.create_string_buffer(64)
    p = ctypes.cast(h, ctypes.c_void_p)
    scratch = ctypes.c_void_p(0x10000000)
    f = ctypes.c_float
    args = lambda q=p, out=p, beta=0.5, chunk=0, sc=scratch, n=1 << 30: (
        q, p, p, 1, 2, 256, 64, f(beta), out, None, None, chunk, sc, n, None)
    assert L.solattn_forward_host(*args(q=None)) == _lib.ERR_ARG
    assert L.solattn_forward_host(*args(out=None)) == _lib.ERR_ARG
    assert L.solattn_forward_host(*args(beta=float("nan"))) == _lib.ERR_ARG
    assert L.solattn_forward_host(*args(chunk=-1)) == _lib.ERR_ARG
    assert L.solattn_forward_host(*args(sc=None)) == _lib.ERR_WORKSPACE
    assert L.solattn_forward_host(*args(sc=ctypes.c_void_p(0x10000010))) == _lib.ERR_ALIGN
    assert L.solattn_forward_host(*args(n=1024)) == _lib.ERR_WORKSPACE
    assert L.solattn_forward_host(p, p, p, 1, 2, 256, 80, f(0.5), p, None, None, 0, scratch, 1 << 30,
                                  None) == _lib.ERR_UNSUPPORTED


def test_plain_c_client_compiles_links_and_passes(L, tmp_path):
    """The boundary is a C ABI: a C program that includes only
    include/solattn.h and links libsolattn.so compiles with gcc and passes its
    host-side checks (no GPU needed)."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "c_client"
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_client.c"), "-L", libdir, "-lsolattn", f"-Wl,-rpath,{libdir}", "-lm",
           "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    proc = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert proc.returncode == 0, proc.stderr
    assert "c client ok" in proc.stdout
