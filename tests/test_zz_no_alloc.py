"""solattn_forward_noalloc: the allocation-free entry point for callers that
cannot allocate device memory (its pooled statistics and workspace live in a
static device array inside the library). Checked through the C ABI against
solattn_pool + solattn_forward with caller-allocated buffers, on two calls in
a row with different inputs (the shared array keeps the previous call's
contents, which must not leak into the next result)."""
import ctypes
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_cov_b200 as sa
from block_sparse_attention_cov_b200 import _lib
from block_sparse_attention_cov_b200.build import build
from block_sparse_attention_cov_b200.inputs import WORKLOADS, Workload, make_qkv

pytestmark = pytest.mark.gpu

REL_L2, MAX_ABS, LSE_ABS = 1e-2, 2e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build()


def _outputs(q):
    B, H, N, d = q.shape
    nb = math.ceil(N / 64)
    return (torch.empty_like(q), torch.empty((B, H, N), dtype=torch.float32, device=q.device),
            torch.empty((B, H, nb), dtype=torch.int32, device=q.device))


def _noalloc(q, k, v, beta, outs):
    B, H, N, d = q.shape
    out, lse, dens = outs
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = _lib.lib().solattn_forward_noalloc(vp(q), vp(k), vp(v), B, H, N, d, ctypes.c_float(beta), vp(out), vp(lse),
                                            vp(dens), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.OK, _lib.strerror(rc)
    return out, lse, dens


def test_noalloc_matches_the_allocating_entry_points_on_two_calls():
    cases = [(WORKLOADS["tiny"], 1.0), (Workload("mid2", 1, 2, 128, (1, 1, 64 * 70 + 9)), 0.5)]
    inputs = [tuple(x.cuda() for x in make_qkv(wl, seed=7)) for wl, _ in cases]
    outs = [_outputs(qkv[0]) for qkv in inputs]
    # the first call on a device loads the library's module (code and static
    # array); what is measured below is that later calls allocate nothing
    _noalloc(*inputs[0], cases[0][1], outs[0])
    torch.cuda.synchronize()
    alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    got = [_noalloc(*qkv, beta, o) for qkv, (_, beta), o in zip(inputs, cases, outs)]  # two calls in a row
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0
    assert _lib.lib().solattn_noalloc_status(None) == _lib.OK
    for (q, k, v), (_, beta), (o1, l1, d1) in zip(inputs, cases, got):
        stats = sa.pool(q, k, v)
        o2, l2, d2 = sa.forward(q, k, v, stats, beta)
        torch.cuda.synchronize()
        a, b = o1.float().cpu().numpy(), o2.float().cpu().numpy()
        rel = np.linalg.norm(a - b) / np.linalg.norm(b)
        assert rel <= REL_L2 and np.abs(a - b).max() <= MAX_ABS
        assert (l1 - l2).abs().max().item() <= LSE_ABS
        assert torch.equal(d1, d2)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # 64 heads x 262144 tokens x d=128 needs ~400 MB of pooled statistics
    B, H, N, d = 1, 64, 262144, 128
    need = ctypes.c_size_t(0)
    assert _lib.lib().solattn_pooled_layout(B, H, N, d, None, None, ctypes.byref(need)) == _lib.OK
    assert need.value + _lib.WORKSPACE_BYTES > _lib.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x7F0000000000)  # rejected before anything touches it
    rc = _lib.lib().solattn_forward_noalloc(fake, fake, fake, B, H, N, d, ctypes.c_float(0.5), fake, None, None, None)
    assert rc == _lib.ERR_SCRATCH
