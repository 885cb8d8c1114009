"""solattn_forward_host: the forward on host buffers, with the (b, h) pairs
copied to the device, attended and copied back in chunks that overlap. Every
pair is independent and the kernels compute each one the same way whatever
else is in the launch, so the results equal, bit for bit, those of
solattn_pool + solattn_forward on device copies of the same inputs; one case is
also checked against the oracle directly."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_cov_b200 as sa
from block_sparse_attention_cov_b200.build import build
from block_sparse_attention_cov_b200.inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build()


def _host_outputs(B, H, N, d, pinned, with_stats=True):
    nb = math.ceil(N / 64)
    out = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    lse = torch.empty((B, H, N), dtype=torch.float32) if with_stats else None
    dens = torch.empty((B, H, nb), dtype=torch.int32) if with_stats else None
    if pinned:
        out = out.pin_memory()
        lse = lse.pin_memory() if lse is not None else None
        dens = dens.pin_memory() if dens is not None else None
    return out, lse, dens


def _device_reference(q, k, v, beta):
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    st = sa.pool(qd, kd, vd)
    out, lse, dens = sa.forward(qd, kd, vd, st, beta)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), dens.cpu()


@pytest.mark.parametrize("chunk_heads", [1, 3, 0, 8])
def test_host_path_equals_device_path_bitwise(chunk_heads):
    wl = Workload("h", 1, 8, 128, (4, 32, 64))  # 8 heads x 8192 tokens
    q, k, v = make_qkv(wl, seed=51)
    beta = 0.8
    ref = _device_reference(q, k, v, beta)
    qp, kp, vp = (x.pin_memory() for x in (q, k, v))
    out, lse, dens = _host_outputs(*q.shape, pinned=True)
    scratch = sa.host_scratch(*q.shape, chunk_heads=chunk_heads)
    sa.forward_host(qp, kp, vp, beta, out, lse, dens, scratch=scratch, chunk_heads=chunk_heads)
    assert sa.status(scratch) == 0  # synchronises the stream: the host buffers are filled
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(dens, ref[2])


def test_host_path_pageable_ragged_and_repeated():
    """Pageable host memory (the copies serialise, the results do not change),
    a ragged shape (two batches, three heads, a partial last block, d = 64),
    NULL lse / density, and two calls back to back on one scratch."""
    wl = Workload("r", 2, 3, 64, (1, 1, 64 * 9 + 21))
    q, k, v = make_qkv(wl, seed=52)
    beta = 0.5
    ref = _device_reference(q, k, v, beta)
    scratch = sa.host_scratch(*q.shape, chunk_heads=2)
    out, lse, dens = _host_outputs(*q.shape, pinned=False)
    sa.forward_host(q, k, v, beta, out, lse, dens, scratch=scratch, chunk_heads=2)
    out2, _, _ = _host_outputs(*q.shape, pinned=False, with_stats=False)
    sa.forward_host(q, k, v, beta, out2, scratch=scratch, chunk_heads=2)
    assert sa.status(scratch) == 0
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(dens, ref[2])
    assert torch.equal(out2, ref[0])


def test_host_path_matches_oracle():
    from oracle import solattn_oracle as orc

    wl = Workload("o", 1, 4, 128, (1, 1, 64 * 13 + 5))
    q, k, v = make_qkv(wl, seed=53)
    beta = 0.7
    out_o, lse_o, dens_o = orc.forward(q, k, v, beta)
    r = orc.route_all(q, k, beta)
    ties = (np.abs(r["shat"] - r["tau"][..., None]) <= 1e-4).sum(-1)
    out, lse, dens = _host_outputs(*q.shape, pinned=True)
    scratch = sa.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), beta, out, lse, dens, chunk_heads=3)
    assert sa.status(scratch) == 0
    diff = np.abs(dens.numpy().astype(np.int64) - dens_o)
    assert (diff[ties == 0] == 0).all() and (diff <= ties).all()
    err = out.float().numpy().astype(np.float64) - out_o
    assert np.linalg.norm(err) / np.linalg.norm(out_o) <= 1e-2 and np.abs(err).max() <= 2e-2
    assert np.abs(lse.numpy() - lse_o).max() <= 1e-3
