"""Strided q, k, v and out (solattn_pool_ex / solattn_forward_ex): the
[B, N, H, d] layout seen through a permute and rows padded to d + 8 elements
give, bit for bit, the results of contiguous [B, H, N, d] inputs (the same
tiles are summed in the same order; only the addressing differs)."""
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


def _bnhd(x):
    """The same values stored as [B, N, H, d], viewed as [B, H, N, d]."""
    return x.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)


def _padded(x, pad=8):
    """The same values in rows of d + pad elements, viewed as [B, H, N, d]."""
    B, H, N, d = x.shape
    base = torch.zeros((B, H, N, d + pad), dtype=x.dtype, device=x.device)
    base[..., :d] = x
    return base[..., :d]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rule", ["threshold", "topk"])
def test_strided_layouts_equal_contiguous_bitwise(d, rule):
    wl = Workload("s", 2, 3, d, (1, 1, 64 * 11 + 37))
    q, k, v = (x.cuda() for x in make_qkv(wl, seed=41))
    kw = {"rule": rule, "topk": 4} if rule == "topk" else {}
    st_c = sa.pool(q, k, v)
    ref = sa.forward(q, k, v, st_c, 0.6, **kw)
    for view in (_bnhd, _padded):
        qs, ks, vs = view(q), view(k), view(v)
        assert not qs.is_contiguous()
        st_s = sa.pool(qs, ks, vs)
        torch.cuda.synchronize()
        for name in ("qbar", "kbar", "vbar", "kmean", "kcov", "kbar16", "vbar16"):
            # pooled statistics: same bits (the alignment gaps between the arrays are never written)
            assert torch.equal(st_s.view(name), st_c.view(name)), name
        out = view(torch.zeros_like(q))
        got = sa.forward(qs, ks, vs, st_s, 0.6, out=out, **kw)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0])  # compares values; the layouts differ
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])


@pytest.mark.parametrize("d", [64, 128])
def test_strided_layout_matches_oracle(d):
    """The [B, N, H, d] layout (and padded rows) against the oracle directly:
    kept counts exact except near ties, out within relative L2 1e-2 and max
    abs 2e-2, lse within 1e-3."""
    import math

    import numpy as np

    from oracle import solattn_oracle as orc

    wl = Workload("s", 2, 3, d, (1, 1, 64 * 11 + 37))
    q, k, v = make_qkv(wl, seed=42)
    beta = 0.6
    out_o, lse_o, dens_o = orc.forward(q, k, v, beta)
    r = orc.route_all(q, k, beta)
    ties = (np.abs(r["shat"] - r["tau"][..., None]) <= 1e-4).sum(-1)
    for view in (_bnhd, _padded):
        qs, ks, vs = (view(x.cuda()) for x in (q, k, v))
        st = sa.pool(qs, ks, vs)
        out = view(torch.zeros_like(q, device="cuda"))
        got, lse, dens = sa.forward(qs, ks, vs, st, beta, out=out)
        torch.cuda.synchronize()
        diff = np.abs(dens.cpu().numpy().astype(np.int64) - dens_o)
        assert (diff[ties == 0] == 0).all() and (diff <= ties).all()
        og = got.float().cpu().numpy().astype(np.float64)
        err = og - out_o
        assert np.linalg.norm(err) / np.linalg.norm(out_o) <= 1e-2 and np.abs(err).max() <= 2e-2
        assert np.abs(lse.cpu().numpy() - lse_o).max() <= 1e-3
        assert math.isfinite(float(np.abs(og).max()))
