"""GPU parity of the per-token correction (solattn_forward_ex, correction=1):
skipped blocks attended as tiles of bf16 pooled keys / values, each column
weighted by n_j, against the oracle's attend(correction="token").

Acceptance as for the block-level correction: |S_i| equal except near ties;
out relative L2 <= 1e-2 and max abs <= 2e-2, lse <= 1e-3 (the pooled operands
are rounded to bf16 like q, k, v)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_cov_b200 as sa
from block_sparse_attention_cov_b200.build import build
from block_sparse_attention_cov_b200.inputs import Workload, make_qkv
from oracle import solattn_oracle as orc

pytestmark = pytest.mark.gpu

REL_L2, MAX_ABS, LSE_ABS, TIE = 1e-2, 2e-2, 1e-3, 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build()


def _check(wl, beta, seed, rule="threshold", topk=0, n_forced=0):
    q, k, v = make_qkv(wl, seed=seed)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    st = sa.pool(qd, kd, vd)
    ws = sa.workspace()
    out, lse, dens = sa.forward(qd, kd, vd, st, beta, ws=ws, rule=rule, topk=topk, n_forced=n_forced,
                                correction="token")
    assert sa.status(ws) == 0
    dens = dens.cpu().numpy()
    og, lg = out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    for b in range(wl.B):
        for h in range(wl.H):
            qq, kk, vv = (x[b, h].double().numpy() for x in (q, k, v))
            r = orc.route_rule(qq, kk, rule, beta if rule == "threshold" else topk, n_forced)
            if rule == "threshold":
                amb = (np.abs(r["shat"] - r["tau"][:, None]) <= TIE).any(1)
            else:
                kth = -np.sort(-r["shat"], axis=1)[:, max(topk, 1) - 1]
                amb = (np.abs(r["shat"] - kth[:, None]) <= TIE).sum(1) > 1
            assert not ((dens[b, h] != r["density"]) & ~amb).any()
            oo, lo, _ = orc.attend(qq, kk, vv, mask=r["mask"], correction="token")
            rows = np.zeros(wl.N, bool)
            for i in np.nonzero(~amb)[0]:
                rows[i * 64:min(wl.N, i * 64 + 64)] = True
            err = og[b, h][rows] - oo[rows]
            assert np.isfinite(og[b, h][rows]).all()
            assert np.linalg.norm(err) / np.linalg.norm(oo[rows]) <= REL_L2, np.linalg.norm(err) / np.linalg.norm(oo[rows])
            assert np.abs(err).max() <= MAX_ABS, np.abs(err).max()
            assert np.abs(lg[b, h][rows] - lo[rows]).max() <= LSE_ABS


MID2 = Workload("mid2", 1, 2, 128, (8, 32, 32))


@pytest.mark.parametrize("beta", [0.0, 0.8, 1.5, math.inf])
def test_token_correction_matches_oracle(beta):
    _check(MID2, beta, seed=61)


def test_token_correction_ragged_d64_and_rules():
    _check(Workload("r", 2, 2, 64, (1, 1, 64 * 9 + 13)), 0.6, seed=62)
    _check(Workload("r", 1, 3, 128, (1, 1, 1000)), 1.0, seed=63, n_forced=2)
    _check(MID2, 0.0, seed=64, rule="topk", topk=9)


def test_token_correction_beta_minus_inf_is_dense():
    """beta = -inf keeps every block, so no correction term remains: the
    per-token path (the one-unit kernel) gives dense attention, checked against
    the oracle's dense attention and against the dense path (the two-unit
    kernel) at the usual tolerances."""
    from oracle import solattn_oracle as orc

    wl = Workload("d", 1, 2, 128, (1, 1, 64 * 7 + 30))
    q_h, k_h, v_h = make_qkv(wl, seed=65)
    q, k, v = (x.cuda() for x in (q_h, k_h, v_h))
    st = sa.pool(q, k, v)
    o1, l1, _ = sa.forward(q, k, v, st, -math.inf, correction="token")
    o2, l2 = sa.dense(q, k, v)
    torch.cuda.synchronize()
    for h in range(wl.H):
        od, ld = orc.dense_attention(*(x[0, h].double().numpy() for x in (q_h, k_h, v_h)))
        for o, l in ((o1, l1), (o2, l2)):
            og = o[0, h].float().cpu().numpy().astype(np.float64)
            assert np.linalg.norm(og - od) / np.linalg.norm(od) <= 1e-2 and np.abs(og - od).max() <= 2e-2
            assert np.abs(l[0, h].cpu().numpy() - ld).max() <= 1e-3
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
