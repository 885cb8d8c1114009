"""GPU parity of the other kept-set rules (top-k, top-p) and of always-kept
prefix blocks, through solattn_forward_ex, against the oracle's route_rule.

Acceptance as for the threshold rule: per query block |S_i| equals the
oracle's, except where the cut is a near tie in fp64 (top-k: another score
within 1e-4 of the k-th largest; top-p: the cumulative mass crosses p within
1e-4 of the total at the cut); out relative L2 <= 1e-2, max abs <= 2e-2 and
lse <= 1e-3 on the query blocks without a near tie.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_cov_b200 as sa
from block_sparse_attention_cov_b200.build import build
from block_sparse_attention_cov_b200.inputs import WORKLOADS, Workload, make_qkv
from oracle import solattn_oracle as orc

pytestmark = pytest.mark.gpu

REL_L2, MAX_ABS, LSE_ABS, TIE = 1e-2, 2e-2, 1e-3, 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build()


def _ambiguous(r, rule, param, N):
    """Per query block: True where the oracle's cut is a near tie."""
    shat = r["shat"]
    nb = shat.shape[1]
    amb = np.zeros(nb, bool)
    if rule == "topk":
        kk = int(param)
        if 0 < kk < nb:
            kth = -np.sort(-shat, axis=1)[:, kk - 1]
            amb = (np.abs(shat - kth[:, None]) <= TIE).sum(1) > 1
    elif rule == "topp":
        if 0.0 < param < 1.0:
            n = orc.block_counts(N).astype(np.float64)
            for i in range(nb):
                order = np.argsort(-shat[i], kind="stable")
                w = n[order] * np.exp(shat[i, order] - shat[i, order[0]])
                cum = np.cumsum(w) - param * w.sum()   # increasing; crosses 0 at the cut
                kp = min(int(np.searchsorted(cum, 0.0, side="left")), nb - 1)
                vstar = shat[i, order[kp]]
                amb[i] = (np.abs(cum) <= TIE * w.sum()).any() or (np.abs(shat[i] - vstar) <= TIE).sum() > 1
    else:
        amb = (np.abs(shat - r["tau"][:, None]) <= TIE).any(1)
    return amb


def _check(wl, rule, param, n_forced, seed):
    q, k, v = make_qkv(wl, seed=seed)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    st = sa.pool(qd, kd, vd)
    ws = sa.workspace()
    kw = {"rule": rule, "n_forced": n_forced}
    if rule == "topk":
        kw["topk"] = int(param)
    elif rule == "topp":
        kw["topp"] = float(param)
    beta = param if rule == "threshold" else 0.0
    out, lse, dens = sa.forward(qd, kd, vd, st, beta, ws=ws, **kw)
    assert sa.status(ws) == 0
    dens = dens.cpu().numpy()
    og, lg = out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    checked = 0
    for b in range(wl.B):
        for h in range(wl.H):
            qq, kk, vv = (x[b, h].double().numpy() for x in (q, k, v))
            r = orc.route_rule(qq, kk, rule, param, n_forced)
            amb = _ambiguous(r, rule, param, wl.N)
            diff = dens[b, h] != r["density"]
            assert not (diff & ~amb).any(), (rule, param, np.nonzero(diff & ~amb))
            oo, lo, _ = orc.attend(qq, kk, vv, mask=r["mask"])
            rows = np.zeros(wl.N, bool)
            for i in np.nonzero(~amb)[0]:
                rows[i * 64:min(wl.N, i * 64 + 64)] = True
            if rows.any():
                err = og[b, h][rows] - oo[rows]
                assert np.isfinite(og[b, h][rows]).all()
                assert np.linalg.norm(err) / np.linalg.norm(oo[rows]) <= REL_L2
                assert np.abs(err).max() <= MAX_ABS
                assert np.abs(lg[b, h][rows] - lo[rows]).max() <= LSE_ABS
                checked += int(rows.sum())
    assert checked > 0


def _wl(B, H, d, N):
    return Workload(f"r{B}x{H}x{N}x{d}", B, H, d, (1, 1, N))


MID2 = Workload("mid2", 1, 2, 128, (8, 32, 32))


@pytest.mark.parametrize("kk", [0, 1, 5, 19, 128, 500])
def test_topk_matches_oracle(kk):
    _check(MID2, "topk", kk, 0, seed=21)


@pytest.mark.parametrize("p", [0.0, 0.3, 0.6, 0.9, 1.0])
def test_topp_matches_oracle(p):
    _check(MID2, "topp", p, 0, seed=22)


@pytest.mark.parametrize("rule,param,n_forced", [("threshold", 1.0, 3), ("threshold", math.inf, 2),
                                                 ("topk", 4, 5), ("topp", 0.5, 1)])
def test_forced_blocks_match_oracle(rule, param, n_forced):
    _check(MID2, rule, param, n_forced, seed=23)


@pytest.mark.parametrize("rule,param", [("topk", 3), ("topp", 0.7)])
def test_rules_ragged_and_d64(rule, param):
    _check(_wl(2, 2, 64, 64 * 9 + 13), rule, param, 1, seed=24)
    _check(_wl(1, 3, 128, 1000), rule, param, 0, seed=25)


def test_topk_all_blocks_equals_dense_attention():
    """top-k with k = N_b keeps every block: dense attention, checked against the
    oracle's dense attention and against the dense path (which runs on the
    two-unit kernel; top-k on the one-unit kernel) at the usual tolerances."""
    wl = _wl(1, 2, 128, 64 * 7 + 9)
    q_h, k_h, v_h = make_qkv(wl, seed=26)
    q, k, v = (x.cuda() for x in (q_h, k_h, v_h))
    st = sa.pool(q, k, v)
    o1, l1, d1 = sa.forward(q, k, v, st, rule="topk", topk=8)
    o2, l2 = sa.dense(q, k, v)
    torch.cuda.synchronize()
    assert (d1.cpu() == 8).all()
    for h in range(wl.H):
        od, ld = orc.dense_attention(*(x[0, h].double().numpy() for x in (q_h, k_h, v_h)))
        for o, l in ((o1, l1), (o2, l2)):
            og = o[0, h].float().cpu().numpy().astype(np.float64)
            assert np.linalg.norm(og - od) / np.linalg.norm(od) <= REL_L2 and np.abs(og - od).max() <= MAX_ABS
            assert np.abs(l[0, h].cpu().numpy() - ld).max() <= LSE_ABS
