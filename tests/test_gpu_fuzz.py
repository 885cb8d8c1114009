"""Seeded random shapes through the C ABI: batch and head counts, d in {64,
128}, lengths from a single token to a few thousand (ragged last blocks, odd
block counts), beta drawn from a normal distribution or +-inf. Every case:
the kept mask bit-exact against the oracle (near ties counted), mu_i / sigma_i
/ tau_i within 1e-5, out within relative L2 1e-2 and max abs 2e-2 and lse
within 1e-3 of the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_cov_b200.inputs import Workload, make_qkv
from hooklib import forward_with_routing
from oracle import solattn_oracle as orc

pytestmark = pytest.mark.gpu
TIE = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    B = int(rng.integers(1, 3))
    H = int(rng.integers(1, 4))
    d = int(rng.choice([64, 128]))
    N = [1, 2, 63, 65][seed] if seed < 4 else int(rng.integers(3, 5000))
    r = rng.random()
    beta = -math.inf if r < 0.1 else (math.inf if r < 0.2 else float(rng.normal(0.5, 0.6)))
    return B, H, d, N, beta


@pytest.mark.parametrize("seed", list(range(16)))
def test_random_shapes_match_oracle(seed):
    B, H, d, N, beta = _case(seed)
    wl = Workload(f"fz{seed}", B, H, d, (1, 1, N))
    q, k, v = make_qkv(wl, seed=seed)
    out, lse, dens, mask, stats = forward_with_routing(*(x.cuda() for x in (q, k, v)), beta)
    out_o, lse_o, _ = orc.forward(q, k, v, beta)
    r = orc.route_all(q, k, beta)
    near = np.abs(r["shat"] - r["tau"][..., None]) <= TIE
    diff = mask != r["mask"]
    assert not (diff & ~near).any(), (B, H, d, N, beta)
    assert (dens.cpu().numpy() == mask.sum(-1)).all()
    fin = np.isfinite(r["tau"])
    tau = stats[..., 2].astype(np.float64)
    np.testing.assert_allclose(tau[fin], r["tau"][fin], rtol=1e-5, atol=1e-5)
    if math.isfinite(beta):
        np.testing.assert_allclose(stats[..., 0], r["mu"], rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(stats[..., 1], r["sigma"], rtol=1e-5, atol=1e-5)
    og = out.float().cpu().numpy().astype(np.float64)
    err = og - out_o
    rel = np.linalg.norm(err) / max(np.linalg.norm(out_o), 1e-30)
    dl = np.abs(lse.cpu().numpy() - lse_o).max()
    print(f"B={B} H={H} d={d} N={N} beta={beta:.3f}: rel-L2 {rel:.2e} max {np.abs(err).max():.2e} "
          f"lse {dl:.2e} near ties {int(near.sum())} flipped {int(diff.sum())}")
    assert rel <= 1e-2 and np.abs(err).max() <= 2e-2 and dl <= 1e-3


def _case_rules(seed):
    rng = np.random.default_rng(2000 + seed)
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
    d = int(rng.choice([64, 128]))
    N = int(rng.integers(2, 4000))
    nb = math.ceil(N / 64)
    rule = ["topk", "topp", "threshold", "threshold"][seed % 4]
    param = {"topk": int(rng.integers(0, nb + 2)), "topp": float(rng.uniform(0.0, 1.05)),
             "threshold": float(rng.normal(0.5, 0.6))}[rule]
    n_forced = int(rng.integers(0, 4)) if seed % 3 == 0 else 0
    correction = "token" if seed % 4 == 3 else "block"
    return B, H, d, N, rule, param, n_forced, correction


@pytest.mark.parametrize("seed", list(range(12)))
def test_random_shapes_other_rules_and_token_correction(seed):
    """Top-k (k from 0 past N_b), top-p (p from 0 past 1), the threshold with
    forced leading blocks and with the per-token correction, on random
    shapes: the kept mask against the oracle's rule (ties at the cut
    counted), and the output against the oracle fed the kernel's kept sets
    (external-mask mode, so that a tie decided the other way cannot move it)."""
    from test_gpu_mask import _rule_near

    B, H, d, N, rule, param, n_forced, correction = _case_rules(seed)
    wl = Workload(f"fr{seed}", B, H, d, (1, 1, N))
    q, k, v = make_qkv(wl, seed=100 + seed)
    kw = {"topk": param} if rule == "topk" else ({"topp": param} if rule == "topp" else {})
    beta = param if rule == "threshold" else 0.0
    out, lse, dens, mask, _ = forward_with_routing(*(x.cuda() for x in (q, k, v)), beta, rule=rule,
                                                   n_forced=n_forced, correction=correction, **kw)
    flips = 0
    for b in range(B):
        for h in range(H):
            r = orc.route_rule(q[b, h].double().numpy(), k[b, h].double().numpy(), rule, param, n_forced)
            near = _rule_near(r, rule, param, N)
            if n_forced:
                assert mask[b, h][:, :min(n_forced, mask.shape[-1])].all()
                near[:, :n_forced] = False
            diff = mask[b, h] != r["mask"]
            assert not (diff & ~near).any(), (seed, b, h, np.argwhere(diff & ~near)[:5])
            flips += int(diff.sum())
    assert (dens.cpu().numpy() == mask.sum(-1)).all()
    out_o, lse_o, _ = orc.forward(q, k, v, beta, masks=mask, correction=correction)
    og = out.float().cpu().numpy().astype(np.float64)
    err = og - out_o
    rel = np.linalg.norm(err) / max(np.linalg.norm(out_o), 1e-30)
    dl = np.abs(lse.cpu().numpy() - lse_o).max()
    print(f"B={B} H={H} d={d} N={N} {rule}({param:.3f}) forced={n_forced} {correction}: rel-L2 {rel:.2e} "
          f"max {np.abs(err).max():.2e} lse {dl:.2e} flipped {flips}")
    assert rel <= 1e-2 and np.abs(err).max() <= 2e-2 and dl <= 1e-3


@pytest.mark.parametrize("seed", list(range(6)))
def test_random_strided_layouts(seed):
    """Random shapes in a strided layout (the [B, N, H, d] order seen through a
    permute, or rows padded by 8 to 40 elements): pooled statistics and
    forward outputs equal the contiguous layout's bit for bit, and match the
    oracle."""
    import block_sparse_attention_cov_b200 as sa

    rng = np.random.default_rng(3000 + seed)
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
    d = int(rng.choice([64, 128]))
    N = int(rng.integers(2, 3000))
    beta = float(rng.normal(0.5, 0.5))
    pad = int(rng.choice([8, 16, 24, 40]))
    wl = Workload(f"fs{seed}", B, H, d, (1, 1, N))
    q, k, v = (x.cuda() for x in make_qkv(wl, seed=200 + seed))

    def view(x):
        if seed % 2 == 0:
            return x.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        base = torch.zeros((B, H, N, d + pad), dtype=x.dtype, device=x.device)
        base[..., :d] = x
        return base[..., :d]

    st_c = sa.pool(q, k, v)
    ref = sa.forward(q, k, v, st_c, beta)
    qs, ks, vs = view(q), view(k), view(v)
    st_s = sa.pool(qs, ks, vs)
    out = view(torch.zeros_like(q))
    got = sa.forward(qs, ks, vs, st_s, beta, out=out)
    torch.cuda.synchronize()
    for name in ("qbar", "kbar", "vbar", "kmean", "kcov", "kbar16", "vbar16"):
        assert torch.equal(st_s.view(name), st_c.view(name)), name  # the alignment gaps are never written
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
    out_o, lse_o, dens_o = orc.forward(q.cpu(), k.cpu(), v.cpu(), beta)
    r = orc.route_all(q.cpu(), k.cpu(), beta)
    ties = (np.abs(r["shat"] - r["tau"][..., None]) <= TIE).sum(-1)
    diff = np.abs(got[2].cpu().numpy().astype(np.int64) - dens_o)
    assert (diff[ties == 0] == 0).all() and (diff <= ties).all()
    err = got[0].float().cpu().numpy().astype(np.float64) - out_o
    rel = np.linalg.norm(err) / np.linalg.norm(out_o)
    print(f"B={B} H={H} d={d} N={N} {'bnhd' if seed % 2 == 0 else f'pad {pad}'}: rel-L2 {rel:.2e}")
    assert rel <= 1e-2 and np.abs(err).max() <= 2e-2
    assert np.abs(got[1].cpu().numpy() - lse_o).max() <= 1e-3
