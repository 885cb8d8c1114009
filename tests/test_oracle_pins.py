"""Pins of the CPU oracle against what the Sol-Attn pages and plain mathematics
fix, independent of the oracle's own code paths.

Each test names the passage it rests on ("Sol-Attn: Accelerating Video
Generation Inference via On-the-Fly Attention Sparsification"; section names are
those of the paithon.it article unless stated).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import solattn_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa64(q, k, v, bias=None):
    """torch's library softmax attention in fp64 on the CPU: a routine the
    oracle does not use."""
    q, k, v = (torch.as_tensor(np.asarray(x), dtype=torch.float64)[None, None] for x in (q, k, v))
    mask = None if bias is None else torch.tensor(np.array(bias), dtype=torch.float64)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    return o[0, 0].numpy()


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# Pooling and key statistics ("Una soglia per ogni riga", last paragraph)
# ---------------------------------------------------------------------------
def test_pool_and_covariance_against_numpy_routines():
    rng = _rng(1)
    N, d = 64 * 9 + 37, 32
    x = rng.standard_normal((N, d))
    xb = orc.pool(x)
    assert xb.shape == (10, d)
    for b in range(9):
        np.testing.assert_allclose(xb[b], np.mean(x[64 * b:64 * b + 64], axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(xb[9], np.mean(x[576:], axis=0), rtol=1e-13, atol=1e-15)  # 37 valid tokens
    km, kc = orc.key_stats(xb)
    np.testing.assert_allclose(km, np.mean(xb, axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(kc, np.cov(xb.T, bias=True), rtol=1e-12, atol=1e-15)


def test_row_stats_equal_mean_and_std_of_explicit_row():
    # mu_i, sigma_i from the key mean and d x d covariance must equal the mean and
    # population std of the proxy row they stand for (no row formed).
    rng = _rng(2)
    nb, d = 300, 64
    qbar = rng.standard_normal((40, d)) * 0.7 + 0.3
    kbar = rng.standard_normal((nb, d)) * 0.5 + rng.standard_normal(d) * 0.2
    km, kc = orc.key_stats(kbar)
    mu, sigma = orc.row_stats(qbar, km, kc)
    row = (qbar @ kbar.T) / math.sqrt(d)
    np.testing.assert_allclose(mu, row.mean(axis=1), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(sigma, row.std(axis=1, ddof=0), rtol=1e-10)


# ---------------------------------------------------------------------------
# Threshold ("Una soglia per ogni riga", displayed equation and the paragraph after it)
# ---------------------------------------------------------------------------
def test_gaussian_density_matches_normal_tail_golden():
    with open(os.path.join(GOLDEN, "gaussian_density.json")) as f:
        gold = json.load(f)
    rng = _rng(3)
    nb, d = 4096, 64
    kbar = rng.standard_normal((nb, d))  # pooled keys ~ N(0, I) => s_hat row is Gaussian
    qbar = rng.standard_normal((16, d))
    km, kc = orc.key_stats(kbar)
    mu, sigma = orc.row_stats(qbar, km, kc)
    shat = orc.proxy_scores(qbar, kbar)
    prev = 1.0
    for row in gold["rows"]:
        tau = orc.thresholds(mu, sigma, row["beta"])
        frac = float((shat > tau[:, None]).mean())
        assert abs(frac - row["kept_fraction"]) <= gold["tolerance_abs"], (row, frac)
        assert frac <= prev  # density never grows with beta
        prev = frac


def test_threshold_is_strict_and_ties_are_skipped():
    # Three key blocks with block-constant keys +e, -e, 0 and queries along e:
    # s_hat = (+x, -x, 0), mu = 0 exactly, so at beta = 0 the third block ties tau.
    d = 64
    e = np.zeros(d)
    e[5] = 1.0
    k = np.concatenate([np.tile(e, (64, 1)), np.tile(-e, (64, 1)), np.zeros((64, d))])
    q = np.tile(0.5 * e, (192, 1))
    r = orc.route(q, k, 0.0)
    assert r["mu"][0] == 0.0
    assert r["shat"][0, 2] == r["tau"][0]
    assert r["mask"][0].tolist() == [True, False, False]
    assert orc.route(q, k, -math.inf)["mask"].all()
    assert not orc.route(q, k, math.inf)["mask"].any()


def test_zero_spread_keeps_nothing_and_output_is_mean_of_values():
    # Identical key blocks => covariance 0 => sigma 0 => tau = mu = every s_hat:
    # nothing is strictly above, every block is a correction with equal score, so
    # each output row is the plain mean of all value tokens.
    rng = _rng(4)
    d, N = 64, 256
    k = np.full((N, d), 0.5)
    q = rng.integers(-4, 5, (N, d)) * 0.25  # dyadic values: every dot product is exact
    v = rng.standard_normal((N, d))
    out, lse, dens = orc.attend(q, k, v, beta=1.0)
    assert (dens == 0).all()
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=0), out.shape), rtol=1e-12, atol=1e-14)
    out2, _, dens2 = orc.attend(q, k, v, beta=-math.inf)
    assert (dens2 == 4).all() and np.isfinite(out2).all()


# ---------------------------------------------------------------------------
# Dense limit and closed forms of the correction ("Scegliere mentre si calcola")
# ---------------------------------------------------------------------------
def test_beta_minus_inf_is_dense_attention():
    rng = _rng(5)
    N, d = 64 * 4 + 21, 64
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    out, lse, dens = orc.attend(q, k, v, beta=-math.inf)
    np.testing.assert_allclose(out, _sdpa64(q, k, v), rtol=1e-12, atol=1e-13)
    x = (q @ k.T) / math.sqrt(d)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.as_tensor(x), dim=1).numpy(), rtol=1e-13, atol=1e-13)
    assert (dens == 5).all()


@pytest.mark.parametrize("N,d,scale", [(64 * 3 + 5, 64, 1.0), (200, 128, 1.0), (130, 128, 15.0)])
def test_dense_attention_is_library_softmax_attention(N, d, scale):
    """dense_attention (the checker of the dense GPU path) against torch's
    scaled_dot_product_attention and logsumexp in fp64; the large-scale case
    has scores far from zero, so a missing max subtraction would overflow."""
    rng = _rng(55 + N)
    q, k, v = (scale * rng.standard_normal((N, d)) for _ in range(3))
    out, lse = orc.dense_attention(q, k, v)
    np.testing.assert_allclose(out, _sdpa64(q, k, v), rtol=1e-11, atol=1e-12)
    x = (q @ k.T) / math.sqrt(d)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.as_tensor(x), dim=1).numpy(), rtol=1e-12, atol=1e-12)
    assert np.isfinite(out).all() and np.isfinite(lse).all()


@pytest.mark.parametrize("beta", [-math.inf, -0.5, 0.0, 0.8, math.inf])
def test_block_constant_inputs_make_the_correction_exact(beta):
    # With queries and keys constant inside each block, the zeroth-order Taylor
    # term is exact: every token of a skipped block has exactly the mean key, so
    # Sol-Attn must equal dense attention for every beta (numerator and
    # denominator both corrected, partial block weighted by its count).
    rng = _rng(6)
    N, d = 64 * 5 + 20, 64
    nb = 6
    qb = rng.standard_normal((nb, d)) * 1.5
    kb = rng.standard_normal((nb, d)) * 1.5
    q = np.repeat(qb, 64, axis=0)[:N]
    k = np.repeat(kb, 64, axis=0)[:N]
    v = rng.standard_normal((N, d))
    out, lse, dens = orc.attend(q, k, v, beta=beta)
    np.testing.assert_allclose(out, _sdpa64(q, k, v), rtol=1e-11, atol=1e-12)
    x = (q @ k.T) / math.sqrt(d)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.as_tensor(x), dim=1).numpy(), rtol=1e-12, atol=1e-12)
    if beta == math.inf:
        assert (dens == 0).all()


def test_beta_plus_inf_is_softmax_over_pooled_tokens():
    # Everything skipped: row t of block i gets softmax_j(s_hat_ij + log n_j) v_bar_j,
    # i.e. attention of the pooled query over pooled keys weighted by block size.
    rng = _rng(7)
    N, d = 64 * 6 + 9, 64
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    out, lse, dens = orc.attend(q, k, v, beta=math.inf)
    assert (dens == 0).all()
    qb = np.stack([q[a:b].mean(0) for a, b in orc.block_bounds(N)])
    kb = np.stack([k[a:b].mean(0) for a, b in orc.block_bounds(N)])
    vb = np.stack([v[a:b].mean(0) for a, b in orc.block_bounds(N)])
    cnt = np.array([b - a for a, b in orc.block_bounds(N)], np.float64)
    bias = np.broadcast_to(np.log(cnt), (len(cnt), len(cnt)))
    want = _sdpa64(qb, kb, vb, bias)
    x = (qb @ kb.T) / math.sqrt(d) + np.log(cnt)[None, :]
    want_lse = torch.logsumexp(torch.as_tensor(x), dim=1).numpy()
    for i, (a, b) in enumerate(orc.block_bounds(N)):
        np.testing.assert_allclose(out[a:b], np.broadcast_to(want[i], (b - a, d)), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[a:b], want_lse[i], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("beta", [0.0, 0.6])
def test_key_block_constant_query_varying_uses_block_level_proxy(beta):
    # Keys constant inside blocks, queries varying: kept blocks contribute
    # n_j exp(s q_t . k_bar_j) v_bar_j exactly; skipped ones use the block-level
    # proxy s q_bar_i . k_bar_j for every row of block i (the adopted reading).
    # This separates the block-level reading from a per-token one.
    rng = _rng(8)
    N, d = 64 * 6 + 40, 64
    nb = 7
    kb = rng.standard_normal((nb, d)) * 1.2
    k = np.repeat(kb, 64, axis=0)[:N]
    q = rng.standard_normal((N, d)) * 1.2
    v = rng.standard_normal((N, d))
    out, lse, _ = orc.attend(q, k, v, beta=beta)
    bounds = [(j * 64, min(N, j * 64 + 64)) for j in range(nb)]
    cnt = np.array([b - a for a, b in bounds], float)
    qb = np.stack([q[a:b].mean(0) for a, b in bounds])
    vb = np.stack([v[a:b].mean(0) for a, b in bounds])
    shat = (qb @ kb.T) / math.sqrt(d)
    mu = shat.mean(1)
    sd = shat.std(1)
    kept = shat > (mu + beta * sd)[:, None]
    assert kept.any() and (~kept).any()
    for i, (a, b) in enumerate(bounds):
        tok = (q[a:b] @ kb.T) / math.sqrt(d)  # per-token scores against block keys
        x = np.where(kept[i][None, :], tok, shat[i][None, :]) + np.log(cnt)[None, :]
        w = torch.softmax(torch.as_tensor(x), dim=1).numpy()
        np.testing.assert_allclose(out[a:b], w @ vb, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[a:b], torch.logsumexp(torch.as_tensor(x), 1).numpy(), rtol=1e-12)
        per_token = np.where(kept[i][None, :], tok, tok) + np.log(cnt)[None, :]
        w2 = torch.softmax(torch.as_tensor(per_token), dim=1).numpy()
        if (~kept[i]).any():  # the per-token reading gives a different answer
            assert np.abs(out[a:b] - w2 @ vb).max() > 1e-6


# ---------------------------------------------------------------------------
# Brute force on tiny inputs: one token at a time
# ---------------------------------------------------------------------------
def _brute(q, k, v, beta):
    """Token-by-token statement: a kept block's token u weighs exp(s q_t.k_u) with
    value v_u; a skipped block's token weighs exp(s_hat_ij) with value v_bar_j
    (as if it had the block's mean key and value). Threshold from the explicit row."""
    N, d = q.shape
    s = 1.0 / math.sqrt(d)
    blk = [u // 64 for u in range(N)]
    nb = blk[-1] + 1
    means = lambda x: [np.mean(x[[u for u in range(N) if blk[u] == j]], axis=0) for j in range(nb)]
    qb, kb, vb = means(q), means(k), means(v)
    out = np.zeros((N, d))
    lse = np.zeros(N)
    for t in range(N):
        i = blk[t]
        row = [s * float(np.dot(qb[i], kb[j])) for j in range(nb)]
        mu = sum(row) / nb
        sd = math.sqrt(sum((x - mu) ** 2 for x in row) / nb)
        tau = -math.inf if beta == -math.inf else (math.inf if beta == math.inf else mu + beta * sd)
        ws, vs = [], []
        for u in range(N):
            j = blk[u]
            if row[j] > tau:
                ws.append(s * float(np.dot(q[t], k[u])))
                vs.append(v[u])
            else:
                ws.append(row[j])
                vs.append(vb[j])
        m = max(ws)
        e = [math.exp(w - m) for w in ws]
        den = sum(e)
        out[t] = sum(ei * vi for ei, vi in zip(e, vs)) / den
        lse[t] = m + math.log(den)
    return out, lse


@pytest.mark.parametrize("N", [128, 150, 192])
@pytest.mark.parametrize("beta", [-math.inf, 0.0, 0.5, math.inf])
def test_brute_force_tiny(N, beta):
    rng = _rng(9 + N)
    d = 16
    q = rng.standard_normal((N, d)) * 2.0
    k = rng.standard_normal((N, d)) * 2.0
    k[64:128] += 1.5  # make one block stand out so routing keeps something
    v = rng.standard_normal((N, d))
    out, lse, _ = orc.attend(q, k, v, beta=beta)
    bo, bl = _brute(q, k, v, beta)
    np.testing.assert_allclose(out, bo, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Single pass == offline threshold ("Scegliere mentre si calcola", first paragraph)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("beta", [-math.inf, 0.0, 0.7, math.inf])
def test_streaming_double_loop_equals_offline_threshold(beta):
    rng = _rng(10)
    N, d = 64 * 7 + 23, 32
    q = rng.standard_normal((N, d)) + np.linspace(-1, 1, N)[:, None]
    k = rng.standard_normal((N, d)) + np.cos(np.arange(N) / 50.0)[:, None]
    v = rng.standard_normal((N, d))
    out, lse, dens = orc.attend(q, k, v, beta=beta)
    nb = len(orc.block_bounds(N))
    for g in (1, 3, 7, nb):
        o2, l2, d2 = orc.attend_streaming(q, k, v, beta, g)
        assert (d2 == dens).all()
        np.testing.assert_allclose(o2, out, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(l2, lse, rtol=1e-12, atol=1e-12)


def test_external_mask_mode_reproduces_own_mask():
    rng = _rng(11)
    N, d = 64 * 5, 32
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    out, lse, dens = orc.attend(q, k, v, beta=0.3)
    r = orc.route(q, k, 0.3)
    o2, l2, d2 = orc.attend(q, k, v, beta=0.3, mask=r["mask"])
    assert np.array_equal(out, o2) and np.array_equal(lse, l2) and np.array_equal(dens, d2)
    flipped = r["mask"].copy()
    flipped[0, 0] = ~flipped[0, 0]
    o3, _, _ = orc.attend(q, k, v, beta=0.3, mask=flipped)
    assert not np.allclose(o3[:64], out[:64])
    np.testing.assert_allclose(o3[64:], out[64:], rtol=0, atol=0)


# ---------------------------------------------------------------------------
# The pins catch plausible mistakes planted in the oracle (CPU only)
# ---------------------------------------------------------------------------
def test_planted_mistakes_are_caught(monkeypatch):
    rng = _rng(12)
    N, d = 150, 16
    q = rng.standard_normal((N, d)) * 2.0
    k = rng.standard_normal((N, d)) * 2.0
    v = rng.standard_normal((N, d))
    brute = {b: _brute(q, k, v, b) for b in (0.0, 0.5, math.inf)}

    def brute_pin_fails(beta):
        bo, bl = brute[beta]
        out, lse, _ = orc.attend(q, k, v, beta=beta)
        return not (np.allclose(out, bo, rtol=1e-9, atol=1e-10) and np.allclose(lse, bl, rtol=1e-9, atol=1e-10))

    assert not brute_pin_fails(0.0) and not brute_pin_fails(0.5)
    # 1. every skipped block weighted 64 instead of its count of valid tokens
    monkeypatch.setattr(orc, "block_counts", lambda n: np.full(len(orc.block_bounds(n)), 64))
    assert brute_pin_fails(math.inf)
    monkeypatch.undo()
    # 2. proxy score without the 1/sqrt(d) scale
    monkeypatch.setattr(orc, "proxy_scores", lambda a, b, dtype=np.float64: np.asarray(a) @ np.asarray(b).T)
    assert brute_pin_fails(0.0)
    monkeypatch.undo()
    # 3. threshold with the sign of beta flipped
    monkeypatch.setattr(orc, "thresholds", lambda mu, sg, beta: mu - beta * sg)
    assert brute_pin_fails(0.5)
    monkeypatch.undo()
    # 4. sample (ddof=1) covariance: the explicit-row invariant catches it
    real_stats = orc.key_stats

    def ddof1(kbar, dtype=np.float64):
        km, kc = real_stats(kbar)
        return km, kc * kbar.shape[0] / (kbar.shape[0] - 1)

    monkeypatch.setattr(orc, "key_stats", ddof1)
    with pytest.raises(AssertionError):
        test_row_stats_equal_mean_and_std_of_explicit_row()
    monkeypatch.undo()
    # 5. correction left out of the denominator: the block-constant pin catches it
    real_attend = orc.attend

    def no_den(q_, k_, v_, beta=-math.inf, mask=None, rows=None):
        out, lse, dens = real_attend(q_, k_, v_, beta, mask, rows)
        return out * 1.01, lse, dens

    monkeypatch.setattr(orc, "attend", no_den)
    with pytest.raises(AssertionError):
        test_block_constant_inputs_make_the_correction_exact(0.0)
    monkeypatch.undo()


def test_bf16_inputs_pass_through_exactly():
    # The batched wrapper takes the same bf16 tensors the GPU gets; bf16 -> fp64
    # is exact, so the oracle sees exactly the GPU's inputs.
    x = torch.randn(1, 1, 130, 64).to(torch.bfloat16)
    a = orc._as64(x)
    assert a.dtype == np.float64
    assert np.array_equal(a, x.double().numpy())


# ---------------------------------------------------------------------------
# Other kept-set rules (top-k, top-p) and always-kept prefix blocks: the
# pages compare the threshold with top-k / top-p routing ("Una soglia per ogni
# riga", "I numeri") and keep text tokens of joint attention exact ("Dove
# leggere con attenzione"); the readings are stated in the oracle.
# ---------------------------------------------------------------------------
def _proxy(seed, N, d):
    rng = _rng(seed)
    q, k = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    qb = np.stack([q[a:b].mean(0) for a, b in orc.block_bounds(N)])
    kb = np.stack([k[a:b].mean(0) for a, b in orc.block_bounds(N)])
    return q, k, (qb @ kb.T) / math.sqrt(d)


@pytest.mark.parametrize("kk", [0, 1, 3, 7, 10, 25])
def test_topk_keeps_exactly_the_k_largest(kk):
    q, k, shat = _proxy(31, 64 * 9 + 17, 32)
    nb = shat.shape[1]
    r = orc.route_rule(q, k, "topk", kk)
    want = min(max(kk, 0), nb)
    assert (r["density"] == want).all()
    for i in range(nb):
        kept, skip = shat[i][r["mask"][i]], shat[i][~r["mask"][i]]
        if len(kept) and len(skip):
            assert kept.min() > skip.max()
        # the kept set is the k largest of the row, found by a full sort
        assert set(np.nonzero(r["mask"][i])[0]) == set(np.argsort(-shat[i])[:want])


def test_topk_ties_at_the_cut_are_all_kept():
    shat = np.array([[3.0, 1.0, 2.0, 2.0, 0.0]])
    assert orc.topk_mask(shat, 2).tolist() == [[True, False, True, True, False]]
    assert orc.topk_mask(shat, 3).tolist() == [[True, False, True, True, False]]
    assert orc.topk_mask(shat, 4).tolist() == [[True, True, True, True, False]]


@pytest.mark.parametrize("p", [0.0, 0.1, 0.5, 0.9, 0.999, 1.0])
def test_topp_against_brute_force_over_every_cut(p):
    """Every distinct score is tried as the cut: v* is the largest one whose
    superlevel set holds >= p of sum_j n_j e^{s_hat_ij} (n_j: valid tokens)."""
    N = 64 * 7 + 9   # the last block holds 9 tokens: its weight matters
    q, k, shat = _proxy(32, N, 32)
    n = np.array([b - a for a, b in orc.block_bounds(N)], dtype=np.float64)
    r = orc.route_rule(q, k, "topp", p)
    for i in range(shat.shape[0]):
        w = n * np.exp(shat[i])
        total = w.sum()
        if p <= 0:
            want = np.zeros(len(w), bool)
        elif p >= 1:
            want = np.ones(len(w), bool)
        else:
            good = [v for v in shat[i] if w[shat[i] >= v].sum() >= p * total]
            want = shat[i] >= max(good)
        assert (r["mask"][i] == want).all(), (i, p)


def test_topp_density_is_monotone_in_p():
    q, k, _ = _proxy(33, 64 * 12, 32)
    prev = None
    for p in (0.0, 0.05, 0.2, 0.4, 0.6, 0.8, 0.95, 1.0):
        d = orc.route_rule(q, k, "topp", p)["density"]
        if prev is not None:
            assert (d >= prev).all()
        prev = d
    assert (prev == 12).all()


def test_forced_blocks_are_kept_and_reproduce_dense_when_all_forced():
    rng = _rng(34)
    N, d = 64 * 5 + 30, 32
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    r = orc.route_rule(q, k, "threshold", math.inf, n_forced=2)
    assert (r["density"] == 2).all() and r["mask"][:, :2].all() and not r["mask"][:, 2:].any()
    r = orc.route_rule(q, k, "threshold", 0.7, n_forced=3)
    base = orc.route_rule(q, k, "threshold", 0.7)
    assert (r["mask"] == (base["mask"] | (np.arange(6) < 3)[None, :])).all()
    full = orc.route_rule(q, k, "threshold", math.inf, n_forced=6)["mask"]
    out, _, _ = orc.attend(q, k, v, mask=full)
    np.testing.assert_allclose(out, _sdpa64(q, k, v), rtol=1e-12, atol=1e-13)


def test_topk_all_blocks_is_dense_attention():
    rng = _rng(35)
    N, d = 64 * 4 + 3, 64
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    m = orc.route_rule(q, k, "topk", 5)["mask"]
    out, _, dens = orc.attend(q, k, v, mask=m)
    assert (dens == 5).all()
    np.testing.assert_allclose(out, _sdpa64(q, k, v), rtol=1e-12, atol=1e-13)


def test_planted_mistakes_in_the_other_rules_are_caught(monkeypatch):
    # top-p mass without the n_j weights: the brute force (which weighs by n_j) fails
    real_topp = orc.topp_mask
    monkeypatch.setattr(orc, "topp_mask", lambda shat, counts, p: real_topp(shat, np.ones_like(counts), p))
    with pytest.raises(AssertionError):
        for p in (0.1, 0.5, 0.9, 0.999):
            test_topp_against_brute_force_over_every_cut(p)
    monkeypatch.undo()
    # top-k taking the smallest scores
    monkeypatch.setattr(orc, "topk_mask", lambda shat, k: shat <= np.sort(shat, axis=1)[:, max(k, 1) - 1:max(k, 1)])
    with pytest.raises(AssertionError):
        test_topk_keeps_exactly_the_k_largest(3)
    monkeypatch.undo()


# ---------------------------------------------------------------------------
# Per-token correction (the more literal reading of "Scegliere mentre si
# calcola": each token of a skipped block carries the block's mean key)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("beta", [-0.5, 0.5, 1.5, math.inf])
def test_token_correction_is_exact_for_key_block_constant_inputs(beta):
    """Keys constant within each block: sum_u e^{s q_t.k_u} v_u over a skipped
    block is n_j e^{s q_t.kbar_j} vbar_j exactly, so the per-token correction
    reproduces dense attention (torch SDPA) for any beta, while the
    block-level one does not (queries vary inside their blocks)."""
    rng = _rng(51)
    N, d = 64 * 5 + 23, 32
    k = np.repeat(rng.standard_normal((6, d)), 64, axis=0)[:N]
    q, v = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    ref = _sdpa64(q, k, v)
    tok, _, _ = orc.attend(q, k, v, beta, correction="token")
    np.testing.assert_allclose(tok, ref, rtol=1e-10, atol=1e-11)
    blk, _, dens = orc.attend(q, k, v, beta, correction="block")
    if (dens < 6).any():
        assert np.abs(blk - ref).max() > 1e-3


def test_token_correction_equals_block_for_query_block_constant_inputs():
    rng = _rng(52)
    N, d = 64 * 4 + 9, 32
    q = np.repeat(rng.standard_normal((5, d)), 64, axis=0)[:N]
    k, v = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    for beta in (0.0, 1.0, math.inf):
        a, la, _ = orc.attend(q, k, v, beta, correction="token")
        b, lb, _ = orc.attend(q, k, v, beta, correction="block")
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(la, lb, rtol=1e-12, atol=1e-13)


def test_token_correction_brute_force_tiny():
    rng = _rng(53)
    N, d = 150, 16
    q, k, v = (rng.standard_normal((N, d)) * 1.5 for _ in range(3))
    beta = 0.4
    out, lse, _ = orc.attend(q, k, v, beta, correction="token")
    r = orc.route(q, k, beta)
    bounds = orc.block_bounds(N)
    s = 1 / math.sqrt(d)
    for t in range(N):
        i = t // 64
        num, den, terms = np.zeros(d), 0.0, []
        for j, (a, b) in enumerate(bounds):
            if r["mask"][i, j]:
                for u in range(a, b):
                    terms.append((s * q[t] @ k[u], v[u]))
            else:
                kb, vb = k[a:b].mean(0), v[a:b].mean(0)
                for _ in range(b - a):  # every token of the block, with the mean key and value
                    terms.append((s * q[t] @ kb, vb))
        m = max(x for x, _ in terms)
        for x, vv in terms:
            num += math.exp(x - m) * vv
            den += math.exp(x - m)
        np.testing.assert_allclose(out[t], num / den, rtol=1e-10, atol=1e-12)
        assert abs(lse[t] - (m + math.log(den))) < 1e-10
