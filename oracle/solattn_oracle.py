"""Sol-Attn oracle: a plain, slow, fp64 CPU statement of what the attention
forward computes.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this module: only the tests, the smoke check and the benchmark's CPU-baseline
leg use it. It shares no code with the CUDA path (no kernels, helpers, tables
or constants); the only thing both sides share is the seeded input generator,
which holds none of the method's arithmetic.

Source: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
Attention Sparsification" (arXiv 2607.24027), as described on the pages
hotpaper.ai (abstract), agihunt.info (English digest) and paithon.it (Italian
article). Section names below are those pages' headings.

Steps, in the pages' order and notation (s = 1/sqrt(d), 64-token blocks):

 1. blocks      -- the sequence is cut into blocks of 64 tokens; block b holds
                   tokens [64b, min(64b+64, N)), n_b of them
                   (paithon.it, "Perché l'attenzione pesa tanto nei video").
 2. pool        -- proxy inputs are block means of the queries and keys (same
                   section: "il prodotto fra la media delle query del blocco e
                   la media delle chiavi"); value means serve the correction.
 3. key stats   -- mean of the pooled keys and their d x d second-moment
                   (covariance) matrix (paithon.it, "Una soglia per ogni
                   riga", last paragraph).
 4. row stats   -- mu_i, sigma_i = mean and standard deviation of the proxy
                   row {s_hat_ij}_j, obtained from step 3 without forming the
                   row (same paragraph).
 5. threshold   -- tau_i = mu_i + beta sigma_i, S_i = {j : s_hat_ij > tau_i}
                   (paithon.it, "Una soglia per ogni riga", the displayed
                   equation; agihunt.info, per-query threshold paragraph).
 6. attention   -- kept blocks are attended exactly; every token of a skipped
                   block is treated as if it had its block's mean key, so the
                   block adds n_j exp(s_hat_ij - m) to the softmax denominator
                   and n_j exp(s_hat_ij - m) v_bar_j to the numerator, in the
                   same softmax state as the exact part (paithon.it, "Scegliere
                   mentre si calcola", third paragraph: zeroth-order Taylor term,
                   proxy scores reused; hotpaper.ai abstract: proxy-score reuse).

Readings taken where the pages are silent or truncated (each listed in the
design notes of this repository):
 * the proxy score carries the same 1/sqrt(d) as the exact scores;
 * the correction of a skipped block uses the block-level score s_hat_ij for
   every row of query block i (not a per-token q_t . k_bar_j);
 * a skipped block weighs n_j (its count of valid tokens);
 * sigma is the population standard deviation (divide by N_b); the covariance
   is computed two-pass; every block counts once whatever its n_j;
 * ties s_hat_ij == tau_i are skipped (strict ">"); a row with sigma_i = 0 is
   constant (all its proxy scores equal mu_i = tau_i), so none of its blocks
   is kept for finite beta;
 * beta = -inf means tau = -inf (all blocks kept, never -inf * 0); beta = +inf
   means tau = +inf (all skipped);
 * pad tokens of the last partial block are not part of any mean and are never
   attended.

The streaming form (`attend_streaming`) follows the double loop of paithon.it
"Scegliere mentre si calcola": an outer loop over pooled keys in groups, with
blocks above tau handed at once to exact attention, skipped ones folded in as
corrections, all into one online-softmax state. The page states that this gives
the same result as thresholding the whole row offline; the tests check it.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64  # tokens per block (paithon.it, "Perché l'attenzione pesa tanto nei video")

__all__ = [
    "BLOCK",
    "block_bounds",
    "block_counts",
    "pool",
    "key_stats",
    "row_stats",
    "thresholds",
    "proxy_scores",
    "route",
    "attend",
    "attend_streaming",
    "dense_attention",
    "forward",
    "route_all",
]


# --------------------------------------------------------------------------
# Step 1: blocks
# --------------------------------------------------------------------------
def block_bounds(N: int):
    """[(start, stop)] of every 64-token block; the last one may be partial."""
    nb = (N + BLOCK - 1) // BLOCK
    return [(b * BLOCK, min(b * BLOCK + BLOCK, N)) for b in range(nb)]


def block_counts(N: int) -> np.ndarray:
    """n_b = number of valid tokens of every block."""
    return np.array([stop - start for start, stop in block_bounds(N)], dtype=np.int64)


# --------------------------------------------------------------------------
# Step 2: block means
# --------------------------------------------------------------------------
def pool(x: np.ndarray, dtype=np.float64) -> np.ndarray:
    """Block means over valid tokens: x [N, d] -> x_bar [N_b, d]."""
    x = np.asarray(x, dtype=dtype)
    out = np.empty((len(block_bounds(x.shape[0])), x.shape[1]), dtype=dtype)
    for b, (start, stop) in enumerate(block_bounds(x.shape[0])):
        out[b] = x[start:stop].sum(axis=0) / (stop - start)
    return out


# --------------------------------------------------------------------------
# Step 3: key statistics
# --------------------------------------------------------------------------
def key_stats(kbar: np.ndarray, dtype=np.float64):
    """Mean k_mean [d] and covariance C [d, d] of the pooled keys, population
    normalisation (divide by N_b), two-pass."""
    kbar = np.asarray(kbar, dtype=dtype)
    nb = kbar.shape[0]
    kmean = kbar.sum(axis=0) / nb
    dev = kbar - kmean
    cov = (dev.T @ dev) / nb
    return kmean, cov


# --------------------------------------------------------------------------
# Step 4: per-row mean and standard deviation of the proxy scores
# --------------------------------------------------------------------------
def row_stats(qbar: np.ndarray, kmean: np.ndarray, kcov: np.ndarray, dtype=np.float64):
    """mu_i = s q_bar_i . k_mean,  sigma_i = s sqrt(q_bar_i^T C q_bar_i)."""
    qbar = np.asarray(qbar, dtype=dtype)
    s = 1.0 / math.sqrt(qbar.shape[1])
    mu = s * (qbar @ kmean)
    quad = np.einsum("id,de,ie->i", qbar, kcov, qbar)
    sigma = s * np.sqrt(np.maximum(quad, 0.0))
    return mu, sigma


# --------------------------------------------------------------------------
# Step 5: threshold
# --------------------------------------------------------------------------
def thresholds(mu: np.ndarray, sigma: np.ndarray, beta: float) -> np.ndarray:
    """tau_i = mu_i + beta sigma_i; beta = -inf / +inf give -inf / +inf.

    A row with sigma_i = 0 is constant: every s_hat_ij equals mu_i = tau_i, so
    under the strict ">" no block passes; its threshold is returned as +inf so
    that rounding in s_hat cannot make a tie look like a pass."""
    if math.isnan(beta):
        raise ValueError("beta is NaN")
    if beta == -math.inf:
        return np.full(mu.shape, -math.inf)
    if beta == math.inf:
        return np.full(mu.shape, math.inf)
    return np.where(sigma == 0.0, math.inf, mu + beta * sigma)


def proxy_scores(qbar: np.ndarray, kbar: np.ndarray, dtype=np.float64) -> np.ndarray:
    """s_hat_ij = q_bar_i . k_bar_j / sqrt(d) (the oracle may form the whole row;
    the method itself never writes it out)."""
    s = 1.0 / math.sqrt(qbar.shape[1])
    return s * (np.asarray(qbar, dtype) @ np.asarray(kbar, dtype).T)


def route(q: np.ndarray, k: np.ndarray, beta: float, dtype=np.float64) -> dict:
    """Routing only (steps 1-5) for one head: q, k [N, d].

    Returns s_hat [N_b, N_b], tau [N_b], mu, sigma, mask [N_b, N_b] (bool,
    True = kept), density [N_b] (= |S_i|), plus the pooled statistics.
    """
    qbar, kbar = pool(q, dtype), pool(k, dtype)
    kmean, kcov = key_stats(kbar, dtype)
    mu, sigma = row_stats(qbar, kmean, kcov, dtype)
    tau = thresholds(mu, sigma, beta)
    shat = proxy_scores(qbar, kbar, dtype)
    mask = shat > tau[:, None]
    return {
        "qbar": qbar,
        "kbar": kbar,
        "kmean": kmean,
        "kcov": kcov,
        "mu": mu,
        "sigma": sigma,
        "tau": tau,
        "shat": shat,
        "mask": mask,
        "density": mask.sum(axis=1).astype(np.int64),
    }


# --------------------------------------------------------------------------
# Other kept-set rules (ablation) and always-kept prefix blocks
# --------------------------------------------------------------------------
# The pages compare the per-row threshold with the top-k and top-p selections
# of earlier methods (paithon.it, "Una soglia per ogni riga": a global top-k
# or top-p gives every row the same budget or needs a sort; "I numeri":
# routing-time comparison threshold / top-k / top-p) and keep text tokens of
# joint attention always exact ("Dove leggere con attenzione"). They define
# neither rule; the readings used here:
#  * top-k keeps the blocks whose proxy score is at least the k-th largest of
#    the row (k clamped to [0, N_b]; equal scores at the cut are all kept);
#  * top-p keeps the blocks whose proxy score is at least v*, the largest
#    value whose superlevel set carries a fraction >= p of the row's mass
#    sum_j n_j exp(s_hat_ij) (the weight a skipped block would get); p <= 0
#    keeps nothing, p >= 1 keeps everything;
#  * forced blocks 0 .. n_forced - 1 are kept in every row in addition to the
#    rule's set.
def topk_mask(shat: np.ndarray, k: int) -> np.ndarray:
    """[N_b, N_b] bool: s_hat_ij >= the k-th largest value of row i."""
    nb = shat.shape[1]
    if k <= 0:
        return np.zeros(shat.shape, bool)
    if k >= nb:
        return np.ones(shat.shape, bool)
    kth = -np.sort(-shat, axis=1)[:, k - 1]
    return shat >= kth[:, None]


def topp_mask(shat: np.ndarray, counts: np.ndarray, p: float) -> np.ndarray:
    """[N_b, N_b] bool: s_hat_ij >= v*_i, v*_i the largest score whose
    superlevel set holds >= p of sum_j n_j exp(s_hat_ij)."""
    nb = shat.shape[1]
    if p <= 0.0:
        return np.zeros(shat.shape, bool)
    if p >= 1.0:
        return np.ones(shat.shape, bool)
    mask = np.zeros(shat.shape, bool)
    for i in range(shat.shape[0]):
        order = np.argsort(-shat[i], kind="stable")
        w = counts[order] * np.exp(shat[i, order] - shat[i, order[0]])
        cum = np.cumsum(w)
        kp = int(np.searchsorted(cum, p * cum[-1], side="left"))  # first index with cum >= p * total
        vstar = shat[i, order[min(kp, nb - 1)]]
        mask[i] = shat[i] >= vstar
    return mask


def route_rule(q: np.ndarray, k: np.ndarray, rule: str, param: float, n_forced: int = 0) -> dict:
    """route() with another kept-set rule: rule = "threshold" (param = beta),
    "topk" (param = k) or "topp" (param = p), plus n_forced always-kept blocks."""
    r = route(q, k, param if rule == "threshold" else 0.0)
    if rule == "topk":
        mask = topk_mask(r["shat"], int(param))
    elif rule == "topp":
        mask = topp_mask(r["shat"], block_counts(q.shape[0]).astype(np.float64), float(param))
    elif rule == "threshold":
        mask = r["mask"].copy()
    else:
        raise ValueError(rule)
    if n_forced > 0:
        mask[:, :n_forced] = True
    r["mask"] = mask
    r["density"] = mask.sum(axis=1).astype(np.int64)
    return r


# --------------------------------------------------------------------------
# Step 6: attention with exact kept blocks and zeroth-order correction
# --------------------------------------------------------------------------
def attend(q, k, v, beta: float = -math.inf, mask=None, rows=None, correction: str = "block", dtype=np.float64):
    """Sol-Attn forward for one head, offline threshold form.

    q, k, v: [N, d]. mask: optional [N_b, N_b] bool to use instead of the
    threshold (external-mask mode). rows: optional list of query-block indices
    to compute (others are left NaN). correction: "block" (the library's
    definition: a skipped block j reuses its proxy score s_hat_ij for every row
    of block i) or "token" (the more literal reading of "Scegliere mentre si
    calcola": every token of the skipped block is taken to carry the block's
    mean key, so row t scores it s q_t . kbar_j; the value is still vbar_j).
    Returns out [N, d], lse [N] (natural log of the softmax denominator of the
    scaled scores), density [N_b] (= |S_i|). dtype: the working precision
    (fp64 for every parity check; fp32 only to time the CPU baseline).
    """
    if correction not in ("block", "token"):
        raise ValueError(correction)
    q = np.asarray(q, dtype)
    k = np.asarray(k, dtype)
    v = np.asarray(v, dtype)
    N, d = q.shape
    s = 1.0 / math.sqrt(d)
    bounds = block_bounds(N)
    n = block_counts(N).astype(dtype)
    r = route(q, k, beta, dtype)
    shat = r["shat"]
    vbar = pool(v, dtype)
    kbar = r["kbar"]
    if mask is None:
        mask = r["mask"]
    mask = np.asarray(mask, dtype=bool)
    out = np.full((N, d), np.nan, dtype=dtype)
    lse = np.full((N,), np.nan, dtype=dtype)
    rows = range(len(bounds)) if rows is None else rows
    for i in rows:
        a, b = bounds[i]
        qi = q[a:b]
        kept = np.nonzero(mask[i])[0]
        skipped = np.nonzero(~mask[i])[0]
        tok = np.concatenate([np.arange(*bounds[j]) for j in kept]) if len(kept) else np.zeros(0, np.int64)
        scores = s * (qi @ k[tok].T)  # exact scores [n_i, tokens of kept blocks]
        if correction == "block":
            corr = np.broadcast_to(shat[i, skipped], (b - a, len(skipped)))  # proxy scores reused
        else:
            corr = s * (qi @ kbar[skipped].T)  # each token against the skipped blocks' mean keys
        m = np.full((b - a,), -math.inf)
        if scores.shape[1]:
            m = np.maximum(m, scores.max(axis=1))
        if corr.shape[1]:
            m = np.maximum(m, corr.max(axis=1))
        e = np.exp(scores - m[:, None])
        c = n[skipped][None, :] * np.exp(corr - m[:, None])
        den = e.sum(axis=1) + c.sum(axis=1)
        num = e @ v[tok] + c @ vbar[skipped]
        out[a:b] = num / den[:, None]
        lse[a:b] = m + np.log(den)
    return out, lse, mask.sum(axis=1).astype(np.int64)


def attend_streaming(q, k, v, beta: float, group: int):
    """Sol-Attn forward for one head in the single-pass form: the outer loop
    walks the pooled keys `group` blocks at a time and scores them; blocks above
    tau go straight to exact attention, the others are folded in as corrections,
    all into one running (max, sum, numerator) state per query row.
    Returns out [N, d], lse [N], density [N_b]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N, d = q.shape
    s = 1.0 / math.sqrt(d)
    bounds = block_bounds(N)
    nb = len(bounds)
    n = block_counts(N).astype(np.float64)
    qbar, kbar, vbar = pool(q), pool(k), pool(v)
    kmean, kcov = key_stats(kbar)
    mu, sigma = row_stats(qbar, kmean, kcov)
    tau = thresholds(mu, sigma, beta)
    out = np.empty((N, d))
    lse = np.empty((N,))
    density = np.zeros((nb,), np.int64)
    for i in range(nb):
        a, b = bounds[i]
        qi = q[a:b]
        m = np.full((b - a,), -math.inf)
        den = np.zeros((b - a,))
        num = np.zeros((b - a, d))
        for g0 in range(0, nb, group):
            js = list(range(g0, min(g0 + group, nb)))
            sc = s * (kbar[js] @ qbar[i])  # proxy scores of this group
            for j, sh in zip(js, sc):
                if sh > tau[i]:
                    density[i] += 1
                    x = s * (qi @ k[bounds[j][0]:bounds[j][1]].T)
                    xv = v[bounds[j][0]:bounds[j][1]]
                    w_new = x
                    cnt = None
                else:
                    w_new = np.full((b - a, 1), sh)
                    xv = vbar[j][None, :]
                    cnt = n[j]
                m_new = np.maximum(m, w_new.max(axis=1))
                scale = np.where(np.isfinite(m), np.exp(m - m_new), 0.0)
                p = np.exp(w_new - m_new[:, None])
                if cnt is not None:
                    p = p * cnt
                den = den * scale + p.sum(axis=1)
                num = num * scale[:, None] + p @ xv
                m = m_new
        out[a:b] = num / den[:, None]
        lse[a:b] = m + np.log(den)
    return out, lse, density


def dense_attention(q, k, v):
    """Plain softmax attention with scale 1/sqrt(d): out [N, d], lse [N]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    s = 1.0 / math.sqrt(q.shape[1])
    x = s * (q @ k.T)
    m = x.max(axis=1)
    e = np.exp(x - m[:, None])
    den = e.sum(axis=1)
    return (e @ v) / den[:, None], m + np.log(den)


# --------------------------------------------------------------------------
# Batched wrappers over [B, H, N, d]
# --------------------------------------------------------------------------
def _as64(t):
    if hasattr(t, "detach"):  # torch tensor (bf16 converts exactly through fp32)
        t = t.detach().to("cpu").float().numpy()
    return np.asarray(t, dtype=np.float64)


def forward(q, k, v, beta: float = -math.inf, masks=None, rows=None, correction: str = "block"):
    """attend() over every (b, h) of [B, H, N, d] inputs (torch or numpy).

    masks: optional [B, H, N_b, N_b] external masks. rows: optional query-block
    list applied to every head. Returns out [B,H,N,d], lse [B,H,N], density
    [B,H,N_b] as numpy arrays.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, N, d = q.shape
    nb = len(block_bounds(N))
    out = np.empty((B, H, N, d))
    lse = np.empty((B, H, N))
    dens = np.empty((B, H, nb), np.int64)
    for b in range(B):
        for h in range(H):
            mk = None if masks is None else np.asarray(masks[b][h], bool)
            out[b, h], lse[b, h], dens[b, h] = attend(q[b, h], k[b, h], v[b, h], beta, mk, rows, correction)
    return out, lse, dens


def route_all(q, k, beta: float):
    """route() over every (b, h): returns a dict of stacked arrays."""
    q, k = _as64(q), _as64(k)
    B, H = q.shape[:2]
    res = [[route(q[b, h], k[b, h], beta) for h in range(H)] for b in range(B)]
    keys = res[0][0].keys()
    return {key: np.stack([np.stack([res[b][h][key] for h in range(H)]) for b in range(B)]) for key in keys}
