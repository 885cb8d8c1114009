"""Writes correction_accuracy.json: how far each reading of the skipped-block
correction lands from exact softmax attention on the synthetic workloads, as
computed by the oracle (fp64) on the seed-0 inputs.

For every query row the three outputs share the kept set of the threshold
rule (paithon.it, "Una soglia per ogni riga"):
  * "block": the library's correction, n_j e^{s_hat_ij - m} per skipped block
    ("Scegliere mentre si calcola", zeroth-order term with the proxy score);
  * "token": the per-token reading, n_j e^{s q_t . kbar_j - m};
  * "none":  the skipped blocks dropped (plain block-sparse attention, the
    softmax restricted to the kept blocks' keys).
Reported per workload and beta: mean kept density, and the relative L2 error
of each output against dense attention over the rows evaluated, plus the
mean absolute error of lse.

The pages print no error values for this comparison, so these numbers pin
nothing; they document the approximation on these inputs.

    python tests/golden/make_correction_accuracy.py
"""
import json
import math
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from block_sparse_attention_cov_b200.inputs import WORKLOADS, make_qkv  # noqa: E402
from oracle import solattn_oracle as orc  # noqa: E402


def kept_only(q, k, v, mask, rows):
    """Softmax over the keys of the kept blocks only (no correction)."""
    N, d = q.shape
    s = 1.0 / math.sqrt(d)
    bounds = orc.block_bounds(N)
    out = np.full((N, d), np.nan)
    lse = np.full((N,), np.nan)
    for i in rows:
        a, b = bounds[i]
        kept = np.nonzero(mask[i])[0]
        if not len(kept):
            continue
        tok = np.concatenate([np.arange(*bounds[j]) for j in kept])
        x = s * (q[a:b] @ k[tok].T)
        m = x.max(axis=1)
        e = np.exp(x - m[:, None])
        out[a:b] = (e @ v[tok]) / e.sum(axis=1)[:, None]
        lse[a:b] = m + np.log(e.sum(axis=1))
    return out, lse


def study(name, heads, betas, rows_per_head=None, seed=0):
    wl = WORKLOADS[name]
    q, k, v = make_qkv(wl, seed=seed, heads=[(0, h) for h in heads])
    nb = math.ceil(wl.N / 64)
    rng = np.random.default_rng(seed)
    acc = {beta: {"density": [], "err": {c: [0.0, 0.0] for c in ("block", "token", "none")},
                  "lse": {c: [] for c in ("block", "token", "none")}} for beta in betas}
    for pos, h in enumerate(heads):  # make_qkv returns the listed heads in order
        qq, kk, vv = (x[0, pos].double().numpy() for x in (q, k, v))
        if rows_per_head is None:
            rows = list(range(nb))
        else:
            rows = sorted({0, nb - 1, *rng.choice(nb, rows_per_head - 2, replace=False).tolist()})
        sel = np.concatenate([np.arange(*orc.block_bounds(wl.N)[i]) for i in rows])
        od, ld = orc.dense_attention(qq[sel], kk, vv)  # rows are independent
        for beta in betas:
            r = orc.route(qq, kk, beta)
            a = acc[beta]
            a["density"].append(float(r["mask"][rows].mean()))
            outs = {
                "block": orc.attend(qq, kk, vv, beta, rows=rows, correction="block")[:2],
                "token": orc.attend(qq, kk, vv, beta, rows=rows, correction="token")[:2],
                "none": kept_only(qq, kk, vv, r["mask"], rows),
            }
            for c, (o, l) in outs.items():
                o, l = o[sel], l[sel]
                ok = np.isfinite(l)  # "none" leaves rows with no kept block empty
                a["err"][c][0] += float(np.sum((o[ok] - od[ok]) ** 2))
                a["err"][c][1] += float(np.sum(od[ok] ** 2))
                a["lse"][c].append(float(np.abs(l[ok] - ld[ok]).mean()) if ok.any() else float("nan"))
    res = []
    for beta in betas:
        a = acc[beta]
        res.append({
            "beta": beta,
            "density": float(np.mean(a["density"])),
            "rel_l2_vs_dense": {c: math.sqrt(e / n) for c, (e, n) in a["err"].items()},
            "mean_abs_lse_vs_dense": {c: float(np.nanmean(x)) for c, x in a["lse"].items()},
        })
    return {"workload": name, "heads": heads, "rows_per_head": rows_per_head or nb, "seed": seed, "results": res}


def main():
    with open(os.path.join(HERE, "calibrated_beta.json")) as f:
        wan_beta = json.load(f)["wan_75k"]["beta"]
    out = {
        "mid": study("mid", list(range(8)), [0.0, 0.5, 1.0, 1.5]),
        "wan_75k": study("wan_75k", [0, 20], [wan_beta], rows_per_head=24),
    }
    path = os.path.join(HERE, "correction_accuracy.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    for w in out.values():
        for r in w["results"]:
            e = r["rel_l2_vs_dense"]
            print(f"{w['workload']:8s} beta {r['beta']:.4f} density {r['density']:.3f}  rel L2 vs dense: "
                  f"block {e['block']:.3f}  token {e['token']:.3f}  none {e['none']:.3f}")


if __name__ == "__main__":
    main()
