"""Writes calibrated_beta.json: for each benchmark workload, the global beta whose
mean kept-block density (over every head and query block, routing oracle in
fp64 on the seed-0 synthetic inputs) equals each target, found by bisection to
1e-4 in beta. Uses only the oracle and the seeded input generator.

The pages set beta once per model for a target mean density ("Sol-Attn",
paithon.it, "Una soglia per ogni riga": one global beta fixes the mean density);
the workloads' targets are 15 % (Wan-like 75.6K), 10 % and 15 % (Hunyuan-like),
and 5/10/15/30 % (length sweep).

    python tests/golden/make_calibrated_beta.py [workload ...]
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from block_sparse_attention_cov_b200.inputs import WORKLOADS, make_qkv  # noqa: E402
from oracle import solattn_oracle as orc  # noqa: E402

TARGETS = {
    "mid": [0.5, 0.3, 0.15, 0.07],
    "wan_75k": [0.15],
    "hunyuan_119k": [0.10, 0.15],
    "sweep_16k": [0.05, 0.10, 0.15, 0.30],
    "sweep_32k": [0.05, 0.10, 0.15, 0.30],
    "sweep_64k": [0.05, 0.10, 0.15, 0.30],
    "sweep_128k": [0.05, 0.10, 0.15, 0.30],
}


def standardized_rows(wl, seed=0):
    """z_ij = (s_hat_ij - mu_i) / sigma_i for every head (kept iff z > beta)."""
    zs = []
    for b in range(wl.B):
        for h in range(wl.H):
            q, k, _ = make_qkv(wl, seed, heads=[(b, h)], threads=1)
            r = orc.route(q[0, 0].double().numpy(), k[0, 0].double().numpy(), 0.0)
            zs.append(((r["shat"] - r["mu"][:, None]) / r["sigma"][:, None]).astype(np.float64).ravel())
    return np.concatenate(zs)


def calibrate(z, target):
    lo, hi = -6.0, 6.0
    while hi - lo > 1e-4:
        mid = 0.5 * (lo + hi)
        if (z > mid).mean() > target:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi), 4)
    return beta, float((z > beta).mean())


def main(names):
    path = os.path.join(HERE, "calibrated_beta.json")
    data = json.load(open(path)) if os.path.exists(path) else {}
    for name in names:
        wl = WORKLOADS[name]
        z = standardized_rows(wl)
        entry = {"seed": 0, "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "targets": {}}
        for t in TARGETS[name]:
            beta, dens = calibrate(z, t)
            entry["targets"][f"{t:.2f}"] = {"beta": beta, "mean_density": dens}
            print(name, t, beta, dens, flush=True)
        first = entry["targets"][f"{TARGETS[name][0]:.2f}"]
        entry["beta"] = first["beta"]
        data[name] = entry
        json.dump(data, open(path, "w"), indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or list(TARGETS))
