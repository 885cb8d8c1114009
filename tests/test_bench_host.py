"""Host-side helpers of bench.py on CPU: the calibrated-beta lookup behind
--beta / --density (tests/golden/calibrated_beta.json, written by the oracle)."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

with open(os.path.join(ROOT, "tests", "golden", "calibrated_beta.json")) as f:
    CAL = json.load(f)


def test_default_beta_is_the_primary_calibration():
    for name, rec in CAL.items():
        assert bench.load_beta(name)[0] == rec["beta"]
    assert bench.load_beta("wan_75k")[0] == pytest.approx(1.0456)


@pytest.mark.parametrize("name", ["hunyuan_119k", "sweep_16k", "sweep_32k", "sweep_64k", "sweep_128k", "mid"])
def test_density_picks_that_target(name):
    for key, rec in CAL[name]["targets"].items():
        assert bench.load_beta(name, float(key))[0] == rec["beta"]
    # a lower density needs a larger beta (fewer blocks above tau)
    betas = [bench.load_beta(name, float(k))[0] for k in sorted(CAL[name]["targets"], key=float)]
    assert betas == sorted(betas, reverse=True)


def test_unknown_density_is_an_error():
    with pytest.raises(KeyError):
        bench.load_beta("wan_75k", 0.42)


def test_stratified_sample_rows():
    """First, last and 30 seeded random query blocks per head; the same rows
    for the same head in both CPU arms (cpu_baseline leg and --impl reference)."""
    rows = bench.sample_rows(1182, 7)
    assert rows[0] == 0 and rows[-1] == 1181 and len(rows) == bench.SAMPLE_BLOCKS == 32
    assert rows == bench.sample_rows(1182, 7) and rows != bench.sample_rows(1182, 8)
    assert bench.sample_rows(3, 0) == [0, 1, 2] and bench.sample_rows(1, 0) == [0]


def test_row_kept_flops_counts_partial_blocks():
    import numpy as np

    # N = 150: blocks of 64, 64, 22 tokens; d = 4
    mask = np.array([[True, False, True], [False, False, False], [True, True, True]])
    f = bench.row_kept_flops(mask, 150, 4)
    assert f.tolist() == [4 * 4 * 64 * (64 + 22), 0.0, 4 * 4 * 22 * 150]


def test_density_stats():
    import torch

    dens = torch.tensor([[[1, 2, 3, 4]]], dtype=torch.int32)
    st = bench.density_stats(dens, 8)
    assert st["mean"] == pytest.approx(2.5 / 8) and st["min"] == 1 / 8 and st["max"] == 4 / 8
    assert st["p50"] == pytest.approx(2.5 / 8)


def test_oracle_head_sample_reports_output_error():
    """The bench line's output_error: against the fp32 oracle on the sampled
    rows, an exact (fp64 oracle) output gives a tiny error and a perturbed one
    is caught at the perturbation's size."""
    import numpy as np

    import bench
    from block_sparse_attention_cov_b200.inputs import Workload, make_qkv
    from oracle import solattn_oracle as orc

    wl = Workload("s", 1, 1, 64, (1, 1, 64 * 40))
    q, k, v = make_qkv(wl, seed=3)
    out64, lse64, _ = orc.attend(*(x[0, 0].double().numpy() for x in (q, k, v)), 0.5)
    _, _, errs = bench.oracle_head_sample(q, k, v, 0.5, 0, 0, out_gpu=out64, lse_gpu=lse64)
    assert errs[0] / errs[1] < 1e-10 and errs[2] < 1e-5 and errs[3] < 1e-5
    bad = out64.copy()
    bad[0, 0] += 0.25  # row 0 belongs to the first block, always sampled
    _, _, errs = bench.oracle_head_sample(q, k, v, 0.5, 0, 0, out_gpu=bad, lse_gpu=lse64)
    assert abs(errs[2] - 0.25) < 1e-4
