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
