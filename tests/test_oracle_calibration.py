"""Pins of the Sequential Temperature Scaling / ECE oracle against closed forms,
hand-computed values and special cases with known answers."""
import numpy as np

from oracle import calibration as cal
from speculative_decoding_draft_sample_b200 import workloads as wl


def test_temperature_grid_is_log_spaced_on_the_stated_range():
    g = cal.temperature_grid()
    assert len(g) == cal.STS_GRID
    assert abs(g[0] - 0.05) < 1e-15 and abs(g[-1] - 20.0) < 1e-12
    ratios = g[1:] / g[:-1]
    np.testing.assert_allclose(ratios, (20.0 / 0.05) ** (1.0 / (cal.STS_GRID - 1)), rtol=1e-12)


def test_ece_hand_computed():
    # two bins: [0, .5) holds .1, .2 (labels 0, 1); [.5, 1] holds .8, .9 (labels 1, 1)
    # |0.15 - 0.5| * 2/4 + |0.85 - 1| * 2/4 = 0.175 + 0.075
    assert abs(cal.ece([0.1, 0.2, 0.8, 0.9], [0, 1, 1, 1], nbins=2) - 0.25) < 1e-15
    # a prediction of exactly 1 falls in the last bin
    assert abs(cal.ece([1.0, 1.0], [1, 0], nbins=4) - 0.5) < 1e-15
    # empty bins contribute nothing
    assert cal.ece([0.55], [1], nbins=10) == abs(0.55 - 1.0)


def test_ece_of_calibrated_predictions_is_small():
    rng = np.random.default_rng(5)
    p = rng.random(400000)
    y = rng.random(400000) < p
    assert cal.ece(p, y) < 0.005


def test_survival_product():
    z = np.array([[0.0, 2.0, -1.0]])
    T = np.array([1.0, 2.0, 0.5])
    want = 0.5 * (1 / (1 + np.exp(-1.0))) * (1 / (1 + np.exp(2.0)))
    assert abs(cal.survival(z, T, 2)[0] - want) < 1e-15


def test_nll_special_cases_pick_the_grid_ends():
    z = np.full((50, 1), 1.5)
    # every label 1, positive logits: the sharpest temperature wins
    assert cal.sts_fit(z, np.ones((50, 1), np.uint8))["index"][0] == 0
    # every label 0, positive logits: the flattest temperature wins
    assert cal.sts_fit(z, np.zeros((50, 1), np.uint8))["index"][0] == cal.STS_GRID - 1


def test_sts_recovers_the_over_confidence_factor():
    z, y = wl.calib_inputs(60000, K=3, gammas=(2.0, 1.5, 0.8), seed=11)
    r = cal.sts_fit(z, y)
    np.testing.assert_allclose(r["T"], [2.0, 1.5, 0.8], rtol=0.1)
    assert np.all(r["ece_after"] < 0.02)
    assert np.all(r["ece_after"] < r["ece_before"])
    assert r["ece_before"].max() > 0.03  # the uncalibrated head is off by several percent
