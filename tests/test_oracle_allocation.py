"""Pins of the oracle's bit allocation (SPECTRA technical summary, "SPECTRA
pipeline" stage 2: reverse water-filling on the latent variances, grouping)."""
import itertools
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


def _floats(s):
    return np.array([float(v) for v in s.split(",")])


@pytest.mark.parametrize("row", list(_rows("waterfill_cases.txt")))
def test_water_fill_golden(row):
    s2, R, theta, Ri, Di = _floats(row[0]), float(row[1]), float(row[2]), _floats(row[3]), _floats(row[4])
    wf = oracle.reverse_water_fill(s2, R)
    assert wf["theta"] == pytest.approx(theta, rel=1e-12)
    np.testing.assert_allclose(wf["R"], Ri, atol=1e-12)
    np.testing.assert_allclose(wf["D"], Di, rtol=1e-12)


def _closed_form_theta(s2, R):
    """Textbook: with the k largest variances active, theta = (prod s2_i)^{1/k} 2^{-2R/k}."""
    s = np.sort(np.asarray(s2, float))[::-1]
    for k in range(1, len(s) + 1):
        theta = math.exp((np.log(s[:k]).sum() - 2 * R * math.log(2)) / k)
        if theta < s[k - 1] and (k == len(s) or theta >= s[k]):
            return theta
    raise AssertionError


@pytest.mark.parametrize("seed", range(6))
def test_water_fill_invariants(seed):
    rng = np.random.default_rng(seed)
    s2 = np.sort(rng.pareto(1.5, 32) + 1e-3)[::-1] * 10.0 ** rng.uniform(-3, 3)
    R = float(rng.uniform(1, 100))
    wf = oracle.reverse_water_fill(s2, R)
    assert wf["R"].sum() == pytest.approx(R, rel=1e-12)
    np.testing.assert_array_equal(wf["D"], np.minimum(wf["theta"], s2))
    assert np.all((wf["R"] == 0) == (s2 <= wf["theta"]))
    assert wf["theta"] == pytest.approx(_closed_form_theta(s2, R), rel=1e-10)
    wf2 = oracle.reverse_water_fill(s2, R + 1.0)
    assert wf2["theta"] < wf["theta"]
    assert np.all(wf2["R"] >= wf["R"] - 1e-12)


def test_equal_variances_equal_rates():
    wf = oracle.reverse_water_fill(np.full(16, 0.3), 40.0)
    np.testing.assert_allclose(wf["R"], 2.5, rtol=1e-12)


@pytest.mark.parametrize("row", list(_rows("dp_cases.txt")))
def test_widths_golden(row):
    g, ovh, budget = int(row[0]), bool(int(row[1])), int(row[2])
    S = _floats(row[3])
    sigma2 = np.repeat(S / g, g)
    w = oracle.allocate_widths(sigma2, g, budget, ovh)
    np.testing.assert_array_equal(w, [int(v) for v in row[4].split(",")])
    assert oracle.allocation_distortion(sigma2, w, g) == float(row[5])


def _brute(sigma2, g, budget, ovh):
    S = oracle.group_mass(sigma2, g)
    best = None
    for combo in itertools.product(oracle.WIDTHS, repeat=len(S)):
        cost = sum(oracle.group_cost(b, g, ovh) for b in combo)
        if cost > budget:
            continue
        d = sum(S[j] * 4.0 ** -b for j, b in enumerate(combo))
        if best is None or d < best[0]:
            best = (d, combo)
    return best


@pytest.mark.parametrize("case", range(24))
def test_widths_match_brute_force(case):
    rng = np.random.default_rng(100 + case)
    g = 8 if case % 2 == 0 else 16
    ovh = case % 3 == 0
    n = 2 + case % 3
    if case % 4 == 0:
        sigma2 = np.sort(rng.exponential(1.0, n * g))[::-1]
    else:
        sigma2 = np.arange(1, n * g + 1) ** -rng.uniform(0.5, 2.5)
    budget = int(rng.integers(g, n * (8 * g + 32)))
    w = oracle.allocate_widths(sigma2, g, budget, ovh)
    d_best, _ = _brute(sigma2, g, budget, ovh)
    assert sum(oracle.group_cost(int(b), g, ovh) for b in w) <= budget
    d = oracle.allocation_distortion(sigma2, w, g)
    assert d == pytest.approx(d_best, rel=1e-13, abs=0)
    # no single-group upgrade that still fits lowers the distortion
    for j in range(n):
        for b in oracle.WIDTHS:
            if b <= w[j]:
                continue
            w2 = w.copy()
            w2[j] = b
            if sum(oracle.group_cost(int(x), g, ovh) for x in w2) <= budget:
                assert oracle.allocation_distortion(sigma2, w2, g) >= d * (1 - 1e-13)


def test_toy_widths_spend_two_bits_per_coordinate(toy_cfg, toy_codec):
    for side in ("K", "V"):
        w = toy_codec["heads"][0][side]["widths"]
        assert sum(8 * int(b) for b in w) <= 64
        assert list(w) == sorted(w, reverse=True)  # energy sorted => non-increasing


def test_more_energy_more_bits():
    """Higher-variance groups never get fewer bits than lower-variance ones."""
    for alpha in (0.8, 1.2, 2.0):
        s2 = np.arange(1, 129) ** -alpha
        for budget in (170, 256, 512):
            w = oracle.allocate_widths(s2, 16, budget, True)
            assert list(w) == sorted(w, reverse=True)
