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


# --- uniform allocation and the energy rank (allocation ablation) -------------------

def test_uniform_allocation_worked_by_hand():
    """Groups of 2, no overhead, budget 8 bits (cost of a group = 2 b).
    sigma2 = [4,4,1,1,.25,.25,0,0]: S = [8,2,.5,0].  Candidates (k, b) -> model
    distortion: b=1: k=3 or 4 -> 10.5/4 = 2.625; b=2: k=2 -> 10/16 + .5 = 1.125,
    k=1 -> 3.0; b=3: k=1 -> 8/64 + 2.5 = 2.625; b=4: k=1 -> 2.53125.  Best (2, 2).
    sigma2 = [8,8,.5 x 6]: S = [16,1,1,1].  b=2, k=2 -> 17/16 + 2 = 3.0625 and
    b=4, k=1 -> 1/16 + 3 = 3.0625 with 8 bits each: fewer groups wins -> (1, 4);
    the grouped water-filling optimum is 2.5 (e.g. [3,1,0,0])."""
    s2 = np.array([4, 4, 1, 1, .25, .25, 0, 0.])
    w = oracle.allocate_widths_uniform(s2, 2, 8, False)
    assert list(w) == [2, 2, 0, 0]
    assert oracle.allocation_distortion(s2, w, 2) == 1.125
    s2 = np.array([8, 8] + [.5] * 6)
    w = oracle.allocate_widths_uniform(s2, 2, 8, False)
    assert list(w) == [4, 0, 0, 0]
    assert oracle.allocation_distortion(s2, w, 2) == 3.0625
    assert oracle.allocation_distortion(s2, oracle.allocate_widths(s2, 2, 8, False), 2) == 2.5


@pytest.mark.parametrize("seed", range(6))
def test_uniform_never_beats_grouped_water_filling(seed):
    """The grouped optimum is taken over a superset of the uniform choices."""
    rng = np.random.default_rng(seed)
    s2 = np.sort(rng.gamma(0.5, size=64))[::-1]
    for budget, ov in ((128, True), (256, True), (96, False)):
        wu = oracle.allocate_widths_uniform(s2, 8, budget, ov)
        wd = oracle.allocate_widths(s2, 8, budget, ov)
        assert sum(oracle.group_cost(int(b), 8, ov) for b in wu) <= budget
        assert len(set(int(b) for b in wu if b > 0)) <= 1
        assert oracle.allocation_distortion(s2, wd, 8) <= oracle.allocation_distortion(s2, wu, 8) + 1e-15


def test_uniform_respects_eligible_groups():
    s2 = np.linspace(4, 1, 32)
    w = oracle.allocate_widths_uniform(s2, 8, 1000, True, n_eligible=2)
    assert list(w[2:]) == [0, 0] and w[0] == w[1] == 8


def test_energy_rank_worked_by_hand():
    """sigma2 = [4,3,2,1] (total 10): cumulative 4, 7, 9, 10 -> threshold .7 reached
    at r = 2, .71 at r = 3, 1.0 at r = 4; [5,0,0] holds all energy at r = 1."""
    assert oracle.energy_rank([4, 3, 2, 1], 0.7) == 2
    assert oracle.energy_rank([4, 3, 2, 1], 0.71) == 3
    assert oracle.energy_rank([4, 3, 2, 1], 1.0) == 4
    assert oracle.energy_rank([4, 3, 2, 1], 0.1) == 1
    assert oracle.energy_rank([5, 0, 0], 1.0) == 1
    with pytest.raises(ValueError):
        oracle.energy_rank([1, 1], 0.0)


def test_energy_rank_monotone_in_threshold():
    s2 = np.sort(np.random.default_rng(3).exponential(size=128))[::-1]
    ranks = [oracle.energy_rank(s2, t) for t in np.linspace(0.05, 1.0, 20)]
    assert ranks == sorted(ranks) and ranks[-1] <= 128
