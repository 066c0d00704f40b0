"""CPU-only checks of the C-ABI library: it loads, exports every declared symbol,
and its host-side math (grouped widths, water-filling, Jacobi eigen, page
layout) agrees with the oracle.  No GPU calls."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def st():
    import spectral_transform_coding_b200 as st
    return st


def test_exports_every_declared_symbol(st):
    header = open(os.path.join(ROOT, "include", "spectra.h")).read()
    declared = set(re.findall(r"^SPECTRA_API [^(]*?\b(spectra_\w+)\(", header, flags=re.M))
    assert len(declared) >= 20
    for name in declared:
        assert hasattr(st.lib, name), name
    from spectral_transform_coding_b200._lib import EXPORTED
    assert declared == set(EXPORTED)
    assert st.lib.spectra_abi_version() == 1


@pytest.mark.parametrize("case", range(40))
def test_widths_match_oracle(st, case):
    rng = np.random.default_rng(case)
    g = 8 if case % 2 else 16
    r = g * int(rng.integers(1, 9))
    s2 = np.sort(rng.exponential(1.0, r) * np.arange(1, r + 1) ** -rng.uniform(0, 2))[::-1].copy()
    budget = int(rng.integers(0, 700))
    ovh = bool(case % 3)
    w = np.zeros(r // g, np.int32)
    d = ctypes.c_double()
    rc = st.lib.spectra_allocate_widths(s2.ctypes.data, r, g, budget, int(ovh), w.ctypes.data, ctypes.byref(d))
    assert rc == 0
    np.testing.assert_array_equal(w, oracle.allocate_widths(s2, g, budget, ovh))
    assert d.value == pytest.approx(oracle.allocation_distortion(s2, w, g), rel=1e-14)


def test_widths_rejects_bad_input(st):
    s2 = np.array([1.0, np.nan] * 8)
    w = np.zeros(1, np.int32)
    assert st.lib.spectra_allocate_widths(s2.ctypes.data, 16, 16, 64, 1, w.ctypes.data, None) == 4
    assert st.lib.spectra_allocate_widths(s2.ctypes.data, 15, 16, 64, 1, w.ctypes.data, None) == 1
    assert b"" != st.lib.spectra_last_error()


@pytest.mark.parametrize("seed", range(8))
def test_water_fill_matches_oracle(st, seed):
    rng = np.random.default_rng(seed)
    s2 = rng.pareto(1.2, 64) + 1e-4
    R = float(rng.uniform(0.5, 200))
    th = ctypes.c_double()
    rates = np.zeros(64)
    assert st.lib.spectra_water_fill(s2.ctypes.data, 64, R, ctypes.byref(th), rates.ctypes.data) == 0
    wf = oracle.reverse_water_fill(s2, R)
    assert th.value == pytest.approx(wf["theta"], rel=1e-10)
    np.testing.assert_allclose(rates, wf["R"], atol=1e-9)


@pytest.mark.parametrize("n", [1, 2, 7, 64, 128])
def test_jacobi_eigen(st, n):
    rng = np.random.default_rng(n)
    A = rng.standard_normal((n, n))
    M = A @ A.T + np.diag(np.arange(n, dtype=float))
    vals = np.zeros(n)
    vecs = np.zeros((n, n))
    assert st.lib.spectra_sym_eigen(M.ctypes.data, n, vals.ctypes.data, vecs.ctypes.data) == 0
    ref, V = np.linalg.eigh(M)
    np.testing.assert_allclose(vals, ref[::-1], rtol=1e-11, atol=1e-11 * ref.max())
    np.testing.assert_allclose(vecs, oracle.sign_fix(V[:, ::-1]), atol=1e-8)
    np.testing.assert_allclose(vecs @ np.diag(vals) @ vecs.T, M, atol=1e-9 * np.abs(M).max())


def test_jacobi_rejects_nan(st):
    M = np.eye(4)
    M[1, 2] = M[2, 1] = np.nan
    v = np.zeros(4)
    V = np.zeros((4, 4))
    assert st.lib.spectra_sym_eigen(M.ctypes.data, 4, v.ctypes.data, V.ctypes.data) == 4


def test_page_layout_matches_oracle(st):
    from spectral_transform_coding_b200.codec import make_config
    rng = np.random.default_rng(3)
    for g, r, nkv, P in ((16, 128, 8, 64), (8, 32, 1, 64), (16, 64, 3, 128), (8, 64, 2, 32)):
        ng = r // g
        widths = rng.choice([0, 1, 2, 3, 4, 8], size=(nkv, 2, ng)).astype(np.int32)
        cfg = make_config(256, nkv, nkv, r, r, g, 512, True, P)
        pb = ctypes.c_int64()
        offs = np.zeros(2 * nkv * 2 * ng, np.int64)
        assert st.lib.spectra_page_layout(ctypes.byref(cfg), widths.ctypes.data, ctypes.byref(pb),
                                          offs.ctypes.data) == 0
        lay = oracle.page_layout([[widths[a, 0], widths[a, 1]] for a in range(nkv)], g, P)
        assert pb.value == lay["page_bytes"]
        plane, sz = offs[: nkv * 2 * ng].reshape(nkv, 2, ng), offs[nkv * 2 * ng:].reshape(nkv, 2, ng)
        for a in range(nkv):
            for s in range(2):
                kept = [j for j in range(ng) if widths[a, s, j] > 0]
                for (b, po, so, col), j in zip(lay["groups"][(a, s)], kept):
                    assert (plane[a, s, j], sz[a, s, j]) == (po, so)
                assert all(plane[a, s, j] == -1 for j in range(ng) if widths[a, s, j] == 0)


def test_invalid_config_rejected(st):
    from spectral_transform_coding_b200.codec import make_config
    w = np.zeros(8, np.int32)
    pb = ctypes.c_int64()
    bad = make_config(256, 4, 1, 64, 32, 12, 64, False, 64)  # group 12
    assert st.lib.spectra_page_layout(ctypes.byref(bad), w.ctypes.data, ctypes.byref(pb), None) == 1
    bad = make_config(256, 4, 1, 64, 32, 8, 64, False, 48)  # page_tokens not multiple of 32
    assert st.lib.spectra_page_layout(ctypes.byref(bad), w.ctypes.data, ctypes.byref(pb), None) == 1


@pytest.mark.parametrize("seed", range(4))
def test_uniform_widths_match_oracle(seed):
    from spectral_transform_coding_b200._lib import lib
    rng = np.random.default_rng(100 + seed)
    s2 = np.ascontiguousarray(np.sort(rng.gamma(0.7, size=128))[::-1])
    for budget, ov, ne in ((512, 1, 8), (256, 1, 8), (256, 1, 3), (170, 1, 8), (64, 0, 8)):
        w = np.zeros(8, np.int32)
        d = ctypes.c_double(0)
        assert lib.spectra_allocate_widths_uniform(s2.ctypes.data, 128, 16, ne, budget, ov, w.ctypes.data,
                                                   ctypes.byref(d)) == 0
        ref = oracle.allocate_widths_uniform(s2, 16, budget, bool(ov), ne)
        np.testing.assert_array_equal(w, ref)
        assert abs(d.value - oracle.allocation_distortion(s2, ref, 16)) <= 1e-12 * max(1.0, d.value)


def test_energy_rank_matches_oracle():
    from spectral_transform_coding_b200._lib import lib
    rng = np.random.default_rng(7)
    s2 = np.ascontiguousarray(np.sort(rng.exponential(size=128))[::-1])
    for thr in (0.5, 0.9, 0.95, 0.99, 1.0):
        r = ctypes.c_int32(0)
        assert lib.spectra_energy_rank(s2.ctypes.data, 128, thr, ctypes.byref(r)) == 0
        assert r.value == oracle.energy_rank(s2, thr)
    assert lib.spectra_energy_rank(s2.ctypes.data, 128, 0.0, ctypes.byref(r)) != 0
