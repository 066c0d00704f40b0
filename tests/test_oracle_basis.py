"""Pins of the oracle's G-weighted transform (SPECTRA technical summary, "SPECTRA
pipeline" stage 1; "Spectral-KV", "Technical principle" 1-2).

Three independent routes must give one basis: the literal SVD of G^{1/2} W, the
eigen-decomposition of W^T G W, and the SVD of the calibration keys K = H W.
"""
import numpy as np
import pytest

import oracle
from workloads import get_config, make_activations, make_weights


def _basis_case(seed=0, d_model=96, d_h=32, n=600, alpha=1.3):
    rng = np.random.default_rng(seed)
    q, _ = np.linalg.qr(rng.standard_normal((d_model, d_model)))
    lam = np.arange(1, d_model + 1) ** -alpha
    H = (rng.standard_normal((n, d_model)) * np.sqrt(lam)) @ q.T
    W = rng.standard_normal((d_model, d_h)) / np.sqrt(d_model)
    return H, W


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_three_routes_agree(seed):
    H, W = _basis_case(seed)
    G = oracle.gram(H)
    lit = oracle.whitened_svd(G, W, 16)
    eig = oracle.latent_basis(G, W, 16)
    ksv = oracle.keys_svd_basis(H, W, 16)
    for other in (eig, ksv):
        np.testing.assert_allclose(other["sigma2"], lit["sigma2"], rtol=1e-9, atol=1e-14)
        # sign-fixed eigenvectors agree column by column
        assert np.abs(other["V"] - lit["V"]).max() < 1e-8
    np.testing.assert_allclose(eig["W_down"], lit["W_down"], rtol=0, atol=1e-10)


def test_keys_route_singular_values_scale_with_n():
    H, W = _basis_case(3)
    K = H @ W
    s = np.linalg.svd(K, compute_uv=False)
    ksv = oracle.keys_svd_basis(H, W, 8)
    np.testing.assert_allclose(ksv["sigma2"] * H.shape[0], np.sort(s)[::-1] ** 2, rtol=1e-10)


def test_latent_covariance_diagonal_and_sorted(toy_cfg, toy_layer, toy_codec):
    """(1/N) C^T C on the calibration set is diagonal and energy sorted."""
    H = toy_layer["H_calib"].astype(np.float64)
    for side, W in (("K", toy_layer["W_K"]), ("V", toy_layer["W_V"])):
        hs = toy_codec["heads"][0][side]
        Wd = np.asarray(W, np.float64) @ hs["V"][:, :toy_cfg.rank]
        C = H @ Wd
        cov = C.T @ C / H.shape[0]
        d = np.diag(cov)
        off = cov - np.diag(d)
        ratio = np.abs(off) / np.sqrt(np.outer(d, d))
        assert ratio.max() <= 1e-8
        assert np.all(np.diff(d) <= 1e-15 * d[0])
        np.testing.assert_allclose(d, hs["sigma2"], rtol=1e-10)


def test_whitening_beats_weight_space_basis():
    """Observation 3: the G-weighted basis keeps at least as much activation energy
    as any rank-r orthonormal basis, in particular the weight-space SVD's."""
    H, W = _basis_case(4, alpha=2.0)
    G = oracle.gram(H)
    r = 6
    lit = oracle.whitened_svd(G, W, r)
    kept = lit["sigma2"][:r].sum()

    def energy(Vr):
        C = H @ W @ Vr
        return (C ** 2).sum() / H.shape[0]

    _, _, Vt = np.linalg.svd(W, full_matrices=False)
    assert energy(Vt.T[:, :r]) <= kept * (1 + 1e-12)
    rng = np.random.default_rng(5)
    for _ in range(20):
        Q, _ = np.linalg.qr(rng.standard_normal((W.shape[1], r)))
        assert energy(Q) <= kept * (1 + 1e-12)
    np.testing.assert_allclose(energy(lit["V"][:, :r]), kept, rtol=1e-10)


def test_sign_rule():
    V = np.array([[0.1, -0.9], [-0.8, 0.2], [0.3, 0.3]])
    F = oracle.sign_fix(V)
    assert F[1, 0] > 0 and F[0, 1] > 0
    np.testing.assert_array_equal(np.abs(F), np.abs(V))


def test_full_rank_reconstruction_is_exact(toy_cfg, toy_layer, toy_codec):
    """With r = d_h and no quantisation, c W_up = h W (V orthogonal)."""
    G = toy_codec["G"]
    W = np.asarray(toy_layer["W_K"], np.float64)
    full = oracle.latent_basis(G, W, W.shape[1])
    h = toy_layer["H_calib"][:50].astype(np.float64)
    c = h @ full["W_down"]
    np.testing.assert_allclose(c @ full["W_up"], h @ W, rtol=0, atol=1e-12 * np.abs(h @ W).max())


def test_wide_config_basis_agrees_with_keys_route():
    """Same agreement on a Llama-shaped head (sub-sampled calibration set)."""
    cfg = get_config("llama")
    H = make_activations(cfg, 1024, stream=2).astype(np.float64)
    W = make_weights(cfg)["W_K"][:, :cfg.d_head].astype(np.float64)
    G = oracle.gram(H)
    eig = oracle.latent_basis(G, W, cfg.rank)
    ksv = oracle.keys_svd_basis(H, W, cfg.rank)
    np.testing.assert_allclose(eig["sigma2"], ksv["sigma2"], rtol=1e-8)
    # compare the leading, well-separated directions
    gaps = -np.diff(eig["sigma2"]) / eig["sigma2"][:-1]
    k = int(np.argmax(gaps < 1e-3)) or 8
    k = min(k, 8)
    assert np.abs(eig["V"][:, :k] - ksv["V"][:, :k]).max() < 1e-6
