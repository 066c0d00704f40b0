"""Special-case pins of the W_O correction reading (SPECTRA technical summary,
"SPECTRA pipeline" stage 1, "Refinement": a closed-form, training-free correction
of W_O for the low-rank truncation residual; the pages give no formula)."""
import numpy as np

import oracle
from workloads import get_config, make_layer


def _small():
    cfg = get_config("toy", d_model=64, n_q_heads=2, n_kv_heads=1, d_head=16, rank=16,
                     group=8, budget_bits=16, calib_tokens=96)
    layer = make_layer(cfg)
    return cfg, layer


def test_no_truncation_gives_identity():
    cfg, layer = _small()
    codec = oracle.calibrate(cfg.with_(budget_bits=8 * 2 * 8), layer["H_calib"], layer["W_K"],
                             layer["W_V"])
    for s in ("K", "V"):
        codec["heads"][0][s]["keep"] = np.arange(cfg.rank)
    res = oracle.wo_correction(layer["H_calib"], layer["W_Q"], layer["W_K"], layer["W_V"],
                               layer["W_O"], codec, cfg.n_q_heads, 1, cfg.d_head, eps_rel=1e-14)
    for M in res["M"]:
        np.testing.assert_allclose(M, np.eye(cfg.d_head), atol=1e-6)


def test_correction_never_increases_residual():
    cfg, layer = _small()
    codec = oracle.calibrate(cfg, layer["H_calib"], layer["W_K"], layer["W_V"])
    assert any(len(codec["heads"][0][s]["keep"]) < cfg.rank for s in ("K", "V"))
    res = oracle.wo_correction(layer["H_calib"], layer["W_Q"], layer["W_K"], layer["W_V"],
                               layer["W_O"], codec, cfg.n_q_heads, 1, cfg.d_head)
    H = layer["H_calib"].astype(np.float64)
    for h, M in enumerate(res["M"]):
        q = H @ layer["W_Q"][:, h * 16:(h + 1) * 16]
        k = H @ layer["W_K"][:, :16]
        v = H @ layer["W_V"][:, :16]
        tr = []
        for side, x in (("K", k), ("V", v)):
            hs = codec["heads"][0][side]
            Vr = hs["V"][:, hs["keep"]]
            tr.append(x @ Vr @ Vr.T)
        O = oracle.causal_attention(q, k, v)
        Oh = oracle.causal_attention(q, tr[0], tr[1])
        assert np.linalg.norm(Oh @ M - O) <= np.linalg.norm(Oh - O) * (1 + 1e-9)


def _orthogonal(n, rng):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))[None, :]


def _closed_form_case(eps_rel, seed=0):
    """A layer whose least-squares correction is known in closed form.

    With nothing truncated on the key side, the truncated and exact attention
    weights A are equal.  The value weights are built as W_V = W_c X with
    X = U^T + B U_perp^T (U: kept value directions, U_perp: dropped ones, B
    arbitrary), so the dropped value components are a fixed linear function of
    the kept ones: the latent output is L = A H W_c and the exact output is
    O = A H W_V = L X.  W_c is chosen so that L^T L = c I.  The least-squares map
    of the reading, M' = (L^T L + eps I)^-1 L^T O with eps = eps_rel tr(L^T L)/n_kept,
    is then exactly X / (1 + eps_rel), and M = U M'."""
    rng = np.random.default_rng(seed)
    n, d_model, d_h, nk = 64, 24, 8, 4
    H = rng.standard_normal((n, d_model))
    W_Q = rng.standard_normal((d_model, d_h)) * 0.3
    W_K = rng.standard_normal((d_model, d_h)) * 0.3
    W_O = rng.standard_normal((d_h, d_model))
    # causal softmax attention weights, written out here independently of the oracle
    s = (H @ W_Q) @ (H @ W_K).T / np.sqrt(d_h)
    s[np.triu_indices(n, 1)] = -np.inf
    A = np.exp(s - s.max(axis=1, keepdims=True))
    A /= A.sum(axis=1, keepdims=True)
    Q1, R1 = np.linalg.qr(A @ H)
    c = 3.7
    W_c = np.sqrt(c) * np.linalg.inv(R1)[:, :nk]      # A H W_c = sqrt(c) Q1[:, :nk]
    Vfull = _orthogonal(d_h, rng)
    U, U_perp = Vfull[:, :nk], Vfull[:, nk:]
    Bm = rng.standard_normal((nk, d_h - nk))
    X = U.T + Bm @ U_perp.T
    W_V = W_c @ X
    codec = {"heads": [{"K": {"V": _orthogonal(d_h, rng), "keep": np.arange(d_h)},
                        "V": {"V": Vfull, "keep": np.arange(nk)}}]}
    res = oracle.wo_correction(H, W_Q, W_K, W_V, W_O, codec, 1, 1, d_h, eps_rel=eps_rel)
    return res, U @ X / (1.0 + eps_rel), W_O, U


def test_closed_form_correction_recovers_dropped_value_directions():
    res, M_expected, W_O, U = _closed_form_case(eps_rel=1e-13)
    np.testing.assert_allclose(res["M"][0], M_expected, rtol=0, atol=1e-9)
    np.testing.assert_allclose(res["W_O"], M_expected @ W_O, rtol=0, atol=1e-8)
    # the correction is not the bare projector onto the kept directions
    assert np.abs(M_expected - U @ U.T).max() > 0.1


def test_closed_form_regularisation_scales_with_mean_eigenvalue():
    # eps = eps_rel tr(L^T L) / n_kept = eps_rel c  ->  M' = X / (1 + eps_rel)
    for eps_rel in (0.25, 1.0):
        res, M_expected, W_O, _ = _closed_form_case(eps_rel=eps_rel, seed=1)
        np.testing.assert_allclose(res["M"][0], M_expected, rtol=0, atol=1e-9)
        np.testing.assert_allclose(res["W_O"], M_expected @ W_O, rtol=0, atol=1e-8)
