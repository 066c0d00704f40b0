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
