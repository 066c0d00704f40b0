"""Pins of the oracle's reconstruction and attention (SPECTRA technical summary,
"SPECTRA pipeline" stage 3: keys and values rebuilt for standard attention;
"Significance and claims": attention directly in the latent space)."""
import math

import numpy as np
import pytest

import oracle
from workloads import make_activations, make_queries


def test_single_token_returns_its_value():
    rng = np.random.default_rng(0)
    K, V, q = rng.standard_normal((1, 8)), rng.standard_normal((1, 8)), rng.standard_normal(8)
    np.testing.assert_array_equal(oracle.softmax_attention(q, K, V), V[0])


def test_uniform_scores_return_the_mean():
    rng = np.random.default_rng(1)
    K, V = rng.standard_normal((37, 16)), rng.standard_normal((37, 16))
    np.testing.assert_allclose(oracle.softmax_attention(np.zeros(16), K, V), V.mean(axis=0),
                               rtol=1e-14, atol=1e-15)


def test_two_token_closed_form():
    d = 4
    K = np.array([[1.0, 0, 0, 0], [0, 2.0, 0, 0]])
    V = np.array([[1.0, 0, 0, 0], [0, 0, 0, 1.0]])
    q = np.array([0.5, 1.5, 0, 0])
    s1, s2 = 0.5 / math.sqrt(d), 3.0 / math.sqrt(d)
    p1 = 1.0 / (1.0 + math.exp(s2 - s1))
    np.testing.assert_allclose(oracle.softmax_attention(q, K, V), [p1, 0, 0, 1 - p1], rtol=1e-15)


def test_latent_fold_identity(toy_cfg, toy_codec):
    """q . k_hat = (q W_up^T) . c_hat for the rebuilt key k_hat = c_hat W_up."""
    rng = np.random.default_rng(2)
    hs = toy_codec["heads"][0]["K"]
    c = rng.standard_normal((50, hs["W_up"].shape[0]))
    q = rng.standard_normal(toy_cfg.d_head)
    direct = (c @ hs["W_up"]) @ q
    folded = c @ (hs["W_up"] @ q)
    np.testing.assert_allclose(folded, direct, rtol=1e-12, atol=1e-12 * np.abs(direct).max())


def test_zero_width_equals_rank_truncation(toy_cfg, toy_layer, toy_codec):
    """Dropping the b = 0 groups is the same as deleting those columns of W_down
    and rows of W_up, bit for bit in fp64."""
    hs = toy_codec["heads"][0]["V"]
    W = np.asarray(toy_layer["W_V"], np.float64)
    Vr = hs["V"][:, :toy_cfg.rank]
    h = toy_layer["H_calib"][:64].astype(np.float64)
    # full-rank latents with the dropped groups zeroed
    c_full = h @ (W @ Vr)
    mask = np.zeros(toy_cfg.rank, bool)
    mask[hs["keep"]] = True
    c_zeroed = np.where(mask[None, :], c_full, 0.0)
    rec_a = c_zeroed[:, hs["keep"]] @ hs["W_up"]
    rec_b = (h @ hs["W_down"]) @ hs["W_up"]
    np.testing.assert_array_equal(rec_a, rec_b)
    # and it is the orthogonal projection of k = h W onto the kept directions
    P = Vr[:, hs["keep"]] @ Vr[:, hs["keep"]].T
    np.testing.assert_allclose(rec_b, (h @ W) @ P, rtol=0, atol=1e-12 * np.abs(rec_b).max())


def _toy_cache(cfg, codec, n_tokens, P=64):
    widths = [[codec["heads"][0]["K"]["widths"], codec["heads"][0]["V"]["widths"]]]
    lay = oracle.page_layout(widths, cfg.group, P)
    n_pages = (n_tokens + P - 1) // P
    pool = np.zeros(lay["page_bytes"] * n_pages, np.uint8)
    table = np.arange(n_pages, dtype=np.int32)[None, :]
    h = make_activations(cfg, n_tokens, stream=3)
    lat = (h.astype(np.float64) @ codec["W_down"]).astype(np.float32)
    lengths = oracle.append_tokens(pool, lay["page_bytes"], lay, widths, cfg.group, P, table,
                                   np.zeros(1, np.int64), np.zeros(n_tokens, np.int64), lat, 1)
    return pool, lay, table, lengths, h, lat, widths


def test_decode_reference_equals_direct_reconstruction(toy_cfg, toy_codec):
    """Cache round trip: append (quantise + pack) then read back equals the direct
    quantise -> dequantise -> rebuild -> softmax attention, including a partial page."""
    n = 200
    pool, lay, table, lengths, h, lat, widths = _toy_cache(toy_cfg, toy_codec, n)
    assert int(lengths[0]) == n
    q = make_queries(toy_cfg, 1)
    W_up = [[toy_codec["heads"][0]["K"]["W_up"], toy_codec["heads"][0]["V"]["W_up"]]]
    out = oracle.decode_reference(pool, lay["page_bytes"], lay, toy_cfg.group, 64, table, lengths,
                                  q, W_up, toy_cfg.n_q_heads, 1)
    nk = len(toy_codec["heads"][0]["K"]["keep"])
    cK = np.concatenate([oracle.dequantize_groups(c, s, z) for _, c, s, z in
                         oracle.quantize_side(lat[:, :nk], widths[0][0], 8)], axis=1)
    cV = np.concatenate([oracle.dequantize_groups(c, s, z) for _, c, s, z in
                         oracle.quantize_side(lat[:, nk:], widths[0][1], 8)], axis=1)
    K = cK @ W_up[0][0]
    V = cV @ W_up[0][1]
    for hq in range(toy_cfg.n_q_heads):
        ref = oracle.softmax_attention(q[0, hq], K, V)
        np.testing.assert_allclose(out[0, hq], ref, rtol=1e-13, atol=1e-13)


def test_quantised_attention_close_to_exact(toy_cfg, toy_layer, toy_codec):
    """Sanity of the whole chain: the 2-bit toy codec's attention output is close to
    exact attention over uncompressed keys/values (loose, statistical)."""
    n = 256
    pool, lay, table, lengths, h, lat, widths = _toy_cache(toy_cfg, toy_codec, n)
    q = make_queries(toy_cfg, 1, score_std=1.0)
    W_up = [[toy_codec["heads"][0]["K"]["W_up"], toy_codec["heads"][0]["V"]["W_up"]]]
    out = oracle.decode_reference(pool, lay["page_bytes"], lay, 8, 64, table, lengths, q, W_up, 4, 1)
    K = h.astype(np.float64) @ toy_layer["W_K"]
    V = h.astype(np.float64) @ toy_layer["W_V"]
    for hq in range(4):
        ref = oracle.softmax_attention(q[0, hq], K, V)
        cos = out[0, hq] @ ref / np.linalg.norm(out[0, hq]) / np.linalg.norm(ref)
        assert cos > 0.8


# --- rotary position embedding of the reconstruct-then-attend path -------------------

def test_rope_is_identity_at_position_zero_and_preserves_norms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 16))
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(5), 10000.0), x)
    y = oracle.rope(x, np.arange(5) * 37, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((1, 32)), rng.standard_normal((1, 32))
    s1 = oracle.rope(q, np.array([10]), 500.0) @ oracle.rope(k, np.array([3]), 500.0).T
    s2 = oracle.rope(q, np.array([1007]), 500.0) @ oracle.rope(k, np.array([1000]), 500.0).T
    np.testing.assert_allclose(s1, s2, rtol=1e-10)


def test_rope_pair_rotation_by_hand():
    """d = 4, theta = 100: pair (x0, x2) turns by p * 100^0 = p, pair (x1, x3) by
    p * 100^(-1/2) = p / 10; at p = pi/2 the first pair maps (1, 0) -> (0, 1)."""
    x = np.array([[1.0, 0.0, 0.0, 2.0]])
    y = oracle.rope(x, np.array([np.pi / 2]), 100.0)
    a2 = np.pi / 20
    np.testing.assert_allclose(y[0], [0.0, -2 * np.sin(a2), 1.0, 2 * np.cos(a2)], atol=1e-15)


def test_rope_decode_without_rotation_equals_latent_route(toy_cfg, toy_codec):
    """theta = 0: reconstruct-then-attend is the same function as the pinned
    latent-space reference on the same pool."""
    pool, lay, table, lengths, h, lat, widths = _toy_cache(toy_cfg, toy_codec, 150)
    q = make_queries(toy_cfg, 1)
    W_up = [[toy_codec["heads"][0]["K"]["W_up"], toy_codec["heads"][0]["V"]["W_up"]]]
    a = oracle.decode_reference(pool, lay["page_bytes"], lay, toy_cfg.group, 64, table, lengths, q, W_up,
                                toy_cfg.n_q_heads, 1)
    b = oracle.decode_reference_rope(pool, lay["page_bytes"], lay, toy_cfg.group, 64, table, lengths, q, W_up,
                                     toy_cfg.n_q_heads, 1, 0.0)
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-13)


def test_rope_decode_equals_rotation_matrices(toy_cfg, toy_codec):
    """With rotation: the same attention written with explicit d x d rotation
    matrices R(p) (pair (i, i + d/2) turned by p * theta^(-2i/d)), keys at
    positions 0..n-1, the query at n-1."""
    n, theta = 130, 50.0
    pool, lay, table, lengths, h, lat, widths = _toy_cache(toy_cfg, toy_codec, n)
    q = make_queries(toy_cfg, 1)
    W_up = [[toy_codec["heads"][0]["K"]["W_up"], toy_codec["heads"][0]["V"]["W_up"]]]
    out = oracle.decode_reference_rope(pool, lay["page_bytes"], lay, toy_cfg.group, 64, table, lengths, q, W_up,
                                       toy_cfg.n_q_heads, 1, theta)
    cK = oracle.read_side(pool, lay["page_bytes"], lay, toy_cfg.group, 64, table[0], n, 0, 0)
    cV = oracle.read_side(pool, lay["page_bytes"], lay, toy_cfg.group, 64, table[0], n, 0, 1)
    K, V = cK @ W_up[0][0], cV @ W_up[0][1]
    d = K.shape[1]
    hd = d // 2

    def R(p):
        m = np.zeros((d, d))
        for i in range(hd):
            a = p * theta ** (-2.0 * i / d)
            m[i, i], m[i, i + hd] = math.cos(a), -math.sin(a)
            m[i + hd, i], m[i + hd, i + hd] = math.sin(a), math.cos(a)
        return m

    Kr = np.stack([R(t) @ K[t] for t in range(n)])
    for hq in range(toy_cfg.n_q_heads):
        qr = R(n - 1) @ q[0, hq].astype(np.float64)
        s = Kr @ qr / math.sqrt(d)
        e = np.exp(s - s.max())
        np.testing.assert_allclose(out[0, hq], (e / e.sum()) @ V, rtol=1e-11, atol=1e-12)
