"""Shared helpers of the GPU parity tests: codecs with seeded factors, oracle
references computed from the same inputs, comparison metrics."""
from __future__ import annotations

import numpy as np

import oracle
from workloads import bf16_round


def torch_mod():
    import torch
    return torch


def dev():
    return torch_mod().device("cuda:0")


def make_cfg(d_model, n_q, n_kv, d_h, rank, group, budget, overhead, P):
    from spectral_transform_coding_b200.codec import make_config
    return make_config(d_model, n_q, n_kv, d_h, rank, group, budget, overhead, P)


def random_factors(d_model, n_kv, d_h, rank, group, widths, seed=0, w_std=0.02):
    """Seeded W_down (bf16 values) for the kept columns and orthonormal W_up rows."""
    rng = np.random.default_rng(seed)
    ng = rank // group
    widths = np.asarray(widths, np.int32).reshape(n_kv, 2, ng)
    n_eff = int(sum(group for a in range(n_kv) for s in range(2) for b in widths[a, s] if b > 0))
    W_down = bf16_round((rng.standard_normal((d_model, max(n_eff, 1))) * w_std).astype(np.float32))
    W_down = W_down[:, :n_eff]
    W_up = np.zeros((n_kv, 2, rank, d_h), np.float32)
    for a in range(n_kv):
        for s in range(2):
            q, _ = np.linalg.qr(rng.standard_normal((d_h, d_h)))
            W_up[a, s] = q[:, :rank].T.astype(np.float32)
    return widths, W_down, W_up


def codec_from(cfg, widths, W_down, W_up):
    import spectral_transform_coding_b200 as st
    return st.Codec.from_factors(cfg, widths, W_down, W_up)


def oracle_widths(widths):
    return [[widths[a, 0], widths[a, 1]] for a in range(widths.shape[0])]


def kept_wup(W_up, widths, group):
    return [[W_up[a, s][oracle.nonzero_coords(widths[a, s], group)] for s in range(2)]
            for a in range(widths.shape[0])]


def synthetic_latents(T, n_eff, seed, decay=0.7, scale=1.0):
    """fp32 latents with a decaying per-column scale and a few exact ties/constants."""
    rng = np.random.default_rng(seed)
    col_scale = scale * (np.arange(n_eff) % 128 + 1.0) ** -decay
    x = (rng.standard_normal((T, n_eff)) * col_scale[None, :]).astype(np.float32)
    if T > 3 and n_eff >= 16:
        x[1, :16] = 0.25   # a constant group (scale 0)
        x[2, :16] = np.float32(1e-8) * np.arange(16, dtype=np.float32)  # a subnormal-scale group
    return x


def oracle_pool_after(cfg_py, widths, pool_bytes_total, page_bytes, table, lengths0, seq_ids, latents, P,
                      base_pool=None):
    pool = np.zeros(pool_bytes_total, np.uint8) if base_pool is None else base_pool.copy()
    lay = oracle.page_layout(oracle_widths(widths), cfg_py["group"], P)
    assert lay["page_bytes"] == page_bytes
    new_len = oracle.append_tokens(pool, page_bytes, lay, oracle_widths(widths), cfg_py["group"], P, table,
                                   lengths0, seq_ids, latents, widths.shape[0])
    return pool, new_len, lay


def attention_rel_err(got, ref):
    """max over (b, q head) of ||got - ref||_inf / ||ref||_inf."""
    got = np.asarray(got, np.float64)
    num = np.abs(got - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return float((num / np.maximum(den, 1e-30)).max())
