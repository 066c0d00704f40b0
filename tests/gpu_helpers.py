"""Shared helpers of the GPU parity tests: codecs with seeded factors, oracle
references computed from the same inputs, comparison metrics."""
from __future__ import annotations

import numpy as np

import oracle
from workloads import random_factors, synthetic_latents  # noqa: F401  (seeded inputs)


def torch_mod():
    import torch
    return torch


def dev():
    return torch_mod().device("cuda:0")


def make_cfg(d_model, n_q, n_kv, d_h, rank, group, budget, overhead, P):
    from spectral_transform_coding_b200.codec import make_config
    return make_config(d_model, n_q, n_kv, d_h, rank, group, budget, overhead, P)


def codec_from(cfg, widths, W_down, W_up):
    import spectral_transform_coding_b200 as st
    return st.Codec.from_factors(cfg, widths, W_down, W_up)


def oracle_widths(widths):
    return [[widths[a, 0], widths[a, 1]] for a in range(widths.shape[0])]


def kept_wup(W_up, widths, group):
    return [[W_up[a, s][oracle.nonzero_coords(widths[a, s], group)] for s in range(2)]
            for a in range(widths.shape[0])]


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
