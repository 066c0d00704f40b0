"""Seeded synthetic inputs (numpy PCG64).

Streams per workload seed (``spawn``): 0 weights, 1 activation basis,
2 calibration activations, 3 cache activations, 4 queries, 5 Student-t scales.

Activations: ``h = z * sqrt(lambda) @ Q^T`` with ``z ~ N(0, I)``,
``lambda_i = i^-alpha`` and ``Q`` a random orthogonal basis.  For the toy layer
``Q`` is Haar (QR of a Gaussian matrix with the sign of diag(R) folded in); for
wide layers (d_model >= 1024) ``Q = Q1 (x) Q2`` is a Kronecker product of two Haar
factors, which is orthogonal and mixes every coordinate but costs O(d^1.5) to
apply.  (The weights are i.i.d. Gaussian, so the law of W^T G W does not depend
on the basis of G.)  Student-t: every token is multiplied by ``sqrt(nu / w)``,
``w ~ chi2(nu)``, one ``w`` per token.

Everything returned is float32; with ``w_bf16`` the values are rounded to the
nearest bfloat16 (ties to even) so that a bf16 copy on the GPU holds the same
numbers.
"""
from __future__ import annotations

import functools

import numpy as np

from .configs import WorkloadConfig

STREAM_WEIGHTS, STREAM_BASIS, STREAM_CALIB, STREAM_CACHE, STREAM_QUERY, STREAM_TSCALE = range(6)


def spawn(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=seed, spawn_key=(stream, sub))
    return np.random.Generator(np.random.PCG64(ss))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16, ties to even (returns float32)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    out = u.astype(np.uint32).view(np.float32)
    return np.where(np.isnan(x), x, out)


def _haar(n: int, rng: np.random.Generator) -> np.ndarray:
    a = rng.standard_normal((n, n))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def _kron_factors(d: int) -> tuple[int, int]:
    best = (1, d)
    for a in range(1, int(d ** 0.5) + 1):
        if d % a == 0:
            best = (a, d // a)
    return best


@functools.lru_cache(maxsize=8)
def _basis(d: int, seed: int):
    rng = spawn(seed, STREAM_BASIS)
    if d < 1024:
        return ("full", _haar(d, rng))
    a, b = _kron_factors(d)
    return ("kron", _haar(a, rng), _haar(b, rng))


def _apply_basis_t(y: np.ndarray, basis) -> np.ndarray:
    """Return y @ Q^T for the basis returned by ``_basis``."""
    if basis[0] == "full":
        return y @ basis[1].T
    _, q1, q2 = basis
    a, b = q1.shape[0], q2.shape[0]
    n = y.shape[0]
    # (Q1 (x) Q2) maps e_i (x) e_j; y @ (Q1 (x) Q2)^T = reshape -> Q1 Y Q2^T.
    y3 = y.reshape(n, a, b)
    y3 = np.einsum("ia,nab->nib", q1, y3, optimize=True)
    y3 = np.einsum("nib,jb->nij", y3, q2, optimize=True)
    return y3.reshape(n, a * b)


def make_activations(cfg: WorkloadConfig, n: int, stream: int, sub: int = 0) -> np.ndarray:
    """``n`` activation rows ``[n, d_model]`` (float32, bf16 values if cfg.w_bf16)."""
    rng = spawn(cfg.seed, stream, sub)
    lam = np.arange(1, cfg.d_model + 1, dtype=np.float64) ** (-cfg.spectrum_exp)
    y = rng.standard_normal((n, cfg.d_model)) * np.sqrt(lam)[None, :]
    h = _apply_basis_t(y, _basis(cfg.d_model, cfg.seed))
    if cfg.dist == "student_t":
        trng = spawn(cfg.seed, STREAM_TSCALE, stream * 1000 + sub)
        w = trng.chisquare(cfg.nu, size=n)
        h = h * np.sqrt(cfg.nu / w)[:, None]
    h = h.astype(np.float32)
    return bf16_round(h) if cfg.w_bf16 else h


def make_weights(cfg: WorkloadConfig) -> dict:
    """W_K, W_V ``[d_model, H_kv*d_h]``, W_Q ``[d_model, H_q*d_h]``, W_O ``[H_q*d_h, d_model]``."""
    rng = spawn(cfg.seed, STREAM_WEIGHTS)
    kv = cfg.n_kv_heads * cfg.d_head
    qd = cfg.n_q_heads * cfg.d_head
    out = {}
    for name, shape in (("W_K", (cfg.d_model, kv)), ("W_V", (cfg.d_model, kv)),
                        ("W_Q", (cfg.d_model, qd)), ("W_O", (qd, cfg.d_model))):
        w = (rng.standard_normal(shape) * cfg.w_std).astype(np.float32)
        out[name] = bf16_round(w) if cfg.w_bf16 else w
    return out


def make_queries(cfg: WorkloadConfig, batch: int, sub: int = 0,
                 score_std: float = 2.0, peaked: bool = False,
                 keys_sample: np.ndarray | None = None) -> np.ndarray:
    """fp32 queries ``[batch, H_q, d_h]``.

    Flat set: Gaussian directions scaled so that ``q.k/sqrt(d_h)`` has standard
    deviation ``score_std`` over ``keys_sample`` (``[n, H_kv, d_h]``, e.g. the
    uncompressed keys of a few cache tokens); without a sample the scale assumes
    unit-variance keys.  Peaked set: each query is the (scaled) key of one
    planted sample token plus noise, so one token dominates its softmax.
    """
    rng = spawn(cfg.seed, STREAM_QUERY, sub)
    q = rng.standard_normal((batch, cfg.n_q_heads, cfg.d_head))
    if peaked and keys_sample is not None:
        idx = rng.integers(0, keys_sample.shape[0], size=(batch, cfg.n_q_heads))
        for b in range(batch):
            for h in range(cfg.n_q_heads):
                k = keys_sample[idx[b, h], h // cfg.gq].astype(np.float64)
                kk = max(float(k @ k), 1e-30)
                # q.k/sqrt(d_h) = peak_score for the planted token.
                q[b, h] = k * (8.0 * np.sqrt(cfg.d_head) / kk) \
                    + 0.05 * q[b, h] * np.sqrt(np.sqrt(cfg.d_head) / kk)
        return q.astype(np.float32)
    if keys_sample is not None:
        for h in range(cfg.n_q_heads):
            ks = keys_sample[:, h // cfg.gq, :].astype(np.float64)
            s = ks @ q[:, h, :].T / np.sqrt(cfg.d_head)
            sd = float(np.std(s)) or 1.0
            q[:, h, :] *= score_std / sd
    else:
        q *= score_std
    return q.astype(np.float32)


def make_layer(cfg: WorkloadConfig, calib_tokens: int | None = None) -> dict:
    """Weights plus calibration activations for one layer."""
    w = make_weights(cfg)
    n = cfg.calib_tokens if calib_tokens is None else calib_tokens
    w["H_calib"] = make_activations(cfg, n, STREAM_CALIB)
    return w


# ----------------------------------------------------------------------------
# Inputs of the library-level parity checks: codec factors and latents drawn
# directly (no calibration), so both sides start from identical numbers.
# ----------------------------------------------------------------------------

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


def synthetic_latents(T, n_eff, seed, decay=0.7, scale=1.0):
    """fp32 latents with a decaying per-column scale and a few exact ties/constants."""
    rng = np.random.default_rng(seed)
    col_scale = scale * (np.arange(n_eff) % 128 + 1.0) ** -decay
    x = (rng.standard_normal((T, n_eff)) * col_scale[None, :]).astype(np.float32)
    if T > 3 and n_eff >= 16:
        x[1, :16] = 0.25   # a constant group (scale 0)
        x[2, :16] = np.float32(1e-8) * np.arange(16, dtype=np.float32)  # a subnormal-scale group
    return x
