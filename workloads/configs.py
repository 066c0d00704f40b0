"""Workload shapes.

Each workload is a single attention layer shaped like a model that the SPECTRA
pages evaluate on ("SPECTRA: Pushing the KV Cache Beyond the 2-Bit Cliff via
Spectral Transform Coding", technical summary, "Experimental results": Llama-3.1-8B
and Qwen2.5-7B), with seeded random weights and activations whose covariance has
a power-law spectrum (or a heavy-tailed Student-t law, the regime that "Ablation,
Statistical Inference, and Validation for KV-Cache Compression" uses to stress
eigen-basis codecs, "Heavy-tailed data").

Budgets are bits per token, per KV head, per side (K or V).  "n x compression vs
fp16" means 16*d_head/n bits; with ``count_overhead`` every non-empty group also
pays 32 bits for its fp16 scale and fp16 zero.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    d_head: int
    rank: int            # latent coordinates kept per head and side (<= d_head)
    group: int           # adjacent latent coordinates sharing one bit width
    budget_bits: int     # per token, per KV head, per side
    count_overhead: bool
    page_tokens: int
    calib_tokens: int
    cache_len: int       # decode context per sequence
    batch: int           # decode sequences
    spectrum_exp: float  # lambda_i = i ** -spectrum_exp
    dist: str            # "gaussian" or "student_t"
    nu: float            # Student-t degrees of freedom (dist == "student_t")
    w_std: float         # std of W_K, W_V, W_Q, W_O entries
    w_bf16: bool         # weights and activations rounded to bf16
    seed: int
    prefill_tokens: int = 0

    @property
    def gq(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_groups(self) -> int:
        return self.rank // self.group

    @property
    def fp16_bits_per_side(self) -> int:
        return 16 * self.d_head

    def with_(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


_LLAMA = dict(d_model=4096, n_q_heads=32, n_kv_heads=8, d_head=128, rank=128,
              group=16, count_overhead=True, page_tokens=64, calib_tokens=8192,
              spectrum_exp=1.2, dist="gaussian", nu=0.0, w_std=0.02, w_bf16=True)

CONFIGS = {
    # single head, fp32 weights N(0, 1/256), lambda_i = i^-1.5, r = 32 in groups
    # of 8, 2 payload bits per latent coordinate (scale/zero not counted).
    "toy": WorkloadConfig(
        name="toy", d_model=256, n_q_heads=4, n_kv_heads=1, d_head=64, rank=32,
        group=8, budget_bits=64, count_overhead=False, page_tokens=64,
        calib_tokens=2048, cache_len=1024, batch=1, spectrum_exp=1.5,
        dist="gaussian", nu=0.0, w_std=1.0 / 16.0, w_bf16=False, seed=0),
    # Llama-3.1-8B-shaped layer, 4x vs fp16 including scale/zero, batch 1 @ 32k.
    "llama": WorkloadConfig(name="llama", budget_bits=512, cache_len=32768,
                            batch=1, seed=1, **_LLAMA),
    # Qwen2.5-7B-shaped layer, 8x (2 bits per original coordinate incl. overhead),
    # batch 1 @ 128k.
    "qwen": WorkloadConfig(
        name="qwen", d_model=3584, n_q_heads=28, n_kv_heads=4, d_head=128,
        rank=128, group=16, budget_bits=256, count_overhead=True, page_tokens=64,
        calib_tokens=8192, cache_len=131072, batch=1, spectrum_exp=2.0,
        dist="gaussian", nu=0.0, w_std=0.02, w_bf16=True, seed=2),
    # Llama shapes, multivariate Student-t (nu = 3) over the power-law
    # covariance, 12x (floor(2048/12) = 170 bits per side), batch 16 @ 32k, in
    # 128-token pages (the decode then takes 8-tile softmax chunks).
    "stress": WorkloadConfig(name="stress", budget_bits=170, cache_len=32768,
                             batch=16, seed=3,
                             **dict(_LLAMA, dist="student_t", nu=3.0, page_tokens=128)),
    # Llama shapes, one 65,536-token prefill chunk encoded for all KV heads at 4x
    # (and 8x, see ``prefill8``), followed by one decode step.
    "prefill": WorkloadConfig(name="prefill", budget_bits=512, cache_len=65536,
                              batch=1, seed=4, prefill_tokens=65536, **_LLAMA),
    "prefill8": WorkloadConfig(name="prefill8", budget_bits=256, cache_len=65536,
                               batch=1, seed=4, prefill_tokens=65536, **_LLAMA),
}


def get_config(name: str, **overrides) -> WorkloadConfig:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg
