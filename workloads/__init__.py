"""Seeded synthetic workloads shared by the tests, the oracle checks and the bench.

This package holds shapes and random-input generators only.  It contains none of
the codec's arithmetic (no Gram, no eigen-basis, no bit allocation, no
quantisation): both the CUDA path and the CPU oracle receive the bytes produced
here and nothing else.
"""
from .configs import CONFIGS, WorkloadConfig, get_config  # noqa: F401
from .synthetic import (  # noqa: F401
    bf16_round,
    make_activations,
    make_layer,
    make_queries,
    make_weights,
    random_factors,
    spawn,
    synthetic_latents,
)
