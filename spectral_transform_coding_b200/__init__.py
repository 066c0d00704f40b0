"""Python binding of libspectra, a B200 (sm_100a) SPECTRA-style latent KV-cache codec.

Every function here marshals arguments into the C ABI declared in
``include/spectra.h``; all computation runs in ``libspectra.so``.  PyTorch only
supplies device memory and streams.  Importing this package without a built
library raises ``ImportError`` (there is no fallback implementation).
"""
from __future__ import annotations

import ctypes
import os

from ._lib import (  # noqa: F401
    SPECTRA_BF16,
    SPECTRA_F32,
    STATUS_NAMES,
    Config,
    SpectraError,
    lib,
    lib_path,
)
from .codec import Codec, LatentCache  # noqa: F401

__all__ = ["Codec", "LatentCache", "Config", "SpectraError", "lib", "lib_path",
           "SPECTRA_F32", "SPECTRA_BF16"]
