"""CPU oracle for the SPECTRA-style latent KV-cache codec.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  The
library under ``spectral_transform_coding_b200`` never imports, links or runs
anything in this package, and this package imports nothing from the library.
"""
from .spectra_oracle import *  # noqa: F401,F403
