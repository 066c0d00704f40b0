"""Allocation ablation: grouped reverse water-filling against uniform widths.

"SPECTRA: Pushing the KV Cache Beyond the 2-Bit Cliff via Spectral Transform
Coding" allocates bits by reverse water-filling ("SPECTRA pipeline", stage 2);
"Ablation, Statistical Inference, and Validation for KV-Cache Compression"
reports that uniform allocation does about as well on synthetic data and that
eigen-basis codecs suffer on heavy-tailed data; "Spectral-KV: SVD-projection KV
cache compression (28x)" truncates at an energy threshold.  This tool measures
those claims with this library's codec: for each data law and budget it
calibrates with each allocation, encodes held-out tokens, and reports

* relMSE_K, relMSE_V: sum ||k^ - k||^2 / sum ||k||^2 over the held-out tokens
  and KV heads (k^ rebuilt from the packed cache by spectra_reconstruct, k exact
  from the layer's weights);
* attention error: max over q heads of ||o^ - o||_inf / ||o||_inf between the
  latent decode (spectra_decode_attend) and exact softmax attention over the
  exact keys and values (fp64).

Run on a GPU:  python -m spectral_transform_coding_b200.ablation [--tokens N]
One JSON line per (law, budget, allocation).  Inputs are seeded synthetic
layers (the workloads package), not a model.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys


def _acts(torch, cfg, n, seed, dev, basis):
    """h = z sqrt(lambda) Q^T (Student-t: times sqrt(nu / w)), bf16, on the GPU."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    lam = torch.arange(1, cfg.d_model + 1, device=dev, dtype=torch.float32) ** (-cfg.spectrum_exp)
    y = torch.randn((n, cfg.d_model), generator=gen, device=dev) * lam.sqrt()
    q1 = torch.from_numpy(basis[1]).to(dev, torch.float32)
    if basis[0] == "kron":
        q2 = torch.from_numpy(basis[2]).to(dev, torch.float32)
        a, b = q1.shape[0], q2.shape[0]
        h = torch.einsum("ia,nab,jb->nij", q1, y.view(n, a, b), q2).reshape(n, a * b)
    else:
        h = y @ q1.T
    if cfg.dist == "student_t":
        w = torch.distributions.Chi2(torch.tensor(cfg.nu, device=dev)).sample((n,))
        h = h * torch.sqrt(cfg.nu / w)[:, None]
    return h.to(torch.bfloat16)


def run(tokens: int = 4096, n_kv: int = 2, seed: int = 11):
    import torch

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import spectral_transform_coding_b200 as st
    from spectral_transform_coding_b200.codec import make_config
    from workloads import get_config
    from workloads.synthetic import _basis

    dev = torch.device("cuda", 0)
    out = []
    for law in ("llama", "stress"):
        for budget in (512, 256):
            cfg = get_config(law, n_kv_heads=n_kv, n_q_heads=4 * n_kv, budget_bits=budget)
            basis = _basis(cfg.d_model, cfg.seed)
            gen = torch.Generator(device=dev)
            gen.manual_seed(1000 * cfg.seed + 17)
            kvw = cfg.n_kv_heads * cfg.d_head
            W_K = (torch.randn((cfg.d_model, kvw), generator=gen, device=dev) * cfg.w_std).to(torch.bfloat16)
            W_V = (torch.randn((cfg.d_model, kvw), generator=gen, device=dev) * cfg.w_std).to(torch.bfloat16)
            H_cal = _acts(torch, cfg, cfg.calib_tokens, seed, dev, basis)
            H = _acts(torch, cfg, tokens, seed + 1, dev, basis)
            K = (H.double() @ W_K.double()).view(tokens, n_kv, cfg.d_head)
            V = (H.double() @ W_V.double()).view(tokens, n_kv, cfg.d_head)
            q = (torch.randn((1, cfg.n_q_heads, cfg.d_head), generator=gen, device=dev) * 0.5)
            gq = cfg.n_q_heads // n_kv
            # exact attention over the exact keys and values (fp64)
            o_ref = torch.empty((cfg.n_q_heads, cfg.d_head), dtype=torch.float64, device=dev)
            for h in range(cfg.n_q_heads):
                a = h // gq
                s = (K[:, a] @ q[0, h].double()) / math.sqrt(cfg.d_head)
                o_ref[h] = torch.softmax(s, 0) @ V[:, a]
            c = make_config(cfg.d_model, cfg.n_q_heads, n_kv, cfg.d_head, cfg.rank, cfg.group, budget,
                            cfg.count_overhead, cfg.page_tokens)
            for allocation, thr in (("waterfill", 0.0), ("uniform", 0.0), ("waterfill", 0.95),
                                    ("uniform", 0.95)):
                codec = st.Codec.calibrate(c, H_cal, W_K, W_V, allocation=allocation, energy_threshold=thr)
                P = cfg.page_tokens
                cache = st.LatentCache(codec, batch=1, max_pages_per_seq=(tokens + P - 1) // P, device=dev)
                codec.encode_append(cache, H, torch.zeros(tokens, dtype=torch.int32, device=dev))
                Kh, Vh = codec.reconstruct(cache, 0, 0, tokens)
                o = codec.decode_attend(cache, q)
                codec.device_status()
                rel_k = float(((Kh.double() - K) ** 2).sum() / (K ** 2).sum())
                rel_v = float(((Vh.double() - V) ** 2).sum() / (V ** 2).sum())
                err = ((o[0].double() - o_ref).abs().amax(1) / o_ref.abs().amax(1)).max().item()
                widths = codec.state()["widths"]
                out.append({
                    "law": "power-law gaussian" if law == "llama" else "student-t (nu=3)",
                    "budget_bits_per_side": budget, "compression_vs_fp16": 16 * cfg.d_head / budget,
                    "allocation": allocation, "energy_threshold": thr,
                    "relMSE_K": rel_k, "relMSE_V": rel_v, "attention_rel_err": err,
                    "kept_groups_per_side": [[int((w > 0).sum()) for w in head] for head in widths],
                    "widths_head0": [list(map(int, w)) for w in widths[0]],
                })
                codec.close()
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--kv-heads", type=int, default=2)
    a = ap.parse_args(argv)
    for r in run(a.tokens, a.kv_heads):
        print(json.dumps(r), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
