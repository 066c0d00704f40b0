"""GPU parity at the shapes the benchmark runs (Llama-3.1-8B- and Qwen2.5-7B-
shaped layers), through the C ABI.

- The decode-step fused encode at d_model 4096 and 3584, so that its loop over
  d_model slices runs more than once.
- The tcgen05 projection at K = d_model = 4096 with 1024 and 2048 latent
  columns and a row count that is not a multiple of the 128-row tile.
- The latent decode at 32,768 + 5 tokens with 8 KV heads (Llama 4x), at
  131,072 + 3 tokens with 7 q heads per KV head (Qwen 8x), and over 16
  sequences of 32,768 + 11 tokens with 8 KV heads at 12x (the heavy-tail stress
  layer's batch), checked on sampled (sequence, q head) pairs against the
  oracle's decode over its own copy of the pool, which must equal the library's
  byte for byte.  The decode's launch plan (split count, stages, chunk length)
  depends only on the head shapes, widths, page size and batch, so these runs
  use the benchmark's.

Bars as in the other parity tests: latents 1e-3 (per token and head-side, L2),
packed pages bit-exact, attention 2e-3 (max over the sampled pairs of
||diff||_inf / ||ref||_inf)."""
import numpy as np
import pytest

import oracle
from gpu_helpers import (attention_rel_err, codec_from, dev, kept_wup, make_cfg, oracle_widths, random_factors,
                         synthetic_latents, torch_mod)
from workloads import bf16_round

pytestmark = pytest.mark.gpu

LLAMA4X = [4, 2, 2, 2, 2, 2, 1, 1]          # widths of a Llama-shaped head side at 4x
QWEN8X_K = [4, 2, 1, 1, 0, 0, 0, 0]         # Qwen-shaped head at 8x
QWEN8X_V = [4, 3, 3, 0, 0, 0, 0, 0]
STRESS12X = [4, 2, 0, 0, 0, 0, 0, 0]        # 170 bits per side with scale/zero


def _codec(d_model, n_q, n_kv, wk, wv, seed, P=64):
    widths = np.array([[wk, wv]] * n_kv, np.int32)
    widths, W_down, W_up = random_factors(d_model, n_kv, 128, 128, 16, widths, seed=seed)
    cfg = make_cfg(d_model, n_q, n_kv, 128, 128, 16, 512, True, P)
    return codec_from(cfg, widths, W_down, W_up), widths, W_down, W_up


def _check_latents(lat, ref, widths):
    c0 = 0
    for a in range(widths.shape[0]):
        for side in range(2):
            nk = int(sum(16 for b in widths[a, side] if b > 0))
            d = lat[:, c0:c0 + nk] - ref[:, c0:c0 + nk]
            rel = np.linalg.norm(d, axis=1) / np.maximum(np.linalg.norm(ref[:, c0:c0 + nk], axis=1), 1e-30)
            assert rel.max() <= 1e-3, (a, side, rel.max())
            c0 += nk


@pytest.mark.parametrize("d_model,n_q,n_kv,wk,wv", [(4096, 32, 8, LLAMA4X, LLAMA4X),
                                                    (3584, 28, 4, QWEN8X_K, QWEN8X_V)])
@pytest.mark.parametrize("T", [1, 16])
def test_fused_encode_full_width(d_model, n_q, n_kv, wk, wv, T):
    """The fused decode-step encode over a full-width layer: latents within 1e-3
    of the oracle's H W_down, pages equal to what the (bit-exact) quantiser
    writes for the same latents, lengths advanced."""
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    codec, widths, W_down, _ = _codec(d_model, n_q, n_kv, wk, wv, seed=11)
    B = 2
    seqs = np.sort(np.arange(T, dtype=np.int32) % B)
    rng = np.random.default_rng(12 + T)
    H = bf16_round(rng.standard_normal((T, d_model)).astype(np.float32))
    table = np.arange(B * 2, dtype=np.int32).reshape(B, 2)
    c1 = st.LatentCache(codec, batch=B, max_pages_per_seq=2, device=dev(), page_table=torch.from_numpy(table))
    c2 = st.LatentCache(codec, batch=B, max_pages_per_seq=2, device=dev(), page_table=torch.from_numpy(table))
    start = np.array([5, 60], np.int32)  # mid-block; sequence 1 crosses into its second page
    c1.lengths.copy_(torch.from_numpy(start))
    c2.lengths.copy_(torch.from_numpy(start))
    lat = torch.empty((T, codec.n_eff), dtype=torch.float32, device=dev())
    codec.encode_append(c1, torch.from_numpy(H).to(dev()).to(torch.bfloat16), torch.from_numpy(seqs).to(dev()),
                        latents_out=lat)
    codec.device_status()
    _check_latents(lat.cpu().numpy(), H.astype(np.float64) @ W_down.astype(np.float64), widths)
    codec.quantize_append(c2, lat, torch.from_numpy(seqs).to(dev()))
    codec.device_status()
    assert np.array_equal(c1.pool.cpu().numpy(), c2.pool.cpu().numpy())
    np.testing.assert_array_equal(c1.lengths.cpu().numpy(), start + np.bincount(seqs, minlength=B))


def test_encode_staged_wait_gives_up_with_a_timeout_status(monkeypatch):
    """A staged W_down copy that never lands (test hook SPECTRA_ENCODE_TEST_DROP_STAGE:
    the first CTA skips its first staged copy) makes that CTA's bounded wait give
    up after the limit (SPECTRA_ENCODE_TEST_WAIT_NS: 2 ms).  The call reports
    SPECTRA_ERR_TIMEOUT through the device error word, every CTA still arrives,
    and later calls on the same workspace write exactly what a fresh workspace
    gives.  The Llama-shaped layer at one token stages the second half of each
    group's W_down rows."""
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    codec, _, _, _ = _codec(4096, 32, 8, LLAMA4X, LLAMA4X, seed=21)
    B = 2
    rng = np.random.default_rng(22)
    H = torch.from_numpy(bf16_round(rng.standard_normal((1, 4096)).astype(np.float32))).to(dev()).to(torch.bfloat16)
    seqs = torch.ones(1, dtype=torch.int32, device=dev())
    table = torch.from_numpy(np.arange(B * 2, dtype=np.int32).reshape(B, 2))

    def cache():
        return st.LatentCache(codec, batch=B, max_pages_per_seq=2, device=dev(), page_table=table)

    ws = torch.zeros(codec.encode_workspace_bytes(1), dtype=torch.uint8, device=dev())
    monkeypatch.setenv("SPECTRA_ENCODE_TEST_DROP_STAGE", "1")
    monkeypatch.setenv("SPECTRA_ENCODE_TEST_WAIT_NS", "2000000")
    codec.encode_append(cache(), H, seqs, workspace=ws)
    with pytest.raises(st.SpectraError) as e:
        codec.device_status()
    assert e.value.status == 6  # SPECTRA_ERR_TIMEOUT
    monkeypatch.delenv("SPECTRA_ENCODE_TEST_DROP_STAGE")
    monkeypatch.delenv("SPECTRA_ENCODE_TEST_WAIT_NS")
    for _ in range(2):
        c1, c2 = cache(), cache()
        codec.encode_append(c1, H, seqs, workspace=ws)
        codec.encode_append(c2, H, seqs, workspace=torch.zeros_like(ws))
        codec.device_status()
        assert torch.equal(c1.pool, c2.pool)
        np.testing.assert_array_equal(c1.lengths.cpu().numpy(), [0, 1])
        assert torch.equal(c1.lengths, c2.lengths)


@pytest.mark.parametrize("n_kv", [4, 8])
def test_projection_tcgen05_full_width(n_kv):
    """H W_down on the tcgen05 GEMM at K = 4096 (64 k-blocks) with N_eff = 128 n_kv
    latent columns (1024 or 2048) and 1000 rows (a ragged last M tile); checked
    on a sample of rows against the fp64 product of the same bf16 values."""
    torch = torch_mod()
    codec, widths, W_down, _ = _codec(4096, 4 * n_kv, n_kv, [2] * 8, [2] * 8, seed=13)
    assert codec.n_eff == 256 * n_kv
    rng = np.random.default_rng(14)
    H = bf16_round(rng.standard_normal((1000, 4096)).astype(np.float32))
    lat = codec.project(torch.from_numpy(H).to(dev()).to(torch.bfloat16)).cpu().numpy()
    rows = np.r_[0:8, 120:136, rng.choice(1000, 40, replace=False), 992:1000]
    _check_latents(lat[rows], H[rows].astype(np.float64) @ W_down.astype(np.float64), widths)


def _long_decode(n_q, n_kv, wk, wv, length, pairs, seed):
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    codec, widths, _, W_up = _codec(512, n_q, n_kv, wk, wv, seed=seed)
    P = 64
    maxp = (length + P - 1) // P + 1
    rng = np.random.default_rng(seed + 1)
    table = rng.permutation(maxp).astype(np.int32)[None, :]
    cache = st.LatentCache(codec, batch=1, max_pages_per_seq=maxp, device=dev(), page_table=torch.from_numpy(table))
    lay = oracle.page_layout(oracle_widths(widths), 16, P)
    pool = np.zeros(cache.pool.numel(), np.uint8)
    lengths = np.zeros(1, np.int64)
    chunk = 8192
    for t0 in range(0, length, chunk):
        n = min(chunk, length - t0)
        lat = synthetic_latents(n, codec.n_eff, seed=seed + 2 + t0 // chunk, decay=0.5, scale=2.0)
        seqs = np.zeros(n, np.int32)
        codec.quantize_append(cache, torch.from_numpy(lat).to(dev()), torch.from_numpy(seqs).to(dev()))
        lengths = oracle.append_tokens(pool, codec.page_bytes, lay, oracle_widths(widths), 16, P, table, lengths,
                                       seqs, lat, n_kv)
    codec.device_status()
    assert int(cache.lengths.cpu()[0]) == length
    assert np.array_equal(cache.pool.cpu().numpy(), pool), "packed cache differs from the oracle's"
    q = (rng.standard_normal((1, n_q, 128)) * 0.6).astype(np.float32)
    out = codec.decode_attend(cache, torch.from_numpy(q).to(dev())).cpu().numpy()
    codec.device_status()
    ref = oracle.decode_reference(pool, codec.page_bytes, lay, 16, P, table, np.array([length]), q,
                                  kept_wup(W_up, widths, 16), n_q, n_kv, pairs=pairs)
    got = np.stack([out[b, h] for b, h in pairs])
    want = np.stack([ref[b, h] for b, h in pairs])
    return attention_rel_err(got, want)


def test_decode_llama_32k_context_8_kv_heads():
    err = _long_decode(32, 8, LLAMA4X, LLAMA4X, 32768 + 5, [(0, 0), (0, 13), (0, 31)], seed=21)
    assert err <= 2e-3, err


def test_decode_qwen_128k_context_gqa7():
    err = _long_decode(28, 4, QWEN8X_K, QWEN8X_V, 131072 + 3, [(0, 0), (0, 20), (0, 27)], seed=31)
    assert err <= 2e-3, err


def test_decode_stress_12x_batch16_32k():
    """16 sequences at 32k with 8 KV heads, 12x widths and the stress workload's
    128-token pages (8-tile softmax chunks).  Sequences 0 and 11
    (sampled) are filled with seeded latents on both sides; the other 14 with
    device-drawn latents that only the library sees (their pages are not
    compared, their outputs not checked)."""
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    seed, n_q, n_kv, B, length, P = 41, 32, 8, 16, 32768 + 11, 128
    sampled = [0, 11]
    codec, widths, _, W_up = _codec(512, n_q, n_kv, STRESS12X, STRESS12X, seed=seed, P=P)
    maxp = (length + P - 1) // P + 1
    rng = np.random.default_rng(seed + 1)
    table = rng.permutation(B * maxp).astype(np.int32).reshape(B, maxp)
    cache = st.LatentCache(codec, batch=B, max_pages_per_seq=maxp, device=dev(), page_table=torch.from_numpy(table))
    lay = oracle.page_layout(oracle_widths(widths), 16, P)
    pool = np.zeros(cache.pool.numel(), np.uint8)
    lengths = np.zeros(B, np.int64)
    gen = torch.Generator(device=dev())
    gen.manual_seed(seed + 2)
    chunk = 8192
    for b in range(B):
        for t0 in range(0, length, chunk):
            n = min(chunk, length - t0)
            seqs = np.full(n, b, np.int32)
            if b in sampled:
                lat = synthetic_latents(n, codec.n_eff, seed=seed + 3 + 100 * b + t0 // chunk, decay=0.5, scale=2.0)
                lengths = oracle.append_tokens(pool, codec.page_bytes, lay, oracle_widths(widths), 16, P, table,
                                               lengths, seqs, lat, n_kv)
                lat_d = torch.from_numpy(lat).to(dev())
            else:
                lat_d = torch.randn((n, codec.n_eff), generator=gen, device=dev()) * 2.0
            codec.quantize_append(cache, lat_d, torch.from_numpy(seqs).to(dev()))
    codec.device_status()
    assert cache.lengths.cpu().tolist() == [length] * B
    got_pool = cache.pool.cpu().numpy()
    for b in sampled:
        for pg in table[b, :(length + P - 1) // P]:
            sl = slice(int(pg) * codec.page_bytes, (int(pg) + 1) * codec.page_bytes)
            assert np.array_equal(got_pool[sl], pool[sl]), f"page {pg} of sequence {b} differs from the oracle's"
    q = (rng.standard_normal((B, n_q, 128)) * 0.6).astype(np.float32)
    out = codec.decode_attend(cache, torch.from_numpy(q).to(dev())).cpu().numpy()
    codec.device_status()
    pairs = [(0, 0), (0, 17), (11, 5), (11, 31)]
    ref = oracle.decode_reference(pool, codec.page_bytes, lay, 16, P, table, lengths, q,
                                  kept_wup(W_up, widths, 16), n_q, n_kv, pairs=pairs)
    err = attention_rel_err(np.stack([out[b, h] for b, h in pairs]), np.stack([ref[b, h] for b, h in pairs]))
    assert err <= 2e-3, err
