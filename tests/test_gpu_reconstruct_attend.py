"""GPU parity of the reconstruct-then-attend decode (keys rebuilt from the packed
cache per tile, optional rotary position embedding) against the oracle's
dequantise, lift, rotate and exact softmax attention over its own pool.

Bar: attention within 2e-3 (max over (sequence, q head) of ||diff||_inf /
||ref||_inf), the bar of the latent decode; the packed pools are checked
byte for byte first, so both sides attend over the same codes."""
import numpy as np
import pytest

import oracle
from gpu_helpers import (attention_rel_err, codec_from, dev, kept_wup, make_cfg, oracle_pool_after, oracle_widths,
                         random_factors, synthetic_latents, torch_mod)
from test_gpu_parity import SHAPES, _setup

pytestmark = pytest.mark.gpu


def _cache_with_tokens(s, lengths, seed):
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    codec, P = s["codec"], s["P"]
    B = len(lengths)
    maxp = max(1, -(-max(lengths) // P))
    rng = np.random.default_rng(seed + 7)
    perm = rng.permutation(B * maxp).astype(np.int32).reshape(B, maxp)
    cache = st.LatentCache(codec, batch=B, max_pages_per_seq=maxp, device=dev(), page_table=torch.from_numpy(perm))
    seqs = np.concatenate([np.full(L, b, np.int32) for b, L in enumerate(lengths)])
    pool_ref = np.zeros(cache.pool.numel(), np.uint8)
    lay = oracle.page_layout(oracle_widths(s["widths"]), s["group"], P)
    if seqs.size:
        lat = synthetic_latents(seqs.size, codec.n_eff, seed=seed + 11, decay=0.5, scale=2.0)
        codec.quantize_append(cache, torch.from_numpy(lat).to(dev()), torch.from_numpy(seqs).to(dev()))
        pool_ref, _, lay = oracle_pool_after({"group": s["group"]}, s["widths"], cache.pool.numel(),
                                             codec.page_bytes, perm, np.zeros(B), seqs, lat, P)
    assert np.array_equal(cache.pool.cpu().numpy(), pool_ref), "packed cache differs from the oracle's"
    return cache, perm, pool_ref, lay, rng


def _rt_case(name, lengths, theta, seed=0, q_scale=0.6):
    torch = torch_mod()
    s = _setup(name, seed=seed)
    codec = s["codec"]
    cache, perm, pool_ref, lay, rng = _cache_with_tokens(s, lengths, seed)
    q = (rng.standard_normal((len(lengths), s["n_q"], s["d_h"])) * q_scale).astype(np.float32)
    out = codec.decode_attend_reconstruct(cache, torch.from_numpy(q).to(dev()), rope_theta=theta)
    codec.device_status()
    ref = oracle.decode_reference_rope(pool_ref, codec.page_bytes, lay, s["group"], s["P"], perm, np.array(lengths),
                                       q, kept_wup(s["W_up"], s["widths"], s["group"]), s["n_q"], s["n_kv"], theta)
    got = out.cpu().numpy()
    for b, L in enumerate(lengths):
        if L == 0:
            assert np.all(got[b] == 0)
    live = [b for b, L in enumerate(lengths) if L > 0]
    return attention_rel_err(got[live], ref[live]), (codec, cache, q, got)


@pytest.mark.parametrize("name", list(SHAPES))
def test_rope_decode_parity(name):
    err, _ = _rt_case(name, [333, 64, 1, 129], 10000.0)
    assert err <= 2e-3, err


@pytest.mark.parametrize("name", ["llama4x", "qwen8x", "g8wide"])
def test_unrotated_matches_oracle_and_latent_decode(name):
    """theta = 0: the oracle's plain reconstruct-then-attend, and the latent-space
    decode of the same cache, which computes the same function."""
    torch = torch_mod()
    err, (codec, cache, q, got) = _rt_case(name, [500, 77], 0.0, seed=2)
    assert err <= 2e-3, err
    lat = codec.decode_attend(cache, torch.from_numpy(q).to(dev())).cpu().numpy()
    codec.device_status()
    assert attention_rel_err(got, lat.astype(np.float64)) <= 2e-3


@pytest.mark.parametrize("lengths", [[1], [63], [64], [65], [0, 17], [2049, 3]])
def test_rope_decode_edge_lengths(lengths):
    err, _ = _rt_case("llama4x", lengths, 500000.0, seed=3)
    assert err <= 2e-3, err


def test_rope_decode_long_context_large_positions():
    """Positions up to 12k with a small base (fast-turning pairs): the angle
    reduction must keep the rotation accurate far from position 0."""
    err, _ = _rt_case("llama4x", [12000], 100.0, seed=4)
    assert err <= 2e-3, err


@pytest.mark.parametrize("name", ["toy", "qwen8x"])
def test_rope_decode_peaked_queries(name):
    err, _ = _rt_case(name, [700, 2000], 10000.0, seed=5, q_scale=3.6)
    assert err <= 2e-3, err


def test_rope_decode_bad_page_id_sets_device_error():
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    s = _setup("llama4x", seed=6)
    codec = s["codec"]
    cache = st.LatentCache(codec, batch=1, max_pages_per_seq=3, device=dev())
    lat = synthetic_latents(150, codec.n_eff, seed=2)
    codec.quantize_append(cache, torch.from_numpy(lat).to(dev()), torch.zeros(150, dtype=torch.int32, device=dev()))
    codec.device_status()
    cache.page_table[0, 1] = cache.n_pages  # one past the pool
    q = torch.zeros((1, s["n_q"], s["d_h"]), dtype=torch.float32, device=dev())
    codec.decode_attend_reconstruct(cache, q, rope_theta=10000.0)
    with pytest.raises(st.SpectraError) as e:
        codec.device_status()
    assert e.value.status == 1


def test_rope_decode_rejects_unsupported_shapes_and_theta():
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    # d_head 256: above what the kernel handles (the codec itself is valid)
    widths, W_down, W_up = random_factors(256, 1, 256, 64, 16, [[[4, 2, 1, 1], [4, 2, 1, 1]]], seed=1)
    codec = codec_from(make_cfg(256, 2, 1, 256, 64, 16, 128, False, 64), widths, W_down, W_up)
    cache = st.LatentCache(codec, batch=1, max_pages_per_seq=1, device=dev())
    q = torch.zeros((1, 2, 256), dtype=torch.float32, device=dev())
    with pytest.raises(st.SpectraError) as e:
        codec.decode_attend_reconstruct(cache, q, rope_theta=10000.0)
    assert e.value.status == 5
    s = _setup("toy")
    cache = st.LatentCache(s["codec"], batch=1, max_pages_per_seq=1, device=dev())
    q = torch.zeros((1, s["n_q"], s["d_h"]), dtype=torch.float32, device=dev())
    for bad in (-1.0, 0.5, float("inf"), float("nan")):
        with pytest.raises(st.SpectraError) as e:
            s["codec"].decode_attend_reconstruct(cache, q, rope_theta=bad)
        assert e.value.status == 1
