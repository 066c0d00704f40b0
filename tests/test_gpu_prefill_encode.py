"""The prefill encode (T >= 64 tokens, no latents requested): the tcgen05
projection GEMM with the quantiser and page writer in its epilogue.

Its accumulators come from the same MMA sequence as the projection GEMM's (same
tile shape and k order), so the pages it writes must equal, byte for byte, those
of the projection followed by the separate quantise kernel on the same H; that
quantise kernel is itself bit-exact against the oracle on the same latents
(test_gpu_parity), and the projection within 1e-3 of the oracle's H W_down
(checked here too).  Appends start mid-block and mid-page, span several
sequences and a ragged last 128-row tile, so both the whole-block stores and the
atomic merges of partial blocks run."""
import numpy as np
import pytest

from gpu_helpers import dev, torch_mod
from test_gpu_fullsize import LLAMA4X, _check_latents, _codec
from test_gpu_parity import _setup
from workloads import bf16_round

pytestmark = pytest.mark.gpu


def _two_routes(codec, d_model, P, counts, start, seed, maxp=None):
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    B = len(counts)
    seqs = np.concatenate([np.full(n, b, np.int32) for b, n in enumerate(counts)])
    T = seqs.size
    maxp = maxp or max(-(-(s + n) // P) for s, n in zip(start, counts)) + 1
    rng = np.random.default_rng(seed)
    table = rng.permutation(B * maxp).astype(np.int32).reshape(B, maxp)
    H = bf16_round(rng.standard_normal((T, d_model)).astype(np.float32))
    Hd = torch.from_numpy(H).to(dev()).to(torch.bfloat16)
    sd = torch.from_numpy(seqs).to(dev())
    caches = []
    for _ in range(2):
        c = st.LatentCache(codec, batch=B, max_pages_per_seq=maxp, device=dev(), page_table=torch.from_numpy(table))
        c.lengths.copy_(torch.from_numpy(np.array(start, np.int32)))
        caches.append(c)
    codec.encode_append(caches[0], Hd, sd)  # fused: no latents requested
    codec.device_status()
    lat = codec.project(Hd)
    codec.quantize_append(caches[1], lat, sd)
    codec.device_status()
    return H, lat.cpu().numpy(), caches, np.array(start) + np.array(counts)


@pytest.mark.parametrize("name", ["llama4x", "allwidths", "g8wide", "zeroside", "qwen8x"])
@pytest.mark.parametrize("counts,start", [([64], [0]), ([300, 1, 700], [5, 64, 17]), ([129, 3000], [0, 33])])
def test_prefill_pages_equal_projection_then_quantise(name, counts, start):
    s = _setup(name, seed=7)
    H, lat, (c1, c2), want = _two_routes(s["codec"], s["d_model"], s["P"], counts, start, seed=8)
    _check_latents(lat, H.astype(np.float64) @ s["W_down"].astype(np.float64), s["widths"])
    a, b = c1.pool.cpu().numpy(), c2.pool.cpu().numpy()
    bad = np.nonzero(a != b)[0]
    assert bad.size == 0, f"{bad.size} bytes differ, first at {bad[:8]}"
    np.testing.assert_array_equal(c1.lengths.cpu().numpy(), want)
    np.testing.assert_array_equal(c2.lengths.cpu().numpy(), want)


def test_prefill_full_width_llama_layer():
    """d_model 4096 (64 k-blocks), 8 KV heads at 4x (N_eff 2048, 8 column tiles),
    8,221 tokens over three sequences: more tiles than SMs, so the persistent
    CTAs reuse both TMEM accumulators many times."""
    codec, widths, W_down, _ = _codec(4096, 32, 8, LLAMA4X, LLAMA4X, seed=15)
    counts, start = [4096, 29, 4096], [0, 7, 100]
    H, lat, (c1, c2), want = _two_routes(codec, 4096, 64, counts, start, seed=16)
    rows = np.r_[0:16, 4090:4140, 8200:8221]
    _check_latents(lat[rows], H[rows].astype(np.float64) @ W_down.astype(np.float64), widths)
    assert np.array_equal(c1.pool.cpu().numpy(), c2.pool.cpu().numpy())
    np.testing.assert_array_equal(c1.lengths.cpu().numpy(), want)


def test_prefill_rejection_writes_nothing():
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    s = _setup("llama4x", seed=5)
    codec, P = s["codec"], s["P"]
    cache = st.LatentCache(codec, batch=2, max_pages_per_seq=2, device=dev())
    cache.lengths.copy_(torch.tensor([P, 0], dtype=torch.int32))
    H = torch.from_numpy(bf16_round(np.ones((100, s["d_model"]), np.float32))).to(dev()).to(torch.bfloat16)
    before = cache.pool.clone()
    # 100 tokens for sequence 0 with P free slots: capacity
    codec.encode_append(cache, H, torch.zeros(100, dtype=torch.int32, device=dev()))
    with pytest.raises(st.SpectraError) as e:
        codec.device_status()
    assert e.value.status == 3
    assert torch.equal(cache.pool, before)
    assert cache.lengths.cpu().tolist() == [P, 0]
