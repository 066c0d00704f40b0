"""spectra_decode_attend_noalloc: decode attention for callers that cannot
allocate device memory while they decode (their buffers are planned ahead of
time, or the device allocator belongs to someone else).  Its scratch is a static
device array inside the library instead of a caller workspace.

Checked through the C ABI, two calls in a row: each output must be bit-identical
to spectra_decode_attend's on the same cache and queries (both run the same
kernels, so any difference means a wrong scratch offset or stale scratch from
the previous call), and within the 2e-3 attention bar of the oracle's decode
over its own copy of the pool (which must equal the library's byte for byte).
This file is collected last so that a failure here cannot hide another test's
result, and it does not depend on state left by other tests.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _case(seed, shape):
    import torch

    import spectral_transform_coding_b200 as st
    from gpu_helpers import codec_from, make_cfg, random_factors, synthetic_latents

    d_model, n_q, n_kv, d_h, rank, group, widths, P, lengths = shape
    w = np.array([widths] * n_kv, np.int32).reshape(n_kv, 2, rank // group)
    w, W_down, W_up = random_factors(d_model, n_kv, d_h, rank, group, w, seed=seed)
    codec = codec_from(make_cfg(d_model, n_q, n_kv, d_h, rank, group, 512, True, P), w, W_down, W_up)
    dev = torch.device("cuda:0")
    B = len(lengths)
    maxp = max(1, (max(lengths) + P - 1) // P)
    rng = np.random.default_rng(seed)
    table = torch.from_numpy(rng.permutation(B * maxp).astype(np.int32).reshape(B, maxp))
    cache = st.LatentCache(codec, batch=B, max_pages_per_seq=maxp, device=dev, page_table=table)
    seqs = np.concatenate([np.full(L, b, np.int32) for b, L in enumerate(lengths)])
    lat = synthetic_latents(seqs.size, codec.n_eff, seed=seed + 1, decay=0.5, scale=2.0)
    codec.quantize_append(cache, torch.from_numpy(lat).to(dev), torch.from_numpy(seqs).to(dev))
    q = torch.from_numpy((rng.standard_normal((B, n_q, d_h)) * 0.6).astype(np.float32)).to(dev)
    oracle_inputs = dict(widths=w, W_up=W_up, group=group, P=P, table=table.numpy(), seqs=seqs, lat=lat,
                         lengths=np.array(lengths), n_q=n_q, n_kv=n_kv)
    return codec, cache, q, oracle_inputs


def _oracle_decode(codec, cache, q, o):
    """The oracle's decode over its own pool, built from the same latents."""
    import oracle
    from gpu_helpers import kept_wup, oracle_pool_after

    pool, _, lay = oracle_pool_after({"group": o["group"]}, o["widths"], cache.pool.numel(), codec.page_bytes,
                                     o["table"], np.zeros(len(o["lengths"])), o["seqs"], o["lat"], o["P"])
    assert np.array_equal(cache.pool.cpu().numpy(), pool), "packed cache differs from the oracle's"
    return oracle.decode_reference(pool, codec.page_bytes, lay, o["group"], o["P"], o["table"], o["lengths"],
                                   q.cpu().numpy(), kept_wup(o["W_up"], o["widths"], o["group"]), o["n_q"],
                                   o["n_kv"])


SHAPES = [
    (512, 8, 2, 128, 128, 16, [[4, 2, 2, 2, 2, 2, 1, 1], [4, 3, 2, 2, 2, 1, 1, 1]], 64, [333, 64, 1, 129]),
    (256, 4, 1, 64, 32, 8, [[4, 2, 1, 1], [4, 2, 1, 1]], 64, [1000, 7]),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_noalloc_matches_workspace_decode_twice(shape):
    import torch

    import spectral_transform_coding_b200 as st
    from gpu_helpers import attention_rel_err

    codec, cache, q, o = _case(3, shape)
    ref = codec.decode_attend(cache, q).cpu().numpy()
    codec.device_status()
    ref_oracle = _oracle_decode(codec, cache, q, o)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        d = cache.desc()
        rc = st.lib.spectra_decode_attend_noalloc(codec._h, ctypes.byref(d), q.data_ptr(), out.data_ptr(),
                                                  stream)
        assert rc == 0, st.lib.spectra_last_error()
        codec.device_status()
        got = out.cpu().numpy()
        assert np.array_equal(got, ref), "differs from spectra_decode_attend on the same inputs"
        err = attention_rel_err(got, ref_oracle)
        assert err <= 2e-3, err


def test_noalloc_rejects_scratch_beyond_its_limit():
    import torch

    import spectral_transform_coding_b200 as st

    # 200 sequences x 64 q heads x (2 + 128) floats of split partials > 4 MiB
    shape = (256, 64, 8, 128, 128, 16, [[4, 2, 2, 2, 2, 2, 1, 1], [4, 3, 2, 2, 2, 1, 1, 1]], 64, [1] * 200)
    codec, cache, q, _ = _case(5, shape)
    out = torch.empty_like(q)
    d = cache.desc()
    rc = st.lib.spectra_decode_attend_noalloc(codec._h, ctypes.byref(d), q.data_ptr(), out.data_ptr(),
                                              torch.cuda.current_stream().cuda_stream)
    assert rc == 3  # SPECTRA_ERR_CAPACITY
    assert b"static area" in st.lib.spectra_last_error()
