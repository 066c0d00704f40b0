"""Decode steps launched back to back give what the same kernels give with the
device synchronised after every call.

A step is the encode of the new tokens, then decode attention.  In the chained
run no host synchronisation or other kernel separates the launches, so the
kernels' early starts under programmatic dependent launch are in play:
- a decode's first page copies are issued before its dependency wait;
- the length it reads there may still be advancing (a hint).
Lengths start just below page boundaries, so some steps cross into a new
page: then the length the decode reads before its wait may lag the final one.
The decode is deterministic (its split-K partition and merge order depend only
on the final length), so the two runs must agree bit for bit."""
import numpy as np
import pytest

from gpu_helpers import dev, synthetic_latents, torch_mod
from test_gpu_parity import _setup
from workloads import bf16_round

pytestmark = pytest.mark.gpu


def _run(codec, P, start, H, Q, seq_ids, maxp, sync, seed):
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    B = len(start)
    cache = st.LatentCache(codec, batch=B, max_pages_per_seq=maxp, device=dev())
    seqs = np.concatenate([np.full(L, b, np.int32) for b, L in enumerate(start)])
    lat = synthetic_latents(seqs.size, codec.n_eff, seed=seed, decay=0.5, scale=2.0)
    codec.quantize_append(cache, torch.from_numpy(lat).to(dev()), torch.from_numpy(seqs).to(dev()))
    torch.cuda.synchronize()
    ews = torch.zeros(codec.encode_workspace_bytes(H.shape[1]), dtype=torch.uint8, device=dev())
    dws = torch.zeros(codec.decode_workspace_bytes(B, cache.capacity), dtype=torch.uint8, device=dev())
    out = torch.zeros_like(Q)
    stream = torch.cuda.Stream(device=dev())
    torch.cuda.synchronize()
    for i in range(H.shape[0]):
        codec.encode_append(cache, H[i], seq_ids, workspace=ews, stream=stream)
        if sync:
            torch.cuda.synchronize()
        codec.decode_attend(cache, Q[i], out[i], workspace=dws, stream=stream)
        if sync:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    codec.device_status()
    return out.cpu(), cache.pool.cpu(), cache.lengths.cpu()


@pytest.mark.parametrize("name,T", [("llama4x", 1), ("qwen8x", 3), ("llama4x", 20)])
def test_chained_steps_equal_synchronised_steps(name, T):
    """T <= 16 runs the fused encode and its commit kernel; T = 20 runs the
    projection, the append plan and the quantise kernel."""
    torch = torch_mod()
    s = _setup(name, seed=4)
    codec, P = s["codec"], s["P"]
    start = [P - 2, 3 * P - 1]
    B = len(start)
    n_steps = max(6, (P + 8) // T)
    maxp = -(-(max(start) + n_steps * T) // P) + 1
    rng = np.random.default_rng(17 + T)
    H = bf16_round(rng.standard_normal((n_steps, B * T, s["d_model"])).astype(np.float32))
    H = torch.from_numpy(H).to(dev()).to(torch.bfloat16)
    Q = torch.from_numpy((rng.standard_normal((n_steps, B, s["n_q"], s["d_h"])) * 0.6).astype(np.float32)).to(dev())
    seq_ids = torch.from_numpy(np.repeat(np.arange(B, dtype=np.int32), T)).to(dev())
    a = _run(codec, P, start, H, Q, seq_ids, maxp, sync=False, seed=5)
    b = _run(codec, P, start, H, Q, seq_ids, maxp, sync=True, seed=5)
    assert torch.equal(a[2], b[2]) and list(a[2].numpy()) == [L + n_steps * T for L in start]
    assert torch.equal(a[1], b[1]), "packed pages differ between chained and synchronised steps"
    assert torch.equal(a[0], b[0]), "decode outputs differ between chained and synchronised steps"


@pytest.mark.parametrize("lag", [1, 65, 1 << 20, -200])
def test_length_hint_does_not_change_the_result(lag, monkeypatch):
    """The decode reads the length before its dependency wait as a hint and copies
    the pages that are full under it early.  The page partition and summation
    order depend only on the final length, so offsetting the hint (the library's
    SPECTRA_DECODE_HINT_LAG test hook) must give the same bits: a positive lag
    moves page copies after the wait, a negative one makes the kernel copy pages
    beyond the length that it must drain unused."""
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    s = _setup("llama4x", seed=6)
    codec, P = s["codec"], s["P"]
    lengths = [333, 64, 1, 2049]
    B, maxp = len(lengths), 40
    cache = st.LatentCache(codec, batch=B, max_pages_per_seq=maxp, device=dev())
    seqs = np.concatenate([np.full(L, b, np.int32) for b, L in enumerate(lengths)])
    lat = synthetic_latents(seqs.size, codec.n_eff, seed=8, decay=0.5, scale=2.0)
    codec.quantize_append(cache, torch.from_numpy(lat).to(dev()), torch.from_numpy(seqs).to(dev()))
    rng = np.random.default_rng(9)
    q = torch.from_numpy((rng.standard_normal((B, s["n_q"], s["d_h"])) * 0.6).astype(np.float32)).to(dev())
    ref = codec.decode_attend(cache, q)
    codec.device_status()
    monkeypatch.setenv("SPECTRA_DECODE_HINT_LAG", str(lag))
    for _ in range(2):
        got = codec.decode_attend(cache, q)
        codec.device_status()
        assert torch.equal(got, ref)


def test_bounded_wait_gives_up_with_a_timeout_status(monkeypatch):
    """A page copy that never lands (test hook SPECTRA_DECODE_TEST_DROP_PAGE: the
    first CTA skips issuing it) makes that CTA's wait for the page give up after
    the limit (shortened to 2 ms by SPECTRA_DECODE_TEST_WAIT_NS), drain its other
    copies and finish; the call reports SPECTRA_ERR_TIMEOUT through the device
    error word, and the next calls on the same context give the exact result."""
    torch = torch_mod()
    import spectral_transform_coding_b200 as st
    s = _setup("llama4x", seed=6)
    codec = s["codec"]
    lengths = [333, 64]
    cache = st.LatentCache(codec, batch=len(lengths), max_pages_per_seq=8, device=dev())
    seqs = np.concatenate([np.full(L, b, np.int32) for b, L in enumerate(lengths)])
    lat = synthetic_latents(seqs.size, codec.n_eff, seed=12, decay=0.5, scale=2.0)
    codec.quantize_append(cache, torch.from_numpy(lat).to(dev()), torch.from_numpy(seqs).to(dev()))
    rng = np.random.default_rng(13)
    q = torch.from_numpy((rng.standard_normal((len(lengths), s["n_q"], s["d_h"])) * 0.6).astype(np.float32)).to(dev())
    ws = torch.zeros(codec.decode_workspace_bytes(len(lengths), cache.capacity), dtype=torch.uint8, device=dev())
    ref = codec.decode_attend(cache, q, workspace=ws)
    codec.device_status()
    monkeypatch.setenv("SPECTRA_DECODE_TEST_DROP_PAGE", "0")
    monkeypatch.setenv("SPECTRA_DECODE_TEST_WAIT_NS", "2000000")
    codec.decode_attend(cache, q, workspace=ws)
    with pytest.raises(st.SpectraError) as e:
        codec.device_status()
    assert e.value.status == 6  # SPECTRA_ERR_TIMEOUT
    monkeypatch.delenv("SPECTRA_DECODE_TEST_DROP_PAGE")
    monkeypatch.delenv("SPECTRA_DECODE_TEST_WAIT_NS")
    for _ in range(2):  # the same workspace: its arrival counters were left at zero
        got = codec.decode_attend(cache, q, workspace=ws)
        codec.device_status()
        assert torch.equal(got, ref)
