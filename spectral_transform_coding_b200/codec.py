"""Thin torch-facing wrappers over the libspectra C ABI (argument marshalling only)."""
from __future__ import annotations

import ctypes

import numpy as np

from ._lib import SPECTRA_BF16, SPECTRA_F32, CacheDesc, CodecInfo, Config, check, lib


def _torch():
    import torch
    return torch


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return SPECTRA_BF16
    if t.dtype == torch.float32:
        return SPECTRA_F32
    raise TypeError("inputs must be bfloat16 or float32")


def make_config(d_model, n_q_heads, n_kv_heads, d_head, rank, group, budget_bits,
                count_overhead, page_tokens) -> Config:
    return Config(int(d_model), int(n_q_heads), int(n_kv_heads), int(d_head), int(rank),
                  int(group), int(budget_bits), int(bool(count_overhead)), int(page_tokens))


class Codec:
    """Owner of one libspectra codec handle (one attention layer)."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        info = CodecInfo()
        check(lib.spectra_codec_get_info(self._h, ctypes.byref(info)), "spectra_codec_get_info")
        self.cfg = info.config
        self.n_groups = info.n_groups
        self.n_eff = info.n_eff
        self.page_bytes = info.page_bytes
        self.bits_per_token = info.bits_per_token
        self.max_kept = info.max_kept

    # -- construction ------------------------------------------------------
    @classmethod
    def calibrate(cls, cfg: Config, H, W_K, W_V, stream=None, allocation: str = "waterfill",
                  energy_threshold: float = 0.0) -> "Codec":
        """allocation: "waterfill" or "uniform"; energy_threshold: 0 (off) or in (0, 1]."""
        dt = _dtype_code(H)
        if _dtype_code(W_K) != dt or _dtype_code(W_V) != dt:
            raise TypeError("H, W_K, W_V must share one dtype")
        modes = {"waterfill": 0, "uniform": 1}
        if allocation not in modes:
            raise ValueError("allocation must be 'waterfill' or 'uniform'")
        h = ctypes.c_void_p()
        check(lib.spectra_calibrate_ex(ctypes.byref(cfg), dt, _ptr(H), H.shape[0], _ptr(W_K), _ptr(W_V),
                                       modes[allocation], float(energy_threshold), ctypes.byref(h),
                                       _stream(stream)), "spectra_calibrate_ex")
        return cls(h)

    @classmethod
    def from_factors(cls, cfg: Config, widths, W_down, W_up, sigma2=None) -> "Codec":
        widths = np.ascontiguousarray(widths, dtype=np.int32)
        W_down = np.ascontiguousarray(W_down, dtype=np.float32)
        W_up = np.ascontiguousarray(W_up, dtype=np.float32)
        s2 = None if sigma2 is None else np.ascontiguousarray(sigma2, dtype=np.float64)
        h = ctypes.c_void_p()
        check(lib.spectra_codec_create(ctypes.byref(cfg), widths.ctypes.data, W_down.ctypes.data,
                                       W_up.ctypes.data, None if s2 is None else s2.ctypes.data,
                                       ctypes.byref(h)), "spectra_codec_create")
        return cls(h)

    @classmethod
    def deserialize(cls, blob: bytes) -> "Codec":
        buf = ctypes.create_string_buffer(blob, len(blob))
        h = ctypes.c_void_p()
        check(lib.spectra_codec_deserialize(buf, len(blob), ctypes.byref(h)), "spectra_codec_deserialize")
        return cls(h)

    def close(self):
        if self._h:
            lib.spectra_codec_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- state -------------------------------------------------------------
    def state(self) -> dict:
        c = self.cfg
        widths = np.zeros((c.n_kv_heads, 2, self.n_groups), np.int32)
        sigma2 = np.zeros((c.n_kv_heads, 2, c.rank), np.float64)
        theta = np.zeros((c.n_kv_heads, 2), np.float64)
        W_down = np.zeros((c.d_model, max(self.n_eff, 1)), np.float32)
        W_up = np.zeros((c.n_kv_heads, 2, c.rank, c.d_head), np.float32)
        check(lib.spectra_codec_get_state(self._h, widths.ctypes.data, sigma2.ctypes.data,
                                          theta.ctypes.data, W_down.ctypes.data, W_up.ctypes.data),
              "spectra_codec_get_state")
        return dict(widths=widths, sigma2=sigma2, theta=theta, W_down=W_down[:, : self.n_eff], W_up=W_up)

    def serialize(self) -> bytes:
        n = ctypes.c_size_t(0)
        check(lib.spectra_codec_serialize(self._h, None, ctypes.byref(n)), "spectra_codec_serialize")
        buf = ctypes.create_string_buffer(n.value)
        check(lib.spectra_codec_serialize(self._h, buf, ctypes.byref(n)), "spectra_codec_serialize")
        return buf.raw[: n.value]

    def encode_workspace_bytes(self, T: int) -> int:
        n = ctypes.c_size_t(0)
        check(lib.spectra_encode_workspace_bytes(self._h, int(T), ctypes.byref(n)), "encode_workspace_bytes")
        return n.value

    def decode_workspace_bytes(self, batch: int, max_len: int) -> int:
        n = ctypes.c_size_t(0)
        check(lib.spectra_decode_workspace_bytes(self._h, int(batch), int(max_len), ctypes.byref(n)),
              "decode_workspace_bytes")
        return n.value

    def decode_reconstruct_workspace_bytes(self, batch: int, max_len: int) -> int:
        n = ctypes.c_size_t(0)
        check(lib.spectra_decode_reconstruct_workspace_bytes(self._h, int(batch), int(max_len), ctypes.byref(n)),
              "decode_reconstruct_workspace_bytes")
        return n.value

    def _workspace(self, nbytes, device):
        torch = _torch()
        return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)

    # -- hot path ----------------------------------------------------------
    def project(self, H, out=None, stream=None):
        torch = _torch()
        if out is None:
            out = torch.empty((H.shape[0], self.n_eff), dtype=torch.float32, device=H.device)
        check(lib.spectra_project(self._h, _ptr(H), H.shape[0], _ptr(out), _stream(stream)), "spectra_project")
        return out

    def quantize_append(self, cache: "LatentCache", latents, seq_ids, workspace=None, stream=None):
        T = latents.shape[0]
        ws = workspace if workspace is not None else self._workspace(self.encode_workspace_bytes(T), latents.device)
        d = cache.desc()
        check(lib.spectra_quantize_append(self._h, ctypes.byref(d), _ptr(latents), _ptr(seq_ids), T,
                                          _ptr(ws), ws.numel(), _stream(stream)), "spectra_quantize_append")

    def encode_append(self, cache: "LatentCache", H, seq_ids, latents_out=None, workspace=None, stream=None):
        T = H.shape[0]
        ws = workspace if workspace is not None else self._workspace(self.encode_workspace_bytes(T), H.device)
        d = cache.desc()
        check(lib.spectra_encode_append(self._h, ctypes.byref(d), _ptr(H), _ptr(seq_ids), T,
                                        _ptr(latents_out), _ptr(ws), ws.numel(), _stream(stream)),
              "spectra_encode_append")
        return latents_out

    def decode_attend(self, cache: "LatentCache", q, out=None, workspace=None, stream=None):
        torch = _torch()
        if out is None:
            out = torch.empty_like(q)
        ws = workspace if workspace is not None else self._workspace(
            self.decode_workspace_bytes(cache.batch, cache.capacity), q.device)
        d = cache.desc()
        check(lib.spectra_decode_attend(self._h, ctypes.byref(d), _ptr(q), _ptr(out), _ptr(ws), ws.numel(),
                                        _stream(stream)), "spectra_decode_attend")
        return out

    def decode_attend_reconstruct(self, cache: "LatentCache", q, rope_theta: float = 0.0, out=None,
                                  workspace=None, stream=None):
        """Decode attention over keys rebuilt from the cache, optionally with rotary
        position embedding (keys at positions 0..len-1, the query at len-1)."""
        torch = _torch()
        if out is None:
            out = torch.empty_like(q)
        ws = workspace if workspace is not None else self._workspace(
            self.decode_reconstruct_workspace_bytes(cache.batch, cache.capacity), q.device)
        d = cache.desc()
        check(lib.spectra_decode_attend_reconstruct(self._h, ctypes.byref(d), _ptr(q), float(rope_theta), _ptr(out),
                                                    _ptr(ws), ws.numel(), _stream(stream)),
              "spectra_decode_attend_reconstruct")
        return out

    def reconstruct(self, cache: "LatentCache", seq: int, t0: int, n: int, stream=None):
        """Keys and values [n][n_kv][d_head] (fp32) of tokens [t0, t0+n) of sequence seq."""
        torch = _torch()
        c = self.cfg
        K = torch.empty((n, c.n_kv_heads, c.d_head), dtype=torch.float32, device=cache.pool.device)
        V = torch.empty_like(K)
        d = cache.desc()
        check(lib.spectra_reconstruct(self._h, ctypes.byref(d), int(seq), int(t0), int(n), _ptr(K), _ptr(V),
                                      _stream(stream)), "spectra_reconstruct")
        return K, V

    def device_status(self, stream=None):
        check(lib.spectra_device_status(self._h, _stream(stream)), "spectra_device_status")

    def wo_correction(self, H, W_Q, W_K, W_V, W_O, stream=None):
        torch = _torch()
        out = torch.empty((W_O.shape[0], W_O.shape[1]), dtype=torch.float32, device=W_O.device)
        check(lib.spectra_wo_correction(self._h, _dtype_code(H), _ptr(H), H.shape[0], _ptr(W_Q), _ptr(W_K),
                                        _ptr(W_V), _ptr(W_O), _ptr(out), _stream(stream)),
              "spectra_wo_correction")
        return out


class LatentCache:
    """Caller-owned paged cache memory (device tensors) described to the library."""

    def __init__(self, codec: Codec, batch: int, max_pages_per_seq: int, n_pages: int | None = None,
                 device="cuda", page_table=None, zero=True):
        torch = _torch()
        self.codec = codec
        self.batch = int(batch)
        self.max_pages = int(max_pages_per_seq)
        self.P = codec.cfg.page_tokens
        self.capacity = self.max_pages * self.P
        self.n_pages = int(n_pages if n_pages is not None else batch * max_pages_per_seq)
        alloc = torch.zeros if zero else torch.empty
        self.pool = alloc((self.n_pages * codec.page_bytes,), dtype=torch.uint8, device=device)
        if page_table is None:
            page_table = torch.arange(self.batch * self.max_pages, dtype=torch.int32, device=device
                                      ).reshape(self.batch, self.max_pages) % self.n_pages
        self.page_table = page_table.to(device=device, dtype=torch.int32).contiguous()
        self.lengths = torch.zeros(self.batch, dtype=torch.int32, device=device)

    def desc(self) -> CacheDesc:
        return CacheDesc(self.pool.data_ptr(), self.n_pages, self.page_table.data_ptr(),
                         self.lengths.data_ptr(), self.batch, self.max_pages)
