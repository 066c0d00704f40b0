"""ctypes declarations of the libspectra C ABI (include/spectra.h)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.environ.get("SPECTRA_LIB", os.path.join(_HERE, "libspectra.so"))

if not os.path.exists(lib_path):
    raise ImportError(
        f"libspectra.so not found at {lib_path}; build it with "
        "`python spectral_transform_coding_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(lib_path)

SPECTRA_F32, SPECTRA_BF16 = 0, 1
SPECTRA_ALLOC_WATERFILL, SPECTRA_ALLOC_UNIFORM = 0, 1
STATUS_NAMES = {0: "OK", 1: "ERR_INVALID", 2: "ERR_CUDA", 3: "ERR_CAPACITY", 4: "ERR_NUMERIC",
                5: "ERR_UNSUPPORTED", 6: "ERR_TIMEOUT", 7: "ERR_ORDER"}


class SpectraError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


class Config(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("d_head", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("group", ctypes.c_int32),
                ("budget_bits", ctypes.c_int32), ("count_overhead", ctypes.c_int32),
                ("page_tokens", ctypes.c_int32)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("pool", ctypes.c_void_p), ("n_pages", ctypes.c_int64),
                ("page_table", ctypes.c_void_p), ("lengths", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32)]


class CodecInfo(ctypes.Structure):
    _fields_ = [("config", Config), ("n_groups", ctypes.c_int32), ("n_eff", ctypes.c_int32),
                ("page_bytes", ctypes.c_int64), ("bits_per_token", ctypes.c_int64),
                ("max_kept", ctypes.c_int32)]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_P = ctypes.POINTER

_SIGS = {
    "spectra_calibrate": [_P(Config), _i32, _vp, _i64, _vp, _vp, _P(_vp), _vp],
    "spectra_calibrate_ex": [_P(Config), _i32, _vp, _i64, _vp, _vp, _i32, ctypes.c_double, _P(_vp), _vp],
    "spectra_codec_create": [_P(Config), _vp, _vp, _vp, _vp, _P(_vp)],
    "spectra_codec_get_info": [_vp, _P(CodecInfo)],
    "spectra_codec_get_state": [_vp, _vp, _vp, _vp, _vp, _vp],
    "spectra_codec_serialize": [_vp, _vp, _P(_sz)],
    "spectra_codec_deserialize": [_vp, _sz, _P(_vp)],
    "spectra_wo_correction": [_vp, _i32, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp],
    "spectra_encode_workspace_bytes": [_vp, _i64, _P(_sz)],
    "spectra_decode_workspace_bytes": [_vp, _i32, _i64, _P(_sz)],
    "spectra_project": [_vp, _vp, _i64, _vp, _vp],
    "spectra_quantize_append": [_vp, _P(CacheDesc), _vp, _vp, _i64, _vp, _sz, _vp],
    "spectra_encode_append": [_vp, _P(CacheDesc), _vp, _vp, _i64, _vp, _vp, _sz, _vp],
    "spectra_decode_attend": [_vp, _P(CacheDesc), _vp, _vp, _vp, _sz, _vp],
    "spectra_decode_attend_noalloc": [_vp, _P(CacheDesc), _vp, _vp, _vp],
    "spectra_device_status": [_vp, _vp],
    "spectra_reconstruct": [_vp, _P(CacheDesc), _i32, _i64, _i64, _vp, _vp, _vp],
    "spectra_decode_reconstruct_workspace_bytes": [_vp, _i32, _i64, _P(ctypes.c_size_t)],
    "spectra_decode_attend_reconstruct": [_vp, _P(CacheDesc), _vp, ctypes.c_double, _vp, _vp, _sz, _vp],
    "spectra_allocate_widths": [_vp, _i32, _i32, _i32, _i32, _vp, _vp],
    "spectra_allocate_widths_uniform": [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp],
    "spectra_energy_rank": [_vp, _i32, ctypes.c_double, _P(_i32)],
    "spectra_water_fill": [_vp, _i32, ctypes.c_double, _vp, _vp],
    "spectra_sym_eigen": [_vp, _i32, _vp, _vp],
    "spectra_page_layout": [_P(Config), _vp, _P(_i64), _vp],
}

for _name, _args in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int

lib.spectra_codec_destroy.argtypes = [_vp]
lib.spectra_codec_destroy.restype = None
lib.spectra_last_error.argtypes = []
lib.spectra_last_error.restype = ctypes.c_char_p
lib.spectra_abi_version.argtypes = []
lib.spectra_abi_version.restype = ctypes.c_int32

EXPORTED = sorted(list(_SIGS) + ["spectra_codec_destroy", "spectra_last_error", "spectra_abi_version"])


def check(status: int, where: str) -> None:
    if status != 0:
        msg = lib.spectra_last_error() or b""
        raise SpectraError(status, where, msg.decode(errors="replace"))
