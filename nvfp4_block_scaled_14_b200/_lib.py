"""ctypes binding of libnvfp4.so: the C-ABI entry points under their own names.

Argument marshalling only; every step of the hot path runs in the library's CUDA kernels.
There is no fallback: if the library cannot be built or loaded, importing the entry points
raises.
"""
import ctypes
import os
import re
import threading

from . import build as _build

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_SHAPE = 2
NVFP4_ERR_ALIGNMENT = 3
NVFP4_ERR_WORKSPACE = 4
NVFP4_ERR_CUDA = 5
NVFP4_ERR_TIMEOUT = 6
NVFP4_ERR_UNSUPPORTED = 7

NVFP4_F32 = 0
NVFP4_BF16 = 1

NVFP4_LINEAR_DEFAULT = 0
NVFP4_LINEAR_RESIDENT_WEIGHTS = 1

NVFP4_OP_QUANTIZE = 0
NVFP4_OP_LINEAR = 1
NVFP4_OP_CALIB_BF16 = 2
NVFP4_OP_CALIB_F32 = 3
NVFP4_OP_LINEAR_DYNAMIC = 4
NVFP4_OP_QUANTIZE_E4M3 = 5
NVFP4_OP_LINEAR_LOWRANK = 6
NVFP4_ACT_IDENTITY = 0
NVFP4_ACT_GELU_TANH = 1

HEADER = os.path.join(os.path.dirname(_build.PKG), "include", "nvfp4.h")

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_int = ctypes.c_int
_u32 = ctypes.c_uint32

NVFP4_SRC_F32 = 0
NVFP4_SRC_BF16 = 1
NVFP4_SRC_E4M3 = 2
NVFP4_MAX_QUANT_JOBS = 8


class QuantJob(ctypes.Structure):
    """nvfp4_quant_job: one tensor of nvfp4_quantize_batch."""
    _fields_ = [("x", ctypes.c_void_p), ("src", ctypes.c_int), ("fp8_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("static_amax", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales_swz", ctypes.c_void_p), ("scales_lin", ctypes.c_void_p),
                ("global_scale", ctypes.c_void_p)]


_SIGNATURES = {
    "nvfp4_status_str": ([_int], ctypes.c_char_p),
    "nvfp4_codes_bytes": ([_i64, _i64], _sz),
    "nvfp4_scales_bytes": ([_i64, _i64, _int], _sz),
    "nvfp4_workspace_bytes": ([_int, _i64, _i64, _i64], _sz),
    "nvfp4_quantize": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "nvfp4_quantize_fp8_src": ([_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
                               _int),
    "nvfp4_quantize_batch": ([ctypes.POINTER(QuantJob), _int, _vp, _sz, _vp], _int),
    "nvfp4_dequantize": ([_vp, _vp, _vp, _i64, _i64, _int, _vp, _vp], _int),
    "nvfp4_linear": ([_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp, _sz, _vp],
                     _int),
    "nvfp4_linear_ex": ([_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp, _sz, _u32,
                         _vp], _int),
    "nvfp4_linear_dynamic": ([_vp, _int, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp, _vp,
                              _sz, _u32, _vp], _int),
    "nvfp4_linear_noalloc": ([_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp],
                             _int),
    "nvfp4_calib_percentile_amax": ([ctypes.POINTER(_vp), _int, _i64, _int, _u32, _u32, _vp,
                                     _vp, _vp, _sz, _vp], _int),
    "nvfp4_linear_nvfp4_out": ([_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp,
                                _vp, _vp, _vp], _int),
    "nvfp4_quantize_e4m3": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "nvfp4_linear_lowrank": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                              _vp, _vp, _sz, _vp], _int),
    "nvfp4_linear_e4m3": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp], _int),
    "nvfp4_selftest_wait_timeout": ([_vp], _int),
    "nvfp4_selftest_grid_exchange": ([_int, _vp, _int, _int, ctypes.c_uint32, ctypes.c_uint32,
                                      _vp, _vp, ctypes.c_size_t, _vp], _int),
    "nvfp4_sync_status": ([_vp], _int),
}

_lib = None
_lock = threading.Lock()


def lib_path() -> str:
    return _build.LIB


def load():
    """Build (if missing or stale) and load libnvfp4.so; raise if that is impossible."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            for name, (args, res) in _SIGNATURES.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = res
            _lib = L
    return _lib


def declared_functions(header: str = HEADER):
    """Names of the functions include/nvfp4.h declares."""
    text = open(header).read()
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


class NVFP4Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = load().nvfp4_status_str(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


def check(status, where="nvfp4"):
    if status != NVFP4_OK:
        raise NVFP4Error(status, where)


def __getattr__(name):
    # nvfp4_* entry points resolve to the loaded library's functions
    if name in _SIGNATURES:
        return getattr(load(), name)
    raise AttributeError(name)
