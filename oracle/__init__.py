"""CPU oracle for the NVFP4 quantized linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package. The product path (``nvfp4_block_scaled_14_b200``) never imports it and shares
no code with it. The arithmetic lives in ``nvfp4_oracle.c`` (plain scalar C); this module only
marshals numpy arrays into it.

Sources of each step (see the header of nvfp4_oracle.c for the full list):
  * "Qwen-Image NVFP4 on a 16 GB Ada GPU", "What NVFP4 is and how it differs from NF4" and
    the figure "First NVFP4 block, as stored in the file" -- the format and decode equation.
  * "Qwen-Rapid-AIO FP8 -> NVFP4", "1. Double Quantization" -- FP8 upcast, then NVFP4.
  * "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details" -- dynamic per-tensor amax.
  * "Qwen-Rapid-AIO FP8 -> NVFP4", "Recommended Model" -- p99.9 static input scales.
  * "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details" / "Layer breakdown" -- FP8
    E4M3 tensorwise round-to-nearest layers (quantize_e4m3, gemm_e4m3).
  * "Qwen Image 2.1: INT4 + FP4", "What I quantized" -- FP4 layers with BF16 rank-128
    branches (lowrank_down, linear_lowrank).
"""
import ctypes
import os

import numpy as np

from . import build_oracle

_lib = None

F32, BF16, E4M3 = 0, 1, 2

_u8p = ctypes.POINTER(ctypes.c_uint8)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        L.ora_e2m1_decode.argtypes = [ctypes.c_int]
        L.ora_e2m1_decode.restype = ctypes.c_double
        L.ora_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.ora_e4m3_decode.restype = ctypes.c_double
        L.ora_e2m1_encode.argtypes = [ctypes.c_float]
        L.ora_e2m1_encode.restype = ctypes.c_int
        L.ora_e4m3_encode_nonneg.argtypes = [ctypes.c_float]
        L.ora_e4m3_encode_nonneg.restype = ctypes.c_uint8
        L.ora_swizzled_offset.argtypes = [_i64, _i64, _i64]
        L.ora_swizzled_offset.restype = _i64
        L.ora_swizzled_bytes.argtypes = [_i64, _i64]
        L.ora_swizzled_bytes.restype = _i64
        L.ora_quantize.argtypes = [_vp, ctypes.c_int, _f32p, _i64, _i64, _f32p, _u8p, _u8p,
                                   _u8p, _f32p]
        L.ora_quantize.restype = ctypes.c_int
        L.ora_dequantize_f32.argtypes = [_u8p, _u8p, ctypes.c_float, _i64, _i64, _f32p]
        L.ora_dequantize_bf16.argtypes = [_u8p, _u8p, ctypes.c_float, _i64, _i64,
                                          ctypes.POINTER(ctypes.c_uint16)]
        L.ora_gemm_f64.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p, ctypes.c_float,
                                   _i64, _i64, _i64, _f64p]
        L.ora_gemm_f64_sampled.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p,
                                           ctypes.c_float, _i64, _i64p, _i64p, _i64, _f64p]
        L.ora_percentile_abs.argtypes = [ctypes.POINTER(_f32p), _i64p, ctypes.c_int,
                                         ctypes.c_uint32, ctypes.c_uint32, _f32p, _f32p]
        L.ora_percentile_abs.restype = ctypes.c_int
        L.ora_e2m1_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.ora_e4m3_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.ora_amax.argtypes = [_f32p, _i64]
        L.ora_amax.restype = ctypes.c_float
        L.ora_gelu_tanh_f64.argtypes = [ctypes.c_double]
        L.ora_gelu_tanh_f64.restype = ctypes.c_double
        L.ora_linear_act_f64_sampled.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p,
                                                 ctypes.c_float, _i64, ctypes.c_int, _i64p,
                                                 _i64p, _i64, _f64p]
        L.ora_act_f64_array.argtypes = [_f64p, _i64, ctypes.c_int, _f64p]
        L.ora_linear_quantize_out.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p,
                                              ctypes.c_float, _i64, _i64, _i64, ctypes.c_float,
                                              ctypes.c_int, _u8p, _u8p, _u8p, _f32p]
        L.ora_linear_quantize_out.restype = ctypes.c_int
        L.ora_quantize_e4m3.argtypes = [_vp, ctypes.c_int, _i64, _f32p, _u8p, _f32p]
        L.ora_quantize_e4m3.restype = ctypes.c_int
        _u16p = ctypes.POINTER(ctypes.c_uint16)
        L.ora_f64_to_bf16.argtypes = [ctypes.c_double]
        L.ora_f64_to_bf16.restype = ctypes.c_uint16
        L.ora_lowrank_down_bf16.argtypes = [_u16p, _u16p, _i64, _i64, _i64, _u16p]
        L.ora_linear_lowrank_f64.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p,
                                             ctypes.c_float, _u16p, _u16p, _u16p, _i64, _i64,
                                             _i64, _i64, _f64p]
        L.ora_linear_lowrank_f64.restype = ctypes.c_int
        L.ora_linear_lowrank_f64_sampled.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p,
                                                     ctypes.c_float, _u16p, _u16p, _u16p, _i64,
                                                     _i64, _i64p, _i64p, _i64, _f64p]
        L.ora_linear_lowrank_f64_sampled.restype = ctypes.c_int
        L.ora_gemm_e4m3_f64.argtypes = [_u8p, ctypes.c_float, _u8p, ctypes.c_float, _i64, _i64,
                                        _i64, _f64p]
        L.ora_gemm_e4m3_f64_sampled.argtypes = [_u8p, ctypes.c_float, _u8p, ctypes.c_float, _i64,
                                                _i64p, _i64p, _i64, _f64p]
        _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


# ---- scalar codecs ---------------------------------------------------------------------

def e2m1_decode(code: int) -> float:
    return lib().ora_e2m1_decode(int(code))


def e4m3_decode(b: int) -> float:
    return lib().ora_e4m3_decode(int(b))


def e2m1_encode(y: float) -> int:
    return lib().ora_e2m1_encode(float(np.float32(y)))


def e4m3_encode(v: float) -> int:
    return lib().ora_e4m3_encode_nonneg(float(np.float32(v)))


def e2m1_encode_array(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float32).ravel()
    out = np.zeros(y.size, np.uint8)
    lib().ora_e2m1_encode_array(_p(y, _f32p), y.size, _p(out, _u8p))
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32).ravel()
    out = np.zeros(v.size, np.uint8)
    lib().ora_e4m3_encode_array(_p(v, _f32p), v.size, _p(out, _u8p))
    return out


def swizzled_offset(row: int, block: int, nblocks: int) -> int:
    return lib().ora_swizzled_offset(row, block, nblocks)


def swizzled_bytes(rows: int, cols: int) -> int:
    return lib().ora_swizzled_bytes(rows, cols)


# ---- array ops -------------------------------------------------------------------------

class Quantized:
    """codes [rows, cols/2] u8, scales_lin [rows, cols/16] u8, scales_swz (flat u8), sg f32."""

    def __init__(self, codes, scales_lin, scales_swz, sg, rows, cols):
        self.codes, self.scales_lin, self.scales_swz = codes, scales_lin, scales_swz
        self.sg, self.rows, self.cols = sg, rows, cols


def _src_dtype(x):
    if x.dtype == np.float32:
        return F32
    if x.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    if x.dtype == np.uint8:  # E4M3 bit patterns
        return E4M3
    raise TypeError(f"unsupported source dtype {x.dtype}")


def quantize(x: np.ndarray, amax=None, fp8_scale=None) -> Quantized:
    """x: float32, or uint16 (bf16 bits), or uint8 (E4M3 bits, times fp8_scale or 1.0)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    lin = np.zeros((rows, cols // 16), np.uint8)
    swz = np.zeros(max(swizzled_bytes(rows, cols), 1), np.uint8)
    sg = np.zeros(1, np.float32)
    am = None if amax is None else np.array([amax], np.float32)
    s8 = None if fp8_scale is None else np.array([fp8_scale], np.float32)
    rc = lib().ora_quantize(x.ctypes.data_as(_vp), _src_dtype(x),
                            None if s8 is None else _p(s8, _f32p), rows, cols,
                            None if am is None else _p(am, _f32p),
                            _p(codes, _u8p), _p(lin, _u8p), _p(swz, _u8p), _p(sg, _f32p))
    if rc != 0:
        raise ValueError(f"oracle quantize failed ({rc}); cols must be a multiple of 16")
    return Quantized(codes, lin, swz, float(sg[0]), rows, cols)


def dequantize(q: Quantized, out_dtype="f32") -> np.ndarray:
    codes = np.ascontiguousarray(q.codes)
    lin = np.ascontiguousarray(q.scales_lin)
    if out_dtype == "f32":
        out = np.zeros((q.rows, q.cols), np.float32)
        lib().ora_dequantize_f32(_p(codes, _u8p), _p(lin, _u8p), q.sg, q.rows, q.cols,
                                 _p(out, _f32p))
    else:
        out = np.zeros((q.rows, q.cols), np.uint16)
        lib().ora_dequantize_bf16(_p(codes, _u8p), _p(lin, _u8p), q.sg, q.rows, q.cols,
                                  out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)))
    return out


def gemm(a: Quantized, w: Quantized) -> np.ndarray:
    """Y = dequant(A) . dequant(W)^T in fp64, [M, N]."""
    assert a.cols == w.cols
    M, N, K = a.rows, w.rows, a.cols
    out = np.zeros((M, N), np.float64)
    lib().ora_gemm_f64(_p(a.codes, _u8p), _p(a.scales_lin, _u8p), a.sg,
                       _p(w.codes, _u8p), _p(w.scales_lin, _u8p), w.sg, M, N, K, _p(out, _f64p))
    return out


def gemm_sampled(a: Quantized, w: Quantized, ms, ns) -> np.ndarray:
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    out = np.zeros(len(ms), np.float64)
    lib().ora_gemm_f64_sampled(_p(a.codes, _u8p), _p(a.scales_lin, _u8p), a.sg,
                               _p(w.codes, _u8p), _p(w.scales_lin, _u8p), w.sg, a.cols,
                               _p(ms, _i64p), _p(ns, _i64p), len(ms), _p(out, _f64p))
    return out


def percentile_abs(arrays, num=999, den=1000):
    """Nearest-rank percentile of |x| over the union of float32 arrays, and the max."""
    arrs = [np.ascontiguousarray(a, np.float32).ravel() for a in arrays]
    ptrs = (_f32p * len(arrs))(*[_p(a, _f32p) for a in arrs])
    lens = np.array([a.size for a in arrs], np.int64)
    pct = np.zeros(1, np.float32)
    mx = np.zeros(1, np.float32)
    rc = lib().ora_percentile_abs(ptrs, _p(lens, _i64p), len(arrs), num, den, _p(pct, _f32p),
                                  _p(mx, _f32p))
    if rc != 0:
        raise ValueError("oracle percentile: empty input or bad ratio")
    return float(pct[0]), float(mx[0])


def source_to_f32(x: np.ndarray, fp8_scale=None) -> np.ndarray:
    """The oracle's own upcast of a bf16 (uint16 bits) / E4M3 (uint8 bits) array to fp32."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x.copy()
    f = np.zeros(x.shape, np.float32)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).reshape(x.shape)
    L = lib()
    lut = np.array([L.ora_e4m3_decode(b) for b in range(256)], np.float32)
    f = lut[x]
    s8 = np.float32(1.0 if fp8_scale is None else fp8_scale)
    return (f * s8).astype(np.float32)


# ---- linear layer with an NVFP4 output (producer epilogue) -------------------------------
ACT_NONE, ACT_GELU_TANH = 0, 1


def gelu_tanh(y: float) -> float:
    return lib().ora_gelu_tanh_f64(float(y))


def linear_act_sampled(a: Quantized, w: Quantized, act, ms, ns) -> np.ndarray:
    """act(sgA sgW acc) in fp64 at (ms[i], ns[i]): the exact value the fused layer encodes."""
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    out = np.zeros(len(ms), np.float64)
    lib().ora_linear_act_f64_sampled(_p(a.codes, _u8p), _p(a.scales_lin, _u8p), a.sg,
                                     _p(w.codes, _u8p), _p(w.scales_lin, _u8p), w.sg, a.cols,
                                     act, _p(ms, _i64p), _p(ns, _i64p), len(ms), _p(out, _f64p))
    return out


def act_array(y: np.ndarray, act) -> np.ndarray:
    """act applied in fp64 to every value of y (e.g. the exact product from gemm)."""
    y = np.ascontiguousarray(y, np.float64)
    out = np.zeros(y.shape, np.float64)
    lib().ora_act_f64_array(_p(y, _f64p), y.size, act, _p(out, _f64p))
    return out


def linear_quantize_out(a: Quantized, w: Quantized, static_amax, act=ACT_NONE) -> Quantized:
    """NVFP4 (static amax) of act(RN32(RN32(acc) * RN32(sgA sgW))), [a.rows x w.rows]."""
    assert a.cols == w.cols
    M, N, K = a.rows, w.rows, a.cols
    codes = np.zeros((M, N // 2), np.uint8)
    lin = np.zeros((M, N // 16), np.uint8)
    swz = np.zeros(max(swizzled_bytes(M, N), 1), np.uint8)
    sg = np.zeros(1, np.float32)
    rc = lib().ora_linear_quantize_out(_p(a.codes, _u8p), _p(a.scales_lin, _u8p), a.sg,
                                       _p(w.codes, _u8p), _p(w.scales_lin, _u8p), w.sg, M, N, K,
                                       float(static_amax), act, _p(codes, _u8p), _p(lin, _u8p),
                                       _p(swz, _u8p), _p(sg, _f32p))
    if rc != 0:
        raise ValueError(f"oracle linear_quantize_out failed ({rc})")
    return Quantized(codes, lin, swz, float(sg[0]), M, N)


# ---- FP8 E4M3 tensorwise layers ----------------------------------------------------------
def quantize_e4m3(x: np.ndarray, amax=None):
    """x: float32 or uint16 (bf16 bits), any shape -> (codes uint8 of x's shape, scale s)."""
    x = np.ascontiguousarray(x)
    dt = _src_dtype(x)
    if dt == E4M3:
        raise TypeError("E4M3 sources are already FP8")
    codes = np.zeros(x.shape, np.uint8)
    s = np.zeros(1, np.float32)
    am = None if amax is None else np.array([amax], np.float32)
    rc = lib().ora_quantize_e4m3(x.ctypes.data_as(_vp), dt, x.size,
                                 None if am is None else _p(am, _f32p), _p(codes, _u8p),
                                 _p(s, _f32p))
    if rc != 0:
        raise ValueError(f"oracle quantize_e4m3 failed ({rc})")
    return codes, float(s[0])


def gemm_e4m3(a_codes, sa, w_codes, sw) -> np.ndarray:
    """Y = sA * sW * eA . eW^T in fp64 from E4M3 codes A [M, K], W [N, K]."""
    a = np.ascontiguousarray(a_codes, np.uint8)
    w = np.ascontiguousarray(w_codes, np.uint8)
    (M, K), (N, K2) = a.shape, w.shape
    assert K == K2
    out = np.zeros((M, N), np.float64)
    lib().ora_gemm_e4m3_f64(_p(a, _u8p), sa, _p(w, _u8p), sw, M, N, K, _p(out, _f64p))
    return out


def gemm_e4m3_sampled(a_codes, sa, w_codes, sw, ms, ns) -> np.ndarray:
    a = np.ascontiguousarray(a_codes, np.uint8)
    w = np.ascontiguousarray(w_codes, np.uint8)
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    out = np.zeros(len(ms), np.float64)
    lib().ora_gemm_e4m3_f64_sampled(_p(a, _u8p), sa, _p(w, _u8p), sw, a.shape[1], _p(ms, _i64p),
                                    _p(ns, _i64p), len(ms), _p(out, _f64p))
    return out


# ---- FP4 linear layer with a BF16 low-rank branch ------------------------------------------
_u16 = ctypes.c_uint16


def f64_to_bf16(v: float) -> int:
    """Nearest bf16 (ties to even) of a double, in one rounding, as bits."""
    return int(lib().ora_f64_to_bf16(float(v)))


def _bits16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 operands are passed as uint16 bit patterns"
    return a


def lowrank_down(x_bits, d_bits) -> np.ndarray:
    """T = bf16(x . D^T) as uint16 bits [M x r]; x [M x K], D [r x K] bf16 bits."""
    x, d = _bits16(x_bits), _bits16(d_bits)
    (M, K), (r, K2) = x.shape, d.shape
    assert K == K2
    t = np.zeros((M, r), np.uint16)
    u16p = ctypes.POINTER(_u16)
    lib().ora_lowrank_down_bf16(_p(x, u16p), _p(d, u16p), M, K, r, _p(t, u16p))
    return t


def linear_lowrank(a: Quantized, w: Quantized, x_bits, d_bits, u_bits) -> np.ndarray:
    """Y = dequant(A) . dequant(W)^T + bf16(x . D^T) . U^T in fp64, [M x N]."""
    x, d, u = _bits16(x_bits), _bits16(d_bits), _bits16(u_bits)
    M, N, K = a.rows, w.rows, a.cols
    r = d.shape[0]
    assert a.cols == w.cols == x.shape[1] == d.shape[1] and x.shape[0] == M
    assert u.shape == (N, r)
    out = np.zeros((M, N), np.float64)
    u16p = ctypes.POINTER(_u16)
    rc = lib().ora_linear_lowrank_f64(_p(a.codes, _u8p), _p(a.scales_lin, _u8p), a.sg,
                                      _p(w.codes, _u8p), _p(w.scales_lin, _u8p), w.sg,
                                      _p(x, u16p), _p(d, u16p), _p(u, u16p), M, N, K, r,
                                      _p(out, _f64p))
    if rc != 0:
        raise MemoryError("oracle linear_lowrank")
    return out


def linear_lowrank_sampled(a: Quantized, w: Quantized, x_bits, d_bits, u_bits, ms, ns):
    x, d, u = _bits16(x_bits), _bits16(d_bits), _bits16(u_bits)
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    out = np.zeros(len(ms), np.float64)
    u16p = ctypes.POINTER(_u16)
    rc = lib().ora_linear_lowrank_f64_sampled(_p(a.codes, _u8p), _p(a.scales_lin, _u8p), a.sg,
                                              _p(w.codes, _u8p), _p(w.scales_lin, _u8p), w.sg,
                                              _p(x, u16p), _p(d, u16p), _p(u, u16p), a.cols,
                                              d.shape[0], _p(ms, _i64p), _p(ns, _i64p), len(ms),
                                              _p(out, _f64p))
    if rc != 0:
        raise MemoryError("oracle linear_lowrank_sampled")
    return out
