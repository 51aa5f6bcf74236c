"""NVFP4 quantized linear layer for NVIDIA B200 (sm_100a).

The compute runs in libnvfp4.so (hand-written CUDA for sm_100a behind the C ABI of
include/nvfp4.h). This module marshals torch tensors into those calls: PyTorch supplies
device memory and the current stream, nothing else.

    q_w = quantize_fp8(w_e4m3, w_scale)       # double quantization of an FP8 checkpoint
    q_x = quantize(x_bf16)                    # dynamic per-tensor amax
    y = linear(q_x, q_w)                      # block-scaled W4A4 GEMM, bf16 out
    pct, mx = calib_percentile_amax(batches)  # static p99.9 input scale
    q_s = quantize(x_bf16, static_amax=pct)
    e_w = quantize_e4m3(w_bf16)               # FP8 E4M3 tensorwise (embed / lm_head layers)
    y8 = linear_e4m3(quantize_e4m3(x_bf16), e_w)
    y_lr = linear_lowrank(q_x, q_w, x_bf16, down, up)  # FP4 + BF16 rank-r branch

The C entry points are also available under their own names (``nvfp4_quantize`` ...).
"""
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import (NVFP4_BF16, NVFP4_F32, NVFP4_LINEAR_DEFAULT, NVFP4_LINEAR_RESIDENT_WEIGHTS,
                   NVFP4_OP_CALIB_BF16, NVFP4_OP_CALIB_F32, NVFP4_OP_LINEAR, NVFP4_OP_QUANTIZE,
                   NVFP4Error, check, load)

__all__ = ["NVFP4Tensor", "quantize", "quantize_fp8", "quantize_batch", "dequantize", "linear",
           "linear_dynamic", "linear_nvfp4_out", "linear_lowrank", "E4M3Tensor", "quantize_e4m3", "linear_e4m3",
           "calib_percentile_amax", "sync_status", "free_workspaces", "load", "NVFP4Error"]


def __getattr__(name):
    if name.startswith("nvfp4_"):
        return getattr(_lib, name)
    raise AttributeError(name)


@dataclass
class NVFP4Tensor:
    """A quantized [rows x cols] matrix: codes [rows, cols/2] u8, scales in the tensor-core
    layout (flat u8) and / or linear [rows, cols/16] u8, global scale (1-element fp32)."""
    codes: torch.Tensor
    scales_swz: torch.Tensor
    scales_lin: torch.Tensor
    global_scale: torch.Tensor
    rows: int
    cols: int


def _stream(device):
    return ctypes_ptr(torch.cuda.current_stream(device).cuda_stream)


def ctypes_ptr(v):
    return v if v else None


def _ptr(t):
    return None if t is None else t.data_ptr()


_ws_cache = {}


def _workspace(device, nbytes):
    """The calling stream's workspace on `device` (grown as needed). A workspace holds a call's
    state until its kernels finish, so calls on different streams, which may run at the same
    time, never share one; a buffer is only ever used (and freed) on the stream that
    allocated it. Each stream that has called the library keeps its workspace (at least
    1 MiB) for the life of the process; free_workspaces() drops them all."""
    if nbytes == 0:
        return None
    idx = device.index if device.index is not None else torch.cuda.current_device()
    key = (idx, torch.cuda.current_stream(idx).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def free_workspaces():
    """Drop every cached workspace (after the device work that used them has finished, e.g.
    after torch.cuda.synchronize()); later calls allocate afresh."""
    _ws_cache.clear()


def _alloc_outputs(rows, cols, device, swizzled, linear):
    L = load()
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    swz = (torch.empty(L.nvfp4_scales_bytes(rows, cols, 1), dtype=torch.uint8, device=device)
           if swizzled else None)
    lin = torch.empty((rows, cols // 16), dtype=torch.uint8, device=device) if linear else None
    gs = torch.empty(1, dtype=torch.float32, device=device)
    return codes, swz, lin, gs


def quantize(x: torch.Tensor, static_amax: torch.Tensor = None, swizzled=True, linear=False,
             out: NVFP4Tensor = None) -> NVFP4Tensor:
    """NVFP4-quantize a 2-D fp32 / bf16 CUDA tensor (row-major, cols % 32 == 0)."""
    if x.dtype not in (torch.float32, torch.bfloat16) or x.dim() != 2 or not x.is_cuda:
        raise TypeError("quantize expects a 2-D CUDA fp32 or bf16 tensor")
    x = x.contiguous()
    rows, cols = x.shape
    if out is None:
        codes, swz, lin, gs = _alloc_outputs(rows, cols, x.device, swizzled, linear)
        out = NVFP4Tensor(codes, swz, lin, gs, rows, cols)
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, 0, cols)
    ws = _workspace(x.device, ws_bytes)
    dt = NVFP4_F32 if x.dtype == torch.float32 else NVFP4_BF16
    st = L.nvfp4_quantize(_ptr(x), dt, rows, cols, _ptr(static_amax), _ptr(out.codes),
                          _ptr(out.scales_swz), _ptr(out.scales_lin), _ptr(out.global_scale),
                          _ptr(ws), ws_bytes, _stream(x.device))
    check(st, "nvfp4_quantize")
    return out


def quantize_fp8(x_e4m3: torch.Tensor, fp8_scale: torch.Tensor = None,
                 static_amax: torch.Tensor = None, swizzled=True, linear=False,
                 out: NVFP4Tensor = None) -> NVFP4Tensor:
    """Double quantization: FP8 E4M3 (uint8 bits or float8_e4m3fn) x fp8_scale -> NVFP4."""
    if x_e4m3.dtype == torch.float8_e4m3fn:
        x_e4m3 = x_e4m3.view(torch.uint8)
    if x_e4m3.dtype != torch.uint8 or x_e4m3.dim() != 2 or not x_e4m3.is_cuda:
        raise TypeError("quantize_fp8 expects a 2-D CUDA uint8 / float8_e4m3fn tensor")
    x_e4m3 = x_e4m3.contiguous()
    rows, cols = x_e4m3.shape
    if out is None:
        codes, swz, lin, gs = _alloc_outputs(rows, cols, x_e4m3.device, swizzled, linear)
        out = NVFP4Tensor(codes, swz, lin, gs, rows, cols)
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, 0, cols)
    ws = _workspace(x_e4m3.device, ws_bytes)
    st = L.nvfp4_quantize_fp8_src(_ptr(x_e4m3), _ptr(fp8_scale), rows, cols, _ptr(static_amax),
                                  _ptr(out.codes), _ptr(out.scales_swz), _ptr(out.scales_lin),
                                  _ptr(out.global_scale), _ptr(ws), ws_bytes,
                                  _stream(x_e4m3.device))
    check(st, "nvfp4_quantize_fp8_src")
    return out


def quantize_batch(jobs) -> list:
    """Quantize several tensors in one pass (one amax launch and one encode launch for all);
    every tensor gets exactly what quantize / quantize_fp8 give it. jobs: a list of dicts with
    keys x (fp32 / bf16 tensor, or uint8 / float8_e4m3fn E4M3 bits), and optionally
    fp8_scale, static_amax, swizzled, linear, out. Returns the NVFP4Tensors."""
    import ctypes
    if not 1 <= len(jobs) <= _lib.NVFP4_MAX_QUANT_JOBS:
        raise ValueError("quantize_batch takes 1 to 8 tensors")
    descs = (_lib.QuantJob * len(jobs))()
    outs, keep = [], []
    dev = None
    for i, jb in enumerate(jobs):
        x = jb["x"]
        if x.dtype == torch.float8_e4m3fn:
            x = x.view(torch.uint8)
        if x.dim() != 2 or not x.is_cuda:
            raise TypeError("quantize_batch expects 2-D CUDA tensors")
        if x.dtype == torch.float32:
            src = _lib.NVFP4_SRC_F32
        elif x.dtype == torch.bfloat16:
            src = _lib.NVFP4_SRC_BF16
        elif x.dtype == torch.uint8:
            src = _lib.NVFP4_SRC_E4M3
        else:
            raise TypeError("quantize_batch: fp32, bf16 or E4M3 tensors")
        x = x.contiguous()
        keep.append(x)
        dev = x.device
        rows, cols = x.shape
        out = jb.get("out")
        if out is None:
            codes, swz, lin, gs = _alloc_outputs(rows, cols, x.device, jb.get("swizzled", True),
                                                 jb.get("linear", False))
            out = NVFP4Tensor(codes, swz, lin, gs, rows, cols)
        outs.append(out)
        d = descs[i]
        d.x, d.src = _ptr(x), src
        d.fp8_scale = _ptr(jb.get("fp8_scale"))
        d.rows, d.cols = rows, cols
        d.static_amax = _ptr(jb.get("static_amax"))
        d.codes, d.scales_swz = _ptr(out.codes), _ptr(out.scales_swz)
        d.scales_lin, d.global_scale = _ptr(out.scales_lin), _ptr(out.global_scale)
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, 0, 0, 0)
    ws = _workspace(dev, ws_bytes)
    st = L.nvfp4_quantize_batch(descs, len(jobs), _ptr(ws), ws_bytes, _stream(dev))
    check(st, "nvfp4_quantize_batch")
    return outs


def dequantize(q: NVFP4Tensor, out_dtype=torch.float32, out: torch.Tensor = None) -> torch.Tensor:
    """fp32 / bf16 values of q [rows, cols]; out: an optional preallocated contiguous output."""
    if q.scales_lin is None:
        raise ValueError("dequantize needs the linear scales (quantize(..., linear=True))")
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=out_dtype, device=q.codes.device)
    elif out.dtype != out_dtype or tuple(out.shape) != (q.rows, q.cols) or not out.is_contiguous():
        raise ValueError("out must be a contiguous [rows, cols] tensor of out_dtype")
    dt = NVFP4_F32 if out_dtype == torch.float32 else NVFP4_BF16
    st = load().nvfp4_dequantize(_ptr(q.codes), _ptr(q.scales_lin), _ptr(q.global_scale),
                                 q.rows, q.cols, dt, _ptr(out), _stream(q.codes.device))
    check(st, "nvfp4_dequantize")
    return out


def linear(a: NVFP4Tensor, w: NVFP4Tensor, out_dtype=torch.bfloat16,
           out: torch.Tensor = None, resident_weights: bool = False) -> torch.Tensor:
    """Y = dequant(a) . dequant(w)^T, [a.rows x w.rows], fp32 accumulation.

    resident_weights: w is not written by work still running on the stream (weights quantized
    ahead of time); lets small-M calls start reading w before the previous kernel finishes."""
    if a.cols != w.cols:
        raise ValueError("K mismatch")
    M, N, K = a.rows, w.rows, a.cols
    dev = a.codes.device
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(NVFP4_OP_LINEAR, M, N, K)
    ws = _workspace(dev, ws_bytes)
    dt = NVFP4_F32 if out.dtype == torch.float32 else NVFP4_BF16
    flags = NVFP4_LINEAR_RESIDENT_WEIGHTS if resident_weights else NVFP4_LINEAR_DEFAULT
    st = L.nvfp4_linear_ex(_ptr(a.codes), _ptr(a.scales_swz), _ptr(a.global_scale),
                           _ptr(w.codes), _ptr(w.scales_swz), _ptr(w.global_scale), M, N, K, dt,
                           _ptr(out), _ptr(ws), ws_bytes, flags, _stream(dev))
    check(st, "nvfp4_linear_ex")
    return out


def linear_dynamic(x: torch.Tensor, w: NVFP4Tensor, out_dtype=torch.bfloat16,
                   out: torch.Tensor = None, resident_weights: bool = False,
                   x_gs_out: torch.Tensor = None) -> torch.Tensor:
    """Y = dequant(quantize(x)) . dequant(w)^T with the dynamic per-tensor amax, from fp32 / bf16
    activations x [M x K]; one fused kernel for M <= 16. x_gs_out (1-element fp32 CUDA tensor)
    receives the activations' global scale."""
    if x.dtype not in (torch.float32, torch.bfloat16) or x.dim() != 2 or not x.is_cuda:
        raise TypeError("linear_dynamic expects a 2-D CUDA fp32 or bf16 tensor")
    x = x.contiguous()
    M, K = x.shape
    if K != w.cols:
        raise ValueError("K mismatch")
    N = w.rows
    dev = x.device
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(_lib.NVFP4_OP_LINEAR_DYNAMIC, M, N, K)
    ws = _workspace(dev, ws_bytes)
    flags = NVFP4_LINEAR_RESIDENT_WEIGHTS if resident_weights else NVFP4_LINEAR_DEFAULT
    st = L.nvfp4_linear_dynamic(_ptr(x), NVFP4_F32 if x.dtype == torch.float32 else NVFP4_BF16,
                                _ptr(w.codes), _ptr(w.scales_swz), _ptr(w.global_scale), M, N, K,
                                NVFP4_F32 if out.dtype == torch.float32 else NVFP4_BF16,
                                _ptr(out), _ptr(x_gs_out), _ptr(ws), ws_bytes, flags,
                                _stream(dev))
    check(st, "nvfp4_linear_dynamic")
    return out


def linear_nvfp4_out(a: NVFP4Tensor, w: NVFP4Tensor, static_amax: torch.Tensor,
                     act: str = "identity", out: NVFP4Tensor = None) -> NVFP4Tensor:
    """NVFP4 (static amax) of act(dequant(a) . dequant(w)^T), quantized in the GEMM's epilogue;
    act is "identity" or "gelu_tanh". The result feeds linear() as its activation operand."""
    if a.cols != w.cols:
        raise ValueError("K mismatch")
    acts = {"identity": _lib.NVFP4_ACT_IDENTITY, "gelu_tanh": _lib.NVFP4_ACT_GELU_TANH}
    if act not in acts:
        raise ValueError(f"act must be one of {sorted(acts)}")
    M, N, K = a.rows, w.rows, a.cols
    dev = a.codes.device
    if out is None:
        codes, swz, _, gs = _alloc_outputs(M, N, dev, True, False)
        out = NVFP4Tensor(codes, swz, None, gs, M, N)
    st = load().nvfp4_linear_nvfp4_out(_ptr(a.codes), _ptr(a.scales_swz), _ptr(a.global_scale),
                                       _ptr(w.codes), _ptr(w.scales_swz), _ptr(w.global_scale),
                                       M, N, K, acts[act], _ptr(static_amax), _ptr(out.codes),
                                       _ptr(out.scales_swz), _ptr(out.global_scale),
                                       _stream(dev))
    check(st, "nvfp4_linear_nvfp4_out")
    return out


def linear_lowrank(a: NVFP4Tensor, w: NVFP4Tensor, x: torch.Tensor, down: torch.Tensor,
                   up: torch.Tensor, out: torch.Tensor = None) -> torch.Tensor:
    """Y = dequant(a) . dequant(w)^T + (x . down^T) . up^T, bf16 [a.rows x w.rows].

    x: the layer's bf16 input [M, K] (a is its NVFP4 quantization); down: bf16 [rank, K];
    up: bf16 [N, rank]. The branch's intermediate is kept in bf16 (divided by the FP4 product's
    global scales, so that both parts share one fp32 tensor-core accumulator)."""
    if a.cols != w.cols:
        raise ValueError("K mismatch")
    M, N, K = a.rows, w.rows, a.cols
    if x.dtype != torch.bfloat16 or down.dtype != torch.bfloat16 or up.dtype != torch.bfloat16:
        raise TypeError("x, down and up must be bfloat16")
    rank = down.shape[0]
    if tuple(x.shape) != (M, K) or tuple(down.shape) != (rank, K) or tuple(up.shape) != (N, rank):
        raise ValueError("shape mismatch: x [M, K], down [rank, K], up [N, rank]")
    x, down, up = x.contiguous(), down.contiguous(), up.contiguous()
    dev = a.codes.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(_lib.NVFP4_OP_LINEAR_LOWRANK, M, rank, 0)
    ws = _workspace(dev, ws_bytes)
    st = L.nvfp4_linear_lowrank(_ptr(a.codes), _ptr(a.scales_swz), _ptr(a.global_scale),
                                _ptr(w.codes), _ptr(w.scales_swz), _ptr(w.global_scale),
                                _ptr(x), _ptr(down), _ptr(up), M, N, K, rank, _ptr(out), _ptr(ws),
                                ws_bytes, _stream(dev))
    check(st, "nvfp4_linear_lowrank")
    return out


@dataclass
class E4M3Tensor:
    """FP8 E4M3 tensorwise: codes [rows, cols] uint8 and one fp32 scale (device, [1])."""
    codes: torch.Tensor
    scale: torch.Tensor

    @property
    def rows(self):
        return self.codes.shape[0]

    @property
    def cols(self):
        return self.codes.shape[1]


def quantize_e4m3(x: torch.Tensor, static_amax: torch.Tensor = None,
                  out: E4M3Tensor = None) -> E4M3Tensor:
    """FP8 E4M3 tensorwise quantize of a 2-D fp32 / bf16 CUDA tensor: s = amax / 448,
    code = sign | E4M3(|x| / s) (nearest, ties to even, saturating)."""
    if x.dtype not in (torch.float32, torch.bfloat16) or x.dim() != 2 or not x.is_cuda:
        raise TypeError("quantize_e4m3 expects a 2-D CUDA fp32 or bf16 tensor")
    x = x.contiguous()
    rows, cols = x.shape
    if out is None:
        out = E4M3Tensor(torch.empty((rows, cols), dtype=torch.uint8, device=x.device),
                         torch.empty(1, dtype=torch.float32, device=x.device))
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(_lib.NVFP4_OP_QUANTIZE_E4M3, 0, 0, 0)
    ws = _workspace(x.device, ws_bytes)
    dt = NVFP4_F32 if x.dtype == torch.float32 else NVFP4_BF16
    st = L.nvfp4_quantize_e4m3(_ptr(x), dt, rows, cols, _ptr(static_amax), _ptr(out.codes),
                               _ptr(out.scale), _ptr(ws), ws_bytes, _stream(x.device))
    check(st, "nvfp4_quantize_e4m3")
    return out


def linear_e4m3(a: E4M3Tensor, w: E4M3Tensor, out_dtype=torch.bfloat16,
                out: torch.Tensor = None) -> torch.Tensor:
    """Y = (sA * sW) * A . W^T from E4M3 codes, [a.rows x w.rows], fp32 accumulation."""
    if a.cols != w.cols:
        raise ValueError("K mismatch")
    M, N, K = a.rows, w.rows, a.cols
    dev = a.codes.device
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    dt = NVFP4_F32 if out.dtype == torch.float32 else NVFP4_BF16
    st = load().nvfp4_linear_e4m3(_ptr(a.codes), _ptr(a.scale), _ptr(w.codes), _ptr(w.scale),
                                  M, N, K, dt, _ptr(out), _stream(dev))
    check(st, "nvfp4_linear_e4m3")
    return out


def calib_percentile_amax(batches, num=999, den=1000):
    """Exact nearest-rank num/den percentile of |x| over all batches, and max |x|.
    Returns two 1-element fp32 CUDA tensors (usable as static_amax)."""
    import ctypes
    batches = [b.contiguous() for b in batches]
    dtype = batches[0].dtype
    n = batches[0].numel()
    if any(b.dtype != dtype or b.numel() != n for b in batches):
        raise ValueError("all batches must share dtype and size")
    dev = batches[0].device
    dt = NVFP4_BF16 if dtype == torch.bfloat16 else NVFP4_F32
    L = load()
    ws_bytes = L.nvfp4_workspace_bytes(NVFP4_OP_CALIB_BF16 if dt == NVFP4_BF16
                                       else NVFP4_OP_CALIB_F32, 0, 0, 0)
    ws = _workspace(dev, ws_bytes)
    out = torch.empty(2, dtype=torch.float32, device=dev)
    ptrs = (ctypes.c_void_p * len(batches))(*[b.data_ptr() for b in batches])
    st = L.nvfp4_calib_percentile_amax(ptrs, len(batches), n, dt, num, den, out.data_ptr(),
                                       out.data_ptr() + 4, _ptr(ws), ws_bytes, _stream(dev))
    check(st, "nvfp4_calib_percentile_amax")
    return out[0:1], out[1:2]


def sync_status(device=None):
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    return load().nvfp4_sync_status(_stream(dev))
