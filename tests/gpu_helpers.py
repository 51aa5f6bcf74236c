"""Shared helpers of the GPU parity tests: move seeded host inputs to the device, run the
library through its C ABI, bring results back, compare with the oracle."""
import numpy as np
import torch

import nvfp4_block_scaled_14_b200 as nv


def dev_tensor(x: np.ndarray) -> torch.Tensor:
    """Host array -> CUDA tensor: float32 as is, uint16 as bf16 bits, uint8 as bytes."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return torch.from_numpy(x).cuda()
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    if x.dtype == np.uint8:
        return torch.from_numpy(x).cuda()
    raise TypeError(x.dtype)


def scalar_dev(v) -> torch.Tensor:
    return torch.tensor([v], dtype=torch.float32, device="cuda")


def gpu_quantize(x: np.ndarray, amax=None, fp8_scale=None):
    t = dev_tensor(x)
    sa = None if amax is None else scalar_dev(amax)
    if x.dtype == np.uint8:
        s8 = None if fp8_scale is None else scalar_dev(fp8_scale)
        q = nv.quantize_fp8(t, s8, static_amax=sa, linear=True)
    else:
        q = nv.quantize(t, static_amax=sa, linear=True)
    torch.cuda.synchronize()
    return q


def host(q):
    return (q.codes.cpu().numpy(), q.scales_swz.cpu().numpy(), q.scales_lin.cpu().numpy(),
            float(q.global_scale.cpu()[0]))


def assert_quant_equal(q, ref):
    codes, swz, lin, sg = host(q)
    assert np.float32(sg).tobytes() == np.float32(ref.sg).tobytes(), (sg, ref.sg)
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}: " \
        f"gpu {codes[tuple(bad[0])]:#04x} oracle {ref.codes[tuple(bad[0])]:#04x}"
    assert np.array_equal(lin, ref.scales_lin)
    assert np.array_equal(swz, ref.scales_swz[:swz.size]) and swz.size == ref.scales_swz.size


def gemm_tolerance(ref: np.ndarray, bf16_out: bool):
    """|gpu - oracle| allowed per element: 1e-3 * max|Y| for the fp32-accumulated product,
    plus one bf16 unit (2^-8 relative) for the output cast when the output is bf16."""
    tol = 1e-3 * float(np.abs(ref).max())
    if bf16_out:
        return tol + np.abs(ref) * 2.0 ** -8
    return tol


def to_numpy_f64(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)
