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


def bf16_rne(v) -> np.ndarray:
    """Nearest bf16 value of each fp64 value, ties to even, in one rounding (as fp64). bf16
    keeps 8 significant bits: v = m * 2^e with 0.5 <= |m| < 1, so m * 256 rounded to an
    integer (numpy's rint rounds half to even) is the kept significand. Normal range only."""
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def gemm_tol(ref: np.ndarray) -> float:
    """Per-element allowance of the fp32-accumulated product against the oracle's exact
    product: 1e-3 * max|Y_ref|, with Y_ref the oracle's values (never the output under test)."""
    return 1e-3 * float(np.abs(ref).max())


def gemm_within(y: np.ndarray, ref: np.ndarray, bf16_out: bool, tol=None) -> np.ndarray:
    """Which outputs pass. fp32 output: |y - Y_ref| <= tol. bf16 output: y is the
    round-to-nearest-even bf16 of some value within tol of Y_ref; rounding is monotone, so that
    is bf16(Y_ref - tol) <= y <= bf16(Y_ref + tol) -- a difference of more than tol only where
    the output cast itself moved the value across a rounding midpoint. tol may be an array
    (per-element allowances added on top of the product's)."""
    if tol is None:
        tol = gemm_tol(ref)
    if bf16_out:
        return (y >= bf16_rne(ref - tol)) & (y <= bf16_rne(ref + tol))
    return np.abs(y - ref) <= tol


def assert_gemm_close(y: np.ndarray, ref: np.ndarray, bf16_out: bool, tol=None, what=""):
    ok = gemm_within(y, ref, bf16_out, tol)
    if not ok.all():
        i = np.unravel_index(np.argmin(ok), ok.shape)
        t = tol if tol is None or np.isscalar(tol) else np.asarray(tol)[i]
        raise AssertionError(f"{what}: {ok.size - int(ok.sum())} of {ok.size} outputs outside "
                             f"the tolerance; first at {tuple(int(j) for j in i)}: gpu {y[i]!r} "
                             f"oracle {ref[i]!r} (tol {t if t is not None else gemm_tol(ref)})")


def to_numpy_f64(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)


# ---- the linear layer with an NVFP4 output: validity bounds --------------------------------

_E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
                         -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])
GELU_TANH_MAX_SLOPE = 1.13   # max over y of d/dy of the tanh-form GELU (1.1289 near y = 1.5)


def unswizzle_scales(swz: np.ndarray, rows: int, nb: int) -> np.ndarray:
    """[rows x nb] scale bytes read out of the swizzled layout through the oracle's index
    function."""
    import oracle as O
    off = np.fromiter((O.swizzled_offset(r, b, nb) for r in range(rows) for b in range(nb)),
                      np.int64, rows * nb)
    return swz[off].reshape(rows, nb)


def product_error_bound(qa, qw, y_exact: np.ndarray) -> np.ndarray:
    """Per-element bound on |acc * alpha - Y_exact| for the tensor cores' fp32 product.
    Each 16-value block's scaled partial sum sA sW sum(eA eW) is exact in fp32 (at most 20
    significant bits); the accumulator takes K/16 of them, each addition off by at most 2 ulps
    of a running sum whose size is at most S = sum_k |a_k w_k| <= ||a_m|| ||w_n||
    (Cauchy-Schwarz over the dequantized rows); the epilogue's alpha = RN(sgA sgW) and the
    product acc * alpha add 2^-22 |Y|."""
    import oracle as O
    K = qa.cols
    na = np.linalg.norm(O.dequantize(qa, "f32").astype(np.float64), axis=1)
    nw = np.linalg.norm(O.dequantize(qw, "f32").astype(np.float64), axis=1)
    s = np.outer(na, nw) * (1.0 + 2.0 ** -20)  # fp32 dequantized values: 2^-24 each
    return (K / 16) * 2.0 ** -23 * s + 2.0 ** -22 * np.abs(y_exact)


def assert_nvfp4_out_valid(codes, swz, sg, qa, qw, y_exact, act, amax, rows=None):
    """The fused layer's NVFP4 output against exact values: v = act(Y_exact) (fp64), with a
    per-element allowance delta = L * (product bound) + 2^-19 |v| (L the activation's largest
    slope; 2^-19 covers the hardware exp2 / reciprocal of the fast GELU, ~2^-22 each). Every
    block's scale must be the E4M3 rounding of a block maximum within the allowance of the exact
    one, and every code (with that scale) the E2M1 rounding of a value within the allowance of
    the exact value. rows: the rows to check (all by default)."""
    import oracle as O
    M, N = y_exact.shape
    nb = N // 16
    rows = np.arange(M) if rows is None else np.asarray(rows)
    y = y_exact[rows]
    v = O.act_array(y, act)
    slope = GELU_TANH_MAX_SLOPE if act == O.ACT_GELU_TANH else 1.0
    bound = product_error_bound(qa, qw, y_exact)[rows]
    delta = slope * bound + 2.0 ** -19 * np.abs(v)
    sg32 = np.float32(sg)
    assert np.float32(amax) / np.float32(2688.0) == sg32
    t = np.float64(np.float32(sg32 * np.float32(6.0)))
    sb = unswizzle_scales(swz, M, nb)[rows].astype(np.int64)
    av, dv = np.abs(v).reshape(len(rows), nb, 16), delta.reshape(len(rows), nb, 16)
    lo = np.maximum(av - dv, 0.0).max(-1)
    hi = (av + dv).max(-1)
    s_lo = O.e4m3_encode_array(lo / t).reshape(lo.shape).astype(np.int64)
    s_hi = O.e4m3_encode_array(hi / t).reshape(hi.shape).astype(np.int64)
    bad = (sb < s_lo) | (sb > s_hi)
    assert not bad.any(), f"{int(bad.sum())} block scales outside the bound, first (row, " \
        f"block) {np.argwhere(bad)[0].tolist()}"
    # codes, with the block's own scale: E2M1(RN32(RN32(v -+ delta) * r)), r = RN(1/(sb sg))
    e4 = np.array([O.e4m3_decode(c) for c in range(256)], np.float32)
    with np.errstate(divide="ignore"):
        r = (np.float32(1.0) / (e4[sb] * sg32)).astype(np.float32)
    r16 = np.repeat(r, 16, axis=1)
    c_lo = O.e2m1_encode_array(np.float32(v - delta) * r16).reshape(v.shape)
    c_hi = O.e2m1_encode_array(np.float32(v + delta) * r16).reshape(v.shape)
    got = codes[rows]
    got = np.stack([got & 15, got >> 4], -1).reshape(v.shape)
    gv, lv, hv = _E2M1_VALUES[got], _E2M1_VALUES[c_lo], _E2M1_VALUES[c_hi]
    zero_blk = np.repeat(sb == 0, 16, axis=1)
    ok = np.where(zero_blk, got == 0, (lv <= gv) & (gv <= hv))
    assert ok.all(), f"{int((~ok).sum())} codes outside the bound, first at " \
        f"{np.argwhere(~ok)[0].tolist()}"
