"""Pins for the CPU oracle: each test ties it to something other than itself -- values the
pages print, closed forms, library routines, invariants, or brute force on tiny inputs."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from conftest import golden_dict, read_golden
from nvfp4_block_scaled_14_b200 import workloads as W

E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e4m3_torch_decode(bits):
    """Library decode of E4M3 bit patterns (torch's float8_e4m3fn)."""
    return torch.from_numpy(np.asarray(bits, np.uint8)).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


# ---- the page's stored bytes and worked example ---------------------------------------

def test_first_block_bytes_decode_low_nibble_first():
    rows = read_golden("first_block.txt")
    assert len(rows) == 8  # 8 bytes = 16 codes = one block
    for byte_s, c0_bits, v0, c1_bits, v1 in rows:
        byte = int(byte_s, 16)
        lo, hi = byte & 15, byte >> 4
        assert lo == int(c0_bits, 2) and hi == int(c1_bits, 2)
        assert O.e2m1_decode(lo) == float(v0)
        assert O.e2m1_decode(hi) == float(v1)


def test_block_holds_plus_minus_six():
    # the printed block holds codes 0111 (6) and 1111 (-6): the block scale maps the block
    # amax to the top of the E2M1 grid, as the oracle's scale rule does.
    vals = [float(v) for r in read_golden("first_block.txt") for v in (r[2], r[4])]
    assert max(vals) == 6.0 and min(vals) == -6.0


def test_e2m1_grid_from_its_definition():
    # sign, two exponent bits, one mantissa bit, values 0..6: magnitudes are
    # {0, 0.5} (subnormal) and 2^(e-1)(1 + m/2) for e = 1..3.
    mags = sorted(O.e2m1_decode(c) for c in range(8))
    assert mags == E2M1_GRID
    for c in range(8):
        assert O.e2m1_decode(c | 8) == -O.e2m1_decode(c)
        assert math.copysign(1.0, O.e2m1_decode(c | 8)) == -1.0


def test_worked_example_decode_chain():
    g = golden_dict("worked_example.txt")
    code = int(g["code_bits"], 2)
    assert O.e2m1_decode(code) == float(g["e2m1_value"])
    sb = O.e4m3_encode(float(g["block_scale"]))
    assert sb == 0x49 and O.e4m3_decode(sb) == 4.5  # 4.5 is exact in E4M3
    sg = np.float32(g["global_scale"])
    # one 16-block holding the code, through the oracle's dequantizer
    codes = np.zeros((1, 8), np.uint8)
    codes[0, 0] = code
    q = O.Quantized(codes, np.array([[sb]], np.uint8), None, float(sg), 1, 16)
    w = O.dequantize(q)[0, 0]
    assert f"{w:.5f}" == g["printed_weight"]
    # the base weight rounds to the printed code (round to nearest on the E2M1 grid)
    y = np.float32(g["base_weight"]) * (np.float32(1.0) / (np.float32(4.5) * sg))
    assert O.e2m1_encode(y) == code


def test_storage_is_4_5_bits_per_weight():
    bits = float(golden_dict("page_statistics.txt")["bits_per_weight"])
    for rows, cols in [(1, 16), (3, 64), (256, 256), (128, 3072)]:
        q = O.quantize(np.zeros((rows, cols), np.float32))
        total = q.codes.nbytes + q.scales_lin.nbytes
        assert total * 8 / (rows * cols) == bits


# ---- codecs against library routines and closed forms ---------------------------------

def _all_e4m3_probe_points():
    mags = e4m3_torch_decode(np.arange(127))
    pts = [mags, (mags[:-1] + mags[1:]) / 2]
    base = np.concatenate(pts).astype(np.float32)
    up = np.nextafter(base, np.float32(np.inf))
    down = np.nextafter(base, np.float32(0))
    g = np.random.Generator(np.random.PCG64(7))
    rnd = np.exp(g.uniform(np.log(1e-6), np.log(464.0), 200000)).astype(np.float32)
    v = np.concatenate([base, up, down, rnd, np.float32([2.0 ** -10, 448.0, 463.99997])])
    return v[(v >= 0) & (v < 464.0)]


def test_e4m3_encoder_matches_torch_cast():
    # torch's float8_e4m3fn cast is round-to-nearest-even; below 464 it never saturates,
    # so the oracle's satfinite encoder must agree bit for bit there.
    v = _all_e4m3_probe_points()
    ours = O.e4m3_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_and_roundtrips():
    for c in range(127):
        assert O.e4m3_encode(O.e4m3_decode(c)) == c
    for v in [464.0, 480.0, 1e6, 3e38]:
        assert O.e4m3_encode(v) == 0x7E
    assert O.e4m3_decode(0x7E) == 448.0
    assert math.isnan(O.e4m3_decode(0x7F)) and math.isnan(O.e4m3_decode(0xFF))
    assert O.e4m3_decode(0x01) == 2.0 ** -9  # smallest subnormal


def _e2m1_by_numpy_round(y):
    """Round-half-to-even on each binade's step with numpy (a library rounding rule),
    saturating at 6; returns the code."""
    a = np.abs(y).astype(np.float64)
    v = np.where(a < 2.0, np.round(a * 2) / 2,
                 np.where(a < 4.0, np.round(a), 2 * np.round(a / 2)))
    v = np.minimum(v, 6.0)
    code = np.searchsorted(np.array(E2M1_GRID), v)
    return (code | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def test_e2m1_encoder_matches_numpy_rounding():
    grid = np.array(E2M1_GRID, np.float32)
    mids = (grid[:-1] + grid[1:]) / 2
    base = np.concatenate([grid, mids, np.float32([6.5, 7.0, 100.0, 1e30])])
    near = np.concatenate([base, np.nextafter(base, np.float32(np.inf)),
                           np.nextafter(base, np.float32(0))])
    g = np.random.Generator(np.random.PCG64(11))
    rnd = g.uniform(0, 7, 200000).astype(np.float32)
    y = np.concatenate([near, -near, rnd, -rnd])
    assert np.array_equal(O.e2m1_encode_array(y), _e2m1_by_numpy_round(y))


def test_e2m1_all_codes_roundtrip():
    for c in range(16):
        assert O.e2m1_encode(O.e2m1_decode(c)) == c  # -0.0 keeps its sign: 0b1000


# ---- block and global scale logic, hand-derived ---------------------------------------

def test_global_scale_and_full_block():
    # amax = 1 -> sg = 1/2688; a block of 1.0s gets the top scale 448 and code 6 (0b0111)
    x = np.ones((1, 16), np.float32)
    q = O.quantize(x)
    assert q.sg == float(np.float32(1.0) / np.float32(2688.0))
    assert q.scales_lin[0, 0] == 0x7E
    assert np.all(q.codes == 0x77)


def test_single_spike_and_zero_blocks():
    x = np.zeros((2, 32), np.float32)
    x[0, 0] = 3.0
    x[1, 17] = -3.0
    q = O.quantize(x)
    assert list(q.codes[0]) == [0x07] + [0] * 15
    assert q.scales_lin[0, 1] == 0 and q.scales_lin[1, 0] == 0
    assert q.codes[1, 8] == 0xF0  # element 17 is the high nibble of byte 8: -6 -> 0b1111


def test_all_zero_tensor():
    q = O.quantize(np.zeros((4, 64), np.float32))
    assert q.sg == 0.0 and not q.codes.any() and not q.scales_lin.any()
    assert not O.dequantize(q).any()


def test_subnormal_block_scale_exact():
    # amax = 2688 gives sg = 1 exactly; a block with max 6 * 2^-9 gets the smallest
    # subnormal scale 2^-9 (0x01); its elements 6*2^-9 and 3*2^-9 encode as 6 and 3.
    x = np.zeros((2, 16), np.float32)
    x[0, 0] = 2688.0
    x[1, 0] = 6 * 2.0 ** -9
    x[1, 1] = -3 * 2.0 ** -9
    q = O.quantize(x)
    assert q.sg == 1.0
    assert q.scales_lin[1, 0] == 0x01
    assert q.codes[1, 0] == (0x7 | (0xD << 4))


def test_static_amax_saturates():
    # static amax 1 with data up to 10: scale saturates at 448 and codes at +-6
    x = np.zeros((1, 16), np.float32)
    x[0, :4] = [10.0, -10.0, 0.5, 1.0]
    q = O.quantize(x, amax=1.0)
    assert q.scales_lin[0, 0] == 0x7E
    assert q.codes[0, 0] == (0x7 | (0xF << 4))


def test_requantize_is_identity():
    # with sg a power of two (amax = 10.5 -> sg = 2^-8) every block's max element maps to
    # +-6, so quantize(dequantize(q)) must reproduce q bit for bit.
    x = W.normal((64, 256), 1.0, 90, 1)
    x = np.clip(x, -10.0, 10.0)
    x[3, 5] = 10.5
    q = O.quantize(x)
    assert q.sg == 2.0 ** -8
    q2 = O.quantize(O.dequantize(q))
    assert q2.sg == q.sg
    assert np.array_equal(q2.codes, q.codes) and np.array_equal(q2.scales_lin, q.scales_lin)


def test_swizzled_layout_positions_and_bijection():
    # hand-derived positions of the 128x4 atom layout
    nb = 12
    assert O.swizzled_offset(0, 0, nb) == 0
    assert O.swizzled_offset(1, 0, nb) == 16
    assert O.swizzled_offset(32, 0, nb) == 4
    assert O.swizzled_offset(0, 1, nb) == 1
    assert O.swizzled_offset(0, 4, nb) == 512
    assert O.swizzled_offset(128, 0, nb) == 3 * 512
    rows, cols = 200, 16 * nb
    offs = {O.swizzled_offset(r, b, nb) for r in range(256) for b in range(nb)}
    assert len(offs) == 256 * nb == O.swizzled_bytes(rows, cols)
    q = O.quantize(W.normal((rows, cols), 1.0, 91, 1))
    for r in range(rows):
        for b in range(nb):
            assert q.scales_swz[O.swizzled_offset(r, b, nb)] == q.scales_lin[r, b]
    pad = np.ones(q.scales_swz.size, bool)
    pad[[O.swizzled_offset(r, b, nb) for r in range(rows) for b in range(nb)]] = False
    assert not q.scales_swz[pad].any()


# ---- sources --------------------------------------------------------------------------

def test_bf16_source_equals_widened_fp32():
    x = W.to_bf16_bits(W.normal((32, 128), 1.0, 92, 1))
    widened = torch.from_numpy(x).view(torch.bfloat16).float().numpy()
    a, b = O.quantize(x), O.quantize(widened)
    assert a.sg == b.sg and np.array_equal(a.codes, b.codes)
    assert np.array_equal(a.scales_lin, b.scales_lin)


def test_double_quant_equals_upcast_then_quantize():
    w8, s8 = W.to_fp8_tensorwise(W.normal((48, 96), 0.02, 93, 1))
    up = (torch.from_numpy(w8).view(torch.float8_e4m3fn).float() * torch.tensor(np.float32(s8))
          ).numpy()
    a, b = O.quantize(w8, fp8_scale=s8), O.quantize(up)
    assert a.sg == b.sg and np.array_equal(a.codes, b.codes)
    assert np.array_equal(a.scales_lin, b.scales_lin)
    # a layer without weight_scale is upcast with scale 1
    ones = torch.from_numpy(w8).view(torch.float8_e4m3fn).float().numpy()
    c, d = O.quantize(w8), O.quantize(ones)
    assert np.array_equal(c.codes, d.codes)


# ---- dequantize, error statistics, nibble order ---------------------------------------

def test_dequantize_bf16_is_rounded_fp32():
    q = O.quantize(W.normal((16, 64), 1.0, 94, 1))
    f = O.dequantize(q, "f32")
    b = O.dequantize(q, "bf16")
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.uint16).numpy()
    assert np.array_equal(b, ref)


def test_error_band_and_nibble_order_control():
    st = golden_dict("page_statistics.txt")
    w = W.normal((256, 1024), 0.02, 95, 1)
    q = O.quantize(w)
    err = np.linalg.norm(O.dequantize(q) - w) / np.linalg.norm(w)
    # plausibility, not parity: Gaussian weights land at the top of the page's band
    assert float(st["error_band_low"]) <= err <= float(st["error_band_high"]) + 0.005
    swapped = ((q.codes & 15) << 4 | (q.codes >> 4)).astype(np.uint8)
    qs = O.Quantized(swapped, q.scales_lin, None, q.sg, q.rows, q.cols)
    err_sw = np.linalg.norm(O.dequantize(qs) - w) / np.linalg.norm(w)
    assert err_sw > 10 * err
    assert abs(err_sw - float(st["error_swapped_order"])) < 0.1


# ---- GEMM -----------------------------------------------------------------------------

def _decode_independent(q):
    """Decode with numpy and torch only: nibble split, E2M1 table from the grid, torch E4M3."""
    lo = q.codes & 15
    hi = q.codes >> 4
    codes = np.stack([lo, hi], -1).reshape(q.rows, q.cols)
    mag = np.array(E2M1_GRID)[codes & 7]
    e = np.where(codes & 8, -mag, mag)
    s = e4m3_torch_decode(q.scales_lin.ravel()).reshape(q.rows, q.cols // 16)
    return e * np.repeat(s, 16, axis=1) * float(q.sg)


@pytest.mark.parametrize("M,N,K", [(4, 8, 32), (7, 5, 48), (16, 16, 64), (33, 9, 160)])
def test_gemm_brute_force(M, N, K):
    a = O.quantize(W.normal((M, K), 1.0, 96, M))
    w = O.quantize(W.normal((N, K), 0.02, 97, N))
    ref = _decode_independent(a) @ _decode_independent(w).T
    assert np.allclose(O.gemm(a, w), ref, rtol=1e-12, atol=1e-15)


def test_gemm_integer_exact_unit_scales():
    # scales 1.0 (0x38) and sg = 1: 2*values are integers and the product is exact
    g = np.random.Generator(np.random.PCG64(98))
    M, N, K = 9, 11, 256
    ac = g.integers(0, 256, (M, K // 2), dtype=np.uint8)
    wc = g.integers(0, 256, (N, K // 2), dtype=np.uint8)
    ones_a = np.full((M, K // 16), 0x38, np.uint8)
    ones_w = np.full((N, K // 16), 0x38, np.uint8)
    a = O.Quantized(ac, ones_a, None, 1.0, M, K)
    w = O.Quantized(wc, ones_w, None, 1.0, N, K)

    def ints(c):
        lo, hi = c & 15, c >> 4
        cc = np.stack([lo, hi], -1).reshape(c.shape[0], -1)
        twice = np.array([0, 1, 2, 3, 4, 6, 8, 12])[cc & 7]
        return np.where(cc & 8, -twice, twice).astype(np.int64)

    exact = (ints(ac) @ ints(wc).T) / 4.0
    assert np.array_equal(O.gemm(a, w), exact)


def test_gemm_sampled_matches_full():
    a = O.quantize(W.normal((20, 64), 1.0, 99, 1))
    w = O.quantize(W.normal((30, 64), 0.02, 99, 2))
    full = O.gemm(a, w)
    ms = np.array([0, 19, 7, 3])
    ns = np.array([29, 0, 15, 3])
    assert np.array_equal(O.gemm_sampled(a, w, ms, ns), full[ms, ns])


# ---- percentile -----------------------------------------------------------------------

def test_percentile_nearest_rank_hand_cases():
    x = np.arange(1, 1001, dtype=np.float32)  # rank ceil(1000 * 0.999) = 999
    assert O.percentile_abs([x]) == (999.0, 1000.0)
    y = np.arange(1, 1002, dtype=np.float32)  # rank ceil(1001 * 0.999) = 1000
    assert O.percentile_abs([-y]) == (1000.0, 1001.0)
    assert O.percentile_abs([np.float32([5.0])]) == (5.0, 5.0)
    assert O.percentile_abs([x], 1, 1000)[0] == 1.0  # rank 1


def test_percentile_matches_numpy_sort_over_union():
    g = np.random.Generator(np.random.PCG64(100))
    parts = [g.standard_t(3, size=n).astype(np.float32) for n in (1000, 1, 4096, 777)]
    allv = np.sort(np.abs(np.concatenate(parts)))
    n = allv.size
    for num, den in [(999, 1000), (1, 2), (1, 1), (9999, 10000)]:
        rank = -(-n * num // den)
        pct, mx = O.percentile_abs(parts, num, den)
        assert pct == allv[rank - 1] and mx == allv[-1]


# ---- FP8 E4M3 tensorwise layers ----------------------------------------------------------

def _e4m3_magnitudes():
    """The 127 finite non-negative E4M3 values in code order, decoded by torch."""
    return e4m3_torch_decode(np.arange(127))


def test_e4m3_tensor_grid_points_are_exact():
    # amax = 56 -> s = 56 / 448 = 1/8 exactly; x = s * v for every finite E4M3 value v of
    # either sign must come back as v's own code (scale, sign bit and code order pinned)
    mags = _e4m3_magnitudes()
    x = np.concatenate([mags, -mags[1:], [56.0]]).astype(np.float32) * np.float32(0.125)
    x[-1] = 56.0  # the amax element itself (its own code: 448 = 0x7E)
    codes, s = O.quantize_e4m3(x.reshape(1, -1))
    assert s == 0.125
    want = np.concatenate([np.arange(127), 0x80 | np.arange(1, 127), [0x7E]]).astype(np.uint8)
    assert np.array_equal(codes.ravel(), want)


def test_e4m3_tensor_is_nearest_value_brute_force():
    # every code decodes to a nearest E4M3 value of the fp32 quotient |x| / s (ties to the
    # even code), found by scanning all 127 magnitudes; the sign bit is x's
    g = np.random.Generator(np.random.PCG64(120))
    x = (g.standard_normal(4000) * np.exp(g.uniform(-8, 3, 4000))).astype(np.float32)
    x[::97] = 0.0
    x[1::211] = -0.0
    codes, s = O.quantize_e4m3(x)
    assert s == np.float32(np.abs(x).max()) / np.float32(448.0)
    mags = _e4m3_magnitudes()
    q = (np.abs(x) / np.float32(s)).astype(np.float64)  # fp32 division, widened exactly
    for xi, qi, c in zip(x, q, codes):
        d = np.abs(mags - min(qi, 448.0))
        best = np.flatnonzero(d == d.min())
        expect = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (c & 0x7F) == expect and (c >> 7) == int(np.signbit(xi))


def test_e4m3_tensor_matches_torch_cast():
    # a library route to the same codes: fp32 quotient, then torch's RNE float8_e4m3fn cast
    g = np.random.Generator(np.random.PCG64(121))
    x = g.standard_normal((37, 48)).astype(np.float32) * np.float32(3.0)
    codes, s = O.quantize_e4m3(x)
    ref = torch.from_numpy(x / np.float32(s)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_e4m3_tensor_bf16_source_and_static_amax():
    g = np.random.Generator(np.random.PCG64(122))
    xf = g.standard_normal((8, 40)).astype(np.float32)
    xb = W.to_bf16_bits(xf)
    cb, sb = O.quantize_e4m3(xb)
    cf, sf = O.quantize_e4m3(W.bf16_bits_to_f32(xb))
    assert sb == sf and np.array_equal(cb, cf)  # bf16 widens exactly
    # static amax below max|x|: s = amax / 448 and the values above it saturate at 448
    c, s = O.quantize_e4m3(xf, amax=0.5)
    assert s == np.float32(0.5) / np.float32(448.0)
    big = np.abs(xf) > 0.5 * (1 + 2 ** -4)
    assert np.all((c[big] & 0x7F) == 0x7E) and np.array_equal(c[big] >> 7, np.signbit(xf[big]))
    # amax 0: sign-only codes; an all-zero tensor: zero codes and s = 0
    c0, s0 = O.quantize_e4m3(xf, amax=0.0)
    assert s0 == 0.0 and np.array_equal(c0, np.where(np.signbit(xf), 0x80, 0).astype(np.uint8))
    cz, sz = O.quantize_e4m3(np.zeros((3, 16), np.float32))
    assert sz == 0.0 and not cz.any()


def test_gemm_e4m3_integer_exact():
    # E4M3 holds the integers -16..16 exactly: with unit scales the product is numpy's integer
    # matmul, and the scales multiply it (a transposed operand or a wrong index would differ)
    g = np.random.Generator(np.random.PCG64(123))
    M, N, K = 7, 13, 96
    ai = g.integers(-16, 17, (M, K))
    wi = g.integers(-16, 17, (N, K))
    ints = np.arange(-16, 17)
    enc = {int(v): int(c) for v, c in zip(ints, torch.from_numpy(ints.astype(np.float32))
                                          .to(torch.float8_e4m3fn).view(torch.uint8).numpy())}
    ac = np.vectorize(enc.get)(ai).astype(np.uint8)
    wc = np.vectorize(enc.get)(wi).astype(np.uint8)
    exact = (ai @ wi.T).astype(np.float64)
    assert np.array_equal(O.gemm_e4m3(ac, 1.0, wc, 1.0), exact)
    assert np.array_equal(O.gemm_e4m3(ac, 0.5, wc, 3.0), 1.5 * exact)
    ms, ns = np.array([0, 6, 3]), np.array([12, 0, 5])
    assert np.array_equal(O.gemm_e4m3_sampled(ac, 0.5, wc, 3.0, ms, ns), 1.5 * exact[ms, ns])


def test_gemm_e4m3_is_dequantized_product():
    # the product of the layer equals the fp64 product of the dequantized operands
    g = np.random.Generator(np.random.PCG64(124))
    a, sa = O.quantize_e4m3(g.standard_normal((5, 64)).astype(np.float32))
    w, sw = O.quantize_e4m3((g.standard_normal((9, 64)) * 0.02).astype(np.float32))
    da = e4m3_torch_decode(a) * sa
    dw = e4m3_torch_decode(w) * sw
    assert np.allclose(O.gemm_e4m3(a, sa, w, sw), da @ dw.T, rtol=1e-12, atol=0)


# ---- linear layer with an NVFP4 output -------------------------------------------------

def test_gelu_tanh_matches_torch():
    y = np.concatenate([np.linspace(-12, 12, 2001), [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0]])
    ref = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    ours = np.array([O.gelu_tanh(v) for v in y])
    assert np.allclose(ours, ref, rtol=1e-13, atol=1e-15)
    assert O.gelu_tanh(0.0) == 0.0 and O.gelu_tanh(40.0) == 40.0 and O.gelu_tanh(-40.0) == 0.0


def _exact_product_operands(M, N, K, seed, a_sg=1.0, w_sg=0.5):
    # unit block scales (0x38) and power-of-two global scales: every partial sum of
    # E2M1 x E2M1 products is a multiple of 1/4 below 2^24, so fp32 holds the product exactly
    g = np.random.Generator(np.random.PCG64(seed))
    ac = g.integers(0, 256, (M, K // 2), dtype=np.uint8)
    wc = g.integers(0, 256, (N, K // 2), dtype=np.uint8)
    a = O.Quantized(ac, np.full((M, K // 16), 0x38, np.uint8), None, a_sg, M, K)
    w = O.Quantized(wc, np.full((N, K // 16), 0x38, np.uint8), None, w_sg, N, K)
    return a, w


@pytest.mark.parametrize("act", [O.ACT_NONE, O.ACT_GELU_TANH])
def test_linear_quantize_out_equals_quantize_of_product(act):
    M, N, K = 5, 64, 96
    a, w = _exact_product_operands(M, N, K, 130)
    y = O.gemm(a, w).astype(np.float32)  # exact: power-of-two scales, small integer sums
    assert np.array_equal(y.astype(np.float64), O.gemm(a, w))
    if act == O.ACT_GELU_TANH:
        y = torch.nn.functional.gelu(torch.from_numpy(y.astype(np.float64)),
                                     approximate="tanh").numpy().astype(np.float32)
    amax = 0.8 * float(np.abs(y).max())  # some values saturate
    ref = O.quantize(y, amax=amax)
    got = O.linear_quantize_out(a, w, amax, act)
    assert got.sg == ref.sg
    assert np.array_equal(got.codes, ref.codes)
    assert np.array_equal(got.scales_lin, ref.scales_lin)
    assert np.array_equal(got.scales_swz, ref.scales_swz)


@pytest.mark.parametrize("act", [O.ACT_NONE, O.ACT_GELU_TANH])
def test_linear_act_sampled_is_activation_of_gemm(act):
    a = O.quantize(W.normal((20, 64), 1.0, 131, 1))
    w = O.quantize(W.normal((30, 64), 0.02, 131, 2))
    ms, ns = np.array([0, 19, 7, 3]), np.array([29, 0, 15, 3])
    y = O.gemm_sampled(a, w, ms, ns)
    if act == O.ACT_GELU_TANH:
        y = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    assert np.allclose(O.linear_act_sampled(a, w, act, ms, ns), y, rtol=1e-14, atol=0)


# ---- FP4 linear layer with a BF16 low-rank branch ("What I quantized") ---------------------

def _bf16(vals) -> np.ndarray:
    """Exactly representable values -> bf16 bits (checked to be exact)."""
    v = np.asarray(vals, np.float32)
    bits = W.to_bf16_bits(v)
    assert np.array_equal(W.bf16_bits_to_f32(bits), v), "value is not a bf16"
    return bits


def _lowrank_operands(M, N, K, seed):
    g = np.random.default_rng(seed)
    x = (g.standard_normal((M, K)) * 0.5).astype(np.float32)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    xb = W.to_bf16_bits(x)
    return O.quantize(W.bf16_bits_to_f32(xb)), O.quantize(w), xb


def test_f64_to_bf16_rounds_once():
    # values exact in fp32 round as torch's fp32 -> bf16 cast does (nearest, ties to even)
    g = np.random.default_rng(7)
    v = (g.standard_normal(4000) * np.exp2(g.integers(-40, 40, 4000))).astype(np.float32)
    v = np.concatenate([v, np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130,
                                       3 * 2 ** -134, 0.0])])
    ref = W.to_bf16_bits(v)
    got = np.array([O.f64_to_bf16(float(t)) for t in v], np.uint16)
    assert np.array_equal(got, ref)
    # one rounding from fp64: 1 + 2^-8 + 2^-30 lies above the tie, so it rounds up, whereas
    # rounding through fp32 first (to the tie 1 + 2^-8) would give 1.0
    assert O.f64_to_bf16(1 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert O.f64_to_bf16(-(1 + 2 ** -8 + 2 ** -30)) == 0xBF81


def test_lowrank_zero_up_is_the_fp4_gemm():
    M, N, K, r = 12, 20, 64, 16
    a, w, xb = _lowrank_operands(M, N, K, 1)
    d = W.to_bf16_bits(np.random.default_rng(2).standard_normal((r, K)).astype(np.float32))
    u = np.zeros((N, r), np.uint16)
    assert np.array_equal(O.linear_lowrank(a, w, xb, d, u), O.gemm(a, w))


def test_lowrank_one_hot_factors_select_entries():
    # D[j] = e_{sel[j]} makes T = x[:, sel] exactly; U[n] = e_{pick[n]} * c[n] then makes the
    # branch c[n] * x[m, sel[pick[n]]]. Swapping D / U, transposing either or dropping the
    # branch gives other entries.
    M, N, K, r = 9, 14, 96, 8
    a, w, xb = _lowrank_operands(M, N, K, 3)
    sel = np.array([5, 77, 0, 31, 95, 12, 64, 40])
    pick = np.arange(N) % r
    c = np.float32([1, -2, 0.5, 4, -0.25, 8, 1, -1, 2, 0.125, -4, 1, 0.5, 16])
    d = np.zeros((r, K), np.float32)
    d[np.arange(r), sel] = 1.0
    u = np.zeros((N, r), np.float32)
    u[np.arange(N), pick] = c
    y = O.linear_lowrank(a, w, xb, _bf16(d), _bf16(u))
    x = W.bf16_bits_to_f32(xb).astype(np.float64)
    expect = O.gemm(a, w) + x[:, sel[pick]] * c.astype(np.float64)[None, :]
    np.testing.assert_allclose(y, expect, rtol=0, atol=1e-12 * np.abs(expect).max())
    # the branch against a library product on exact small integers: any summation order
    g = np.random.default_rng(4)
    xi = g.integers(-2, 3, (M, K)).astype(np.float32)
    di = g.integers(-1, 2, (r, K)).astype(np.float32)
    ui = g.integers(-3, 4, (N, r)).astype(np.float32)
    xib = _bf16(xi)
    zero_a = O.quantize(np.zeros((M, K), np.float32))
    lr = O.linear_lowrank(zero_a, w, xib, _bf16(di), _bf16(ui))
    t = torch.from_numpy(xi.astype(np.float64)) @ torch.from_numpy(di.astype(np.float64)).T
    assert torch.all(t.abs() <= 256)  # |T| <= 2 * 96: integers this small are bf16s
    ref = (t @ torch.from_numpy(ui.astype(np.float64)).T).numpy()
    assert np.array_equal(lr, ref)


def test_lowrank_intermediate_is_rounded_once_to_bf16():
    # T = x . D^T with D = ones: each row's sum is set by hand; U = identity reads T back.
    K, r = 32, 6
    rows = [
        ([1.0, 2.0 ** -9], 1.0),                             # below half an ulp: down
        ([1.0, 2.0 ** -8], 1.0),                             # tie, even neighbour 1.0
        ([1.0, 2.0 ** -7, 2.0 ** -8], 1.0 + 2.0 ** -6),      # tie, even neighbour 1 + 2^-6
        ([1.0, 2.0 ** -8, 2.0 ** -30], 1.0 + 2.0 ** -7),     # just above the tie: up
        ([-1.0, -(2.0 ** -7), -(2.0 ** -8)], -(1.0 + 2.0 ** -6)),
        ([3.0, 2.0 ** -7], 3.0),                             # ulp of 3 is 2^-6
    ]
    x = np.zeros((len(rows), K), np.float32)
    for i, (vals, _) in enumerate(rows):
        x[i, :len(vals)] = vals
    d = np.zeros((r, K), np.float32)
    d[:, :] = 1.0
    zero_a = O.quantize(np.zeros((len(rows), K), np.float32))
    zero_w = O.quantize(np.zeros((r, K), np.float32))
    u = np.eye(r, dtype=np.float32)
    y = O.linear_lowrank(zero_a, zero_w, _bf16(x), _bf16(d), _bf16(u))
    for i, (_, t) in enumerate(rows):
        assert np.all(y[i] == t), (i, y[i], t)
    t_bits = O.lowrank_down(_bf16(x), _bf16(d))
    assert np.array_equal(W.bf16_bits_to_f32(t_bits)[:, 0], np.float32([t for _, t in rows]))


def test_lowrank_sampled_matches_full_and_scales_linearly():
    M, N, K, r = 10, 24, 128, 16
    a, w, xb = _lowrank_operands(M, N, K, 5)
    g = np.random.default_rng(6)
    d = W.to_bf16_bits((g.standard_normal((r, K)) * 0.05).astype(np.float32))
    u = W.to_bf16_bits((g.standard_normal((N, r)) * 0.05).astype(np.float32))
    y = O.linear_lowrank(a, w, xb, d, u)
    ms, ns = g.integers(0, M, 40), g.integers(0, N, 40)
    assert np.array_equal(O.linear_lowrank_sampled(a, w, xb, d, u, ms, ns), y[ms, ns])
    # doubling U doubles the branch exactly (a power-of-two scale of every term)
    u2 = W.to_bf16_bits(W.bf16_bits_to_f32(u) * 2)
    base = O.gemm(a, w)
    assert np.array_equal(O.linear_lowrank(a, w, xb, d, u2) - base, 2 * (y - base))
