"""The GPU tests' comparison helpers, checked on the CPU: the bf16 rounding they use against
torch's cast, the GEMM acceptance rule on constructed cases, and the NVFP4-output validity
check against the oracle's own fused layer (accepted) and against planted mistakes in it
(rejected)."""
import numpy as np
import torch

import oracle as O
from gpu_helpers import assert_nvfp4_out_valid, bf16_rne, gemm_within
from nvfp4_block_scaled_14_b200 import workloads as W


def test_bf16_rne_matches_torch_cast_on_fp32_values():
    g = np.random.Generator(np.random.PCG64(5))
    x = np.concatenate([g.standard_normal(200000) * 10.0 ** g.integers(-20, 20, 200000),
                        [1.0, -1.0, 3.0, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)]])
    x = x.astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(bf16_rne(x.astype(np.float64)), want)


def test_bf16_rne_rounds_fp64_once():
    # just above a tie in fp64 (not representable in fp32): one rounding goes up
    assert bf16_rne(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7
    assert bf16_rne(1.0 + 2.0 ** -8) == 1.0                      # tie to even (down)
    assert bf16_rne(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6      # tie to even (up)
    assert bf16_rne(0.0) == 0.0


def test_gemm_within_bf16_rule():
    ref = np.array([1.0, 100.0, -3.3, 0.0])
    tol = 1e-3 * 100.0
    ok = gemm_within(bf16_rne(ref), ref, True)
    assert ok.all()
    # a value more than tol away, before the cast, fails; one within tol passes
    assert not gemm_within(bf16_rne(ref + 4 * tol), ref, True)[0]
    assert gemm_within(bf16_rne(ref + 0.5 * tol), ref, True).all()
    # fp32 rule: plain |y - ref| <= tol
    assert not gemm_within(ref + 1.01 * tol, ref, False).any()
    assert gemm_within(ref - 0.99 * tol, ref, False).all()


def _fused_case(act):
    M, N, K = 40, 96, 256
    qa = O.quantize(W.to_bf16_bits(W.normal((M, K), 1.0, 90, 1)))
    qw = O.quantize(W.to_bf16_bits(W.normal((N, K), 0.02, 90, 2)))
    y = O.gemm(qa, qw)
    amax = 0.9 * float(np.abs(O.act_array(y, act)).max())
    return qa, qw, y, amax, O.linear_quantize_out(qa, qw, amax, act)


def test_nvfp4_out_check_accepts_the_oracles_fused_layer():
    for act in (O.ACT_NONE, O.ACT_GELU_TANH):
        qa, qw, y, amax, out = _fused_case(act)
        assert_nvfp4_out_valid(out.codes, out.scales_swz, out.sg, qa, qw, y, act, amax)


def test_nvfp4_out_check_rejects_planted_mistakes():
    qa, qw, y, amax, out = _fused_case(O.ACT_GELU_TANH)
    nb = y.shape[1] // 16
    # a code moved by two grid steps in the largest block of row 3
    b = int(np.argmax(out.scales_lin[3]))
    codes = out.codes.copy()
    lo = codes[3, b * 8] & 15
    codes[3, b * 8] = (codes[3, b * 8] & 0xF0) | ((lo + 2) & 7 if lo < 6 else lo - 2)
    try:
        assert_nvfp4_out_valid(codes, out.scales_swz, out.sg, qa, qw, y, O.ACT_GELU_TANH, amax)
        raise RuntimeError("a wrong code passed")
    except AssertionError:
        pass
    # a block scale one E4M3 step too large
    swz = out.scales_swz.copy()
    off = O.swizzled_offset(5, nb - 1, nb)
    swz[off] += 1
    try:
        assert_nvfp4_out_valid(out.codes, swz, out.sg, qa, qw, y, O.ACT_GELU_TANH, amax)
        raise RuntimeError("a wrong scale passed")
    except AssertionError:
        pass
    # the identity layer's output checked as GELU's
    _, _, _, amax_i, out_i = _fused_case(O.ACT_NONE)
    try:
        assert_nvfp4_out_valid(out_i.codes, out_i.scales_swz, out_i.sg, qa, qw, y,
                               O.ACT_GELU_TANH, amax_i)
        raise RuntimeError("the wrong activation passed")
    except AssertionError:
        pass
