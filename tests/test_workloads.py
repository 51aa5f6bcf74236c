"""The seeded synthetic inputs follow the recipe the design notes state: shapes, dtypes,
distributions, the outlier and heavy-tail fractions, and determinism (the CUDA path and the
oracle consume the same bytes)."""
import numpy as np

from nvfp4_block_scaled_14_b200 import workloads as W


def test_draws_are_deterministic_and_distinct_per_tensor():
    a = W.normal((64, 64), 1.0, 7, 1)
    assert np.array_equal(a, W.normal((64, 64), 1.0, 7, 1))
    assert not np.array_equal(a, W.normal((64, 64), 1.0, 7, 2))
    assert not np.array_equal(a, W.normal((64, 64), 1.0, 8, 1))


def test_bf16_bits_round_trip_and_round_to_nearest():
    x = np.float32([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0])
    b = W.to_bf16_bits(x)
    assert b.dtype == np.uint16
    got = W.bf16_bits_to_f32(b)
    assert got.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0]  # ties to even


def test_attention_projection_recipe():
    wl = W.attn_proj()
    assert wl.W_e4m3.shape == (3072, 3072) and wl.W_e4m3.dtype == np.uint8
    assert wl.X_bf16.shape == (4096, 3072) and wl.X_bf16.dtype == np.uint16
    # 0.1 % of the 3072 channels (3) scaled x20
    assert len(wl.outlier_cols) == 3
    x = W.bf16_bits_to_f32(wl.X_bf16).astype(np.float64)
    col_std = x.std(axis=0)
    assert np.all(col_std[wl.outlier_cols] > 15) and np.median(col_std) < 1.05
    # FP8 storage with s8 = amax / 448: the largest code is 448 in magnitude
    assert wl.w_scale > 0
    assert int((wl.W_e4m3 & 0x7F).max()) == 0x7E  # E4M3 448


def test_mlp_and_decode_recipe():
    mp = W.mlp_pair(M=64)
    assert mp.W1.shape == (12288, 3072) and mp.W2.shape == (3072, 12288)
    x2 = W.bf16_bits_to_f32(mp.X2)
    assert x2.shape == (64, 12288) and x2.min() > -0.2  # GELU(z): skewed, bounded below
    w = W.bf16_bits_to_f32(mp.W1[:512]).astype(np.float64)
    assert abs(w.std() - 0.02) < 0.001
    dc = W.decode(Ms=(1, 8))
    assert dc.W.shape == (12288, 4096) and sorted(dc.X) == [1, 8]
    assert abs(W.bf16_bits_to_f32(dc.W[:256]).astype(np.float64).std() - 0.015) < 0.001


def test_calibration_batches_have_one_percent_heavy_tails():
    b = W.bf16_bits_to_f32(W.calib_batch(0, M=512, K=3072)).astype(np.float64)
    assert b.shape == (512, 3072)
    # Student-t(3) draws on 1 % of the entries: far more |x| > 5 than a normal gives (~6e-7)
    frac = np.mean(np.abs(b) > 5.0)
    assert 1e-4 < frac < 1e-2
    assert not np.array_equal(W.calib_batch(1, M=8), W.calib_batch(2, M=8))


def test_lowrank_factors_recipe():
    d, u = W.lowrank_factors(N=3072, K=3072, r=128)
    assert d.shape == (128, 3072) and u.shape == (3072, 128)
    for m in (d, u):
        assert abs(W.bf16_bits_to_f32(m).astype(np.float64).std() - 0.02) < 0.001
