"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded
inputs. Codes, E4M3 scales (both layouts), global scales and percentiles are compared bit for
bit; GEMM outputs element by element within 1e-3 * max|Y_ref| of the oracle's exact product
(max over the oracle's values), bf16 outputs as the bf16 rounding of a value within that
tolerance."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_14_b200 as nv
import oracle as O
from gpu_helpers import (assert_gemm_close, assert_nvfp4_out_valid, assert_quant_equal, dev_tensor,
                         gemm_tol, gemm_within, gpu_quantize, host, scalar_dev, to_numpy_f64)
from nvfp4_block_scaled_14_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    nv.load()


# ---------------------------------------------------------------------------------------
# quantize
# ---------------------------------------------------------------------------------------

def test_quantize_tiny_workload():
    t = W.tiny()
    for x in (t.W, t.X):
        assert_quant_equal(gpu_quantize(x), O.quantize(x))


@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 96), (127, 160), (129, 64), (300, 1056),
                                       (64, 32), (256, 4096)])
@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_quantize_ragged_shapes(rows, cols, kind):
    x = W.normal((rows, cols), 1.0, 20, rows * 7 + cols)
    x[rows // 2, cols // 3] = 17.0  # an outlier channel value
    if kind == "bf16":
        x = W.to_bf16_bits(x)
    assert_quant_equal(gpu_quantize(x), O.quantize(x))


@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_quantize_static_amax_saturates(kind):
    x = W.normal((200, 288), 1.0, 21, 1)
    if kind == "bf16":
        x = W.to_bf16_bits(x)
    for amax in (0.5, 2.0, 3.3, 1e3):
        assert_quant_equal(gpu_quantize(x, amax=amax), O.quantize(x, amax=amax))


# Tensors of 16 MB and more take the single-pass kernel (shared-memory resident, grid-wide
# barrier); these shapes also have rows that end inside a 128-row band, and (4064 columns)
# a block count per row that is not a multiple of 4, so the swizzled padding is exercised.
@pytest.mark.parametrize("kind,rows,cols", [("f32", 1100, 4064), ("bf16", 2100, 4064),
                                            ("e4m3", 4100, 4096)])
@pytest.mark.parametrize("static", [False, True])
def test_quantize_single_pass_sizes(kind, rows, cols, static):
    x = W.normal((rows, cols), 1.0, 23, rows + cols)
    x[rows - 1, cols - 1] = 19.0
    amax = 7.5 if static else None
    if kind == "e4m3":
        w8, s8 = W.to_fp8_tensorwise(x)
        assert w8.nbytes >= 16 << 20
        assert_quant_equal(gpu_quantize(w8, amax=amax, fp8_scale=s8),
                           O.quantize(w8, amax=amax, fp8_scale=s8))
        return
    if kind == "bf16":
        x = W.to_bf16_bits(x)
    assert x.nbytes >= 16 << 20
    assert_quant_equal(gpu_quantize(x, amax=amax), O.quantize(x, amax=amax))


# Tensors beyond what the CTAs' shared memory holds (148 x 192 KB) take the streamed
# single-launch kernel: two passes through a shared-memory ring, the second back to front
# (the last chunks of each CTA's range still in the ring). Ragged rows and block counts that are
# not a multiple of 4 again.
@pytest.mark.parametrize("kind,rows,cols", [("f32", 2100, 4064), ("bf16", 4100, 4064),
                                            ("e4m3", 8200, 4096), ("bf16", 4096, 12288)])
@pytest.mark.parametrize("static", [False, True])
def test_quantize_streamed_sizes(kind, rows, cols, static):
    x = W.normal((rows, cols), 1.0, 25, rows + cols)
    x[rows - 1, cols - 1] = 21.0
    x[0, 17] = -13.0
    amax = 9.5 if static else None
    if kind == "e4m3":
        w8, s8 = W.to_fp8_tensorwise(x)
        assert w8.nbytes > 148 * 192 * 1024
        assert_quant_equal(gpu_quantize(w8, amax=amax, fp8_scale=s8),
                           O.quantize(w8, amax=amax, fp8_scale=s8))
        return
    if kind == "bf16":
        x = W.to_bf16_bits(x)
    assert x.nbytes > 148 * 192 * 1024
    assert_quant_equal(gpu_quantize(x, amax=amax), O.quantize(x, amax=amax))


def test_quantize_batch_matches_single_calls():
    # a weight re-quantized from FP8, bf16 activations, an fp32 tensor with a static amax, a
    # tiny ragged one: one batched call gives each exactly its own quantization
    w8, s8 = W.to_fp8_tensorwise(W.normal((3072, 3072), 0.02, 33, 1))
    xb = W.to_bf16_bits(W.normal((1000, 3072), 1.0, 33, 2))
    xf = W.normal((300, 1056), 1.0, 33, 3)
    xt = W.to_bf16_bits(W.normal((7, 96), 1.0, 33, 4))
    jobs = [{"x": dev_tensor(w8), "fp8_scale": scalar_dev(s8), "linear": True},
            {"x": dev_tensor(xb), "linear": True},
            {"x": dev_tensor(xf), "static_amax": scalar_dev(2.5), "linear": True},
            {"x": dev_tensor(xt), "linear": True}]
    q = nv.quantize_batch(jobs)
    torch.cuda.synchronize()
    assert_quant_equal(q[0], O.quantize(w8, fp8_scale=s8))
    assert_quant_equal(q[1], O.quantize(xb))
    assert_quant_equal(q[2], O.quantize(xf, amax=2.5))
    assert_quant_equal(q[3], O.quantize(xt))
    assert nv.sync_status() == 0


@pytest.mark.parametrize("case", ["dynamic", "x_static", "w_static", "both_static",
                                  "fp32_ragged", "b_bf16_ragged", "b_fp32_ragged"])
def test_quantize_batch_single_launch_pair(case):
    # two tensors that take the one-launch pair kernel (the larger held in shared memory, the
    # smaller in registers): each gets exactly its single-call result
    w8, s8 = W.to_fp8_tensorwise(W.normal((3072, 3072), 0.02, 34, 1))
    if case == "fp32_ragged":
        xa = W.normal((2050, 3104), 1.0, 34, 3)                 # 25.4 MB fp32, ragged rows
    else:
        xa = W.to_bf16_bits(W.normal((4096, 3072), 1.0, 34, 2))  # the attention projection
    ax = 3.5 if case in ("x_static", "both_static") else None
    aw = 0.05 if case in ("w_static", "both_static") else None
    jobs = [{"x": dev_tensor(xa), "linear": True}]
    if case == "b_bf16_ragged":   # pad blocks (66 per row) and pad rows (1000 rows)
        xb = W.to_bf16_bits(W.normal((1000, 1056), 0.5, 34, 4))
        jobs.append({"x": dev_tensor(xb), "linear": True})
    elif case == "b_fp32_ragged":
        xb = W.normal((300, 1056), 0.5, 34, 5)
        jobs.append({"x": dev_tensor(xb), "linear": True})
    else:
        jobs.append({"x": dev_tensor(w8), "fp8_scale": scalar_dev(s8), "linear": True})
    if ax is not None:
        jobs[0]["static_amax"] = scalar_dev(ax)
    if aw is not None:
        jobs[1]["static_amax"] = scalar_dev(aw)
    if case == "w_static":
        jobs = jobs[::-1]  # order of the jobs does not matter
    q = nv.quantize_batch(jobs)
    torch.cuda.synchronize()
    assert nv.sync_status() == 0
    if case == "w_static":
        q = q[::-1]
    assert_quant_equal(q[0], O.quantize(xa, amax=ax))
    if case.startswith("b_"):
        assert_quant_equal(q[1], O.quantize(xb))
    else:
        assert_quant_equal(q[1], O.quantize(w8, amax=aw, fp8_scale=s8))


def test_quantize_batch_rejects_bad_jobs():
    from nvfp4_block_scaled_14_b200 import _lib as L
    lib = L.load()
    assert lib.nvfp4_quantize_batch(None, 1, None, 0, None) == L.NVFP4_ERR_INVALID_ARG
    jobs = (L.QuantJob * 9)()
    assert lib.nvfp4_quantize_batch(jobs, 9, None, 0, None) == L.NVFP4_ERR_INVALID_ARG
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")  # cols not a multiple of 32
    q = gpu_quantize(W.to_bf16_bits(W.normal((4, 64), 1.0, 33, 5)))
    j = (L.QuantJob * 1)()
    j[0].x, j[0].src, j[0].rows, j[0].cols = x.data_ptr(), L.NVFP4_SRC_BF16, 4, 48
    j[0].static_amax = q.global_scale.data_ptr()
    j[0].codes, j[0].scales_swz = q.codes.data_ptr(), q.scales_swz.data_ptr()
    j[0].global_scale = q.global_scale.data_ptr()
    assert lib.nvfp4_quantize_batch(j, 1, None, 0, None) == L.NVFP4_ERR_SHAPE


def test_quantize_fp8_source_double_quant():
    w8, s8 = W.to_fp8_tensorwise(W.normal((320, 384), 0.02, 22, 1))
    assert_quant_equal(gpu_quantize(w8, fp8_scale=s8), O.quantize(w8, fp8_scale=s8))
    # a layer without weight_scale: scale read as 1.0
    assert_quant_equal(gpu_quantize(w8), O.quantize(w8))
    # static amax on the upcast values
    assert_quant_equal(gpu_quantize(w8, amax=0.03, fp8_scale=s8),
                       O.quantize(w8, amax=0.03, fp8_scale=s8))


def test_quantize_degenerate_inputs():
    z = np.zeros((130, 64), np.float32)
    q = gpu_quantize(z)
    codes, swz, lin, sg = host(q)
    assert sg == 0.0 and not codes.any() and not swz.any() and not lin.any()
    # empty tensor: global scale 0
    e = nv.quantize(torch.zeros((0, 64), device="cuda"), linear=True)
    torch.cuda.synchronize()
    assert float(e.global_scale.cpu()[0]) == 0.0
    # zero blocks inside a nonzero tensor, subnormal block scales
    x = np.zeros((3, 64), np.float32)
    x[0, 0] = 2688.0
    x[1, 16:32] = 6 * 2.0 ** -9
    x[2, 5] = -1e-3
    assert_quant_equal(gpu_quantize(x), O.quantize(x))


def _probe_values(grid, n_random, lo, hi, seed):
    g = np.float32(grid)
    mids = (g[:-1] + g[1:]) / 2
    base = np.concatenate([g, mids]).astype(np.float32)
    pts = [base]
    cur_up, cur_dn = base.copy(), base.copy()
    for _ in range(4):  # four ulps either side of every grid point and midpoint
        cur_up = np.nextafter(cur_up, np.float32(np.inf))
        cur_dn = np.nextafter(cur_dn, np.float32(0))
        pts += [cur_up, cur_dn]
    r = np.random.Generator(np.random.PCG64(seed))
    pts.append(r.uniform(lo, hi, n_random).astype(np.float32))
    v = np.concatenate(pts)
    return v[(v >= lo) & (v <= hi)]


def test_e2m1_rounding_of_the_hardware_matches_oracle():
    # static amax 2688 -> sg = 1; each block holds one 6.0, so its scale is 1.0 and every
    # other value is encoded as itself: the codes show the E2M1 rounding directly.
    vals = _probe_values([0, 0.5, 1, 1.5, 2, 3, 4, 6], 20000, 0.0, 6.0, 30)
    tiny = np.float32([1e-30, 1e-10, 2.0 ** -126, 2.0 ** -149, 0.0])
    vals = np.concatenate([vals, -vals, tiny, -tiny]).astype(np.float32)
    per = 15
    nblk = -(-vals.size // per)
    buf = np.zeros(nblk * per, np.float32)
    buf[:vals.size] = vals
    blocks = np.concatenate([np.full((nblk, 1), 6.0, np.float32), buf.reshape(nblk, per)], 1)
    rows = -(-nblk // 2)
    x = np.zeros((rows * 2, 16), np.float32)
    x[:nblk] = blocks
    x = x.reshape(rows, 32)
    assert_quant_equal(gpu_quantize(x, amax=2688.0), O.quantize(x, amax=2688.0))


def test_e4m3_rounding_of_the_hardware_matches_oracle():
    # static amax 448 -> sg * 6 == 1.0 in fp32, so each block's scale is E4M3(block max).
    e4m3 = np.array([O.e4m3_decode(c) for c in range(127)], np.float32)
    vals = _probe_values(e4m3, 20000, 2.0 ** -12, 448.0, 31)
    vals = np.concatenate([vals, np.float32([500.0, 1e4])])
    rows = -(-vals.size // 2)
    x = np.zeros((rows, 32), np.float32)
    flat = np.zeros(rows * 2, np.float32)
    flat[:vals.size] = vals
    x[:, 0] = flat[0::2]
    x[:, 16] = flat[1::2]
    x[:, 1] = flat[0::2] * np.float32(0.37)
    ref = O.quantize(x, amax=448.0)
    sg = np.float32(448.0) / np.float32(2688.0)
    assert np.float32(sg) * np.float32(6.0) == np.float32(1.0)
    assert_quant_equal(gpu_quantize(x, amax=448.0), ref)


@pytest.mark.parametrize("amax", [333.3, 1.0, 0.0123, 7.77e3])
def test_e4m3_scale_near_rounding_midpoints(amax):
    # block maxima placed within a few ulps of (E4M3 midpoint) * (6 * sg) for a global scale
    # whose reciprocal is inexact: the scale's rounding decision sits right at a boundary.
    sg = np.float32(amax) / np.float32(2688.0)
    t = np.float64(np.float32(sg * np.float32(6.0)))
    e4 = np.array([O.e4m3_decode(c) for c in range(127)], np.float64)
    mids = np.concatenate([(e4[:-1] + e4[1:]) / 2, e4])
    base = (mids * t).astype(np.float32)
    pts = [base]
    up, dn = base.copy(), base.copy()
    for _ in range(6):
        up = np.nextafter(up, np.float32(np.inf))
        dn = np.nextafter(dn, np.float32(0))
        pts += [up, dn]
    r = np.random.Generator(np.random.PCG64(32))
    pts.append((r.uniform(0, 450, 5000) * t).astype(np.float32))
    v = np.concatenate(pts)
    v = v[(v > 0) & (v <= np.float32(amax))]
    rows = -(-v.size // 2)
    flat = np.zeros(rows * 2, np.float32)
    flat[:v.size] = v
    x = np.zeros((rows, 32), np.float32)
    x[:, 0] = flat[0::2]
    x[:, 16] = flat[1::2]
    x[:, 5] = flat[0::2] * np.float32(0.5)
    x[0, 1] = np.float32(amax)  # the tensor amax itself
    assert_quant_equal(gpu_quantize(x, amax=amax), O.quantize(x, amax=amax))
    # the same values through the dynamic-amax path
    assert_quant_equal(gpu_quantize(x), O.quantize(x))


# ---------------------------------------------------------------------------------------
# dequantize
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(64, 256), (33, 96), (1, 32)])
def test_dequantize_bit_exact(rows, cols):
    x = W.normal((rows, cols), 0.02, 23, rows)
    ref = O.quantize(x)
    q = gpu_quantize(x)
    f = nv.dequantize(q, torch.float32).cpu().numpy()
    b = nv.dequantize(q, torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(f.view(np.uint32), O.dequantize(ref, "f32").view(np.uint32))
    assert np.array_equal(b, O.dequantize(ref, "bf16"))


@pytest.mark.parametrize("offset", [0, 16])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_dequantize_output_alignment(offset, out):
    # a 32-byte-aligned output takes 256-bit stores, a 16-byte-aligned one 128-bit stores:
    # both give the oracle's bits (through the C ABI, at an offset into a larger buffer)
    rows, cols = 300, 1056
    x = W.normal((rows, cols), 0.02, 24, rows)
    ref = O.dequantize(O.quantize(x), out)
    q = gpu_quantize(x)
    esz = 4 if out == "f32" else 2
    buf = torch.zeros(rows * cols * esz + 64, dtype=torch.uint8, device="cuda")
    base = buf.data_ptr()
    base += (-base) % 32 + offset
    st = nv.nvfp4_dequantize(q.codes.data_ptr(), q.scales_lin.data_ptr(), q.global_scale.data_ptr(),
                             rows, cols, 0 if out == "f32" else 1, base,
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    start = base - buf.data_ptr()
    got = buf[start:start + rows * cols * esz].cpu().numpy()
    want = ref.view(np.uint8).reshape(-1)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------------------

def _run_linear(xa, xw, out_dtype, amax_a=None):
    qa, qw = gpu_quantize(xa, amax=amax_a), gpu_quantize(xw)
    y = nv.linear(qa, qw, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ra, rw = O.quantize(xa, amax=amax_a), O.quantize(xw)
    assert_quant_equal(qa, ra)
    assert_quant_equal(qw, rw)
    return to_numpy_f64(y), ra, rw


def test_linear_tiny_workload_fp32_out():
    t = W.tiny()
    y, ra, rw = _run_linear(t.X, t.W, torch.float32)
    ref = O.gemm(ra, rw)
    assert_gemm_close(y, ref, False, what="tiny workload")


@pytest.mark.parametrize("M,N,K", [
    (300, 520, 1056),   # >128 rows: BN=256 tiles, ragged M, N and K, split-K
    (129, 256, 256),
    (256, 264, 512),
    (1, 384, 512), (5, 384, 512), (8, 384, 512), (16, 200, 320), (17, 256, 256),
    (33, 384, 512), (100, 384, 512), (128, 384, 512),   # small M: swap-AB
    (64, 1024, 2048),   # swap-AB, many k-tiles per split
    # small M: K split over a thread-block cluster, partials summed through distributed
    # shared memory (uneven k-ranges, odd cluster sizes, the widest B tile)
    (8, 1536, 3072), (3, 640, 1792), (128, 2560, 1024), (64, 12288, 512), (1, 128, 4096),
    # output rows whose byte stride is not a multiple of 16: no TMA store, direct stores
    (8, 1004, 512), (3, 100, 256), (130, 1004, 256),
])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_linear_matches_oracle(M, N, K, out):
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, 24, M))
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, 25, N))
    odt = torch.bfloat16 if out == "bf16" else torch.float32
    y, ra, rw = _run_linear(xa, xw, odt)
    assert_gemm_close(y, O.gemm(ra, rw), out == "bf16", what=f"{M}x{N}x{K} {out}")


@pytest.mark.parametrize("M,N,K", [(8, 1536, 3072), (1, 12288, 1024), (64, 640, 768),
                                   (128, 256, 2048)])
def test_linear_resident_weights_back_to_back(M, N, K):
    # the resident-weights flag lets each small-M call start reading W while the previous
    # call still runs; a chain of calls with different W (and the activations quantized just
    # before the first) must give every call's own result
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, 30, M))
    a_dev = dev_tensor(xa)
    ws = [W.to_bf16_bits(W.normal((N, K), 0.02, 31, N + i)) for i in range(3)]
    qws = [gpu_quantize(x) for x in ws]
    torch.cuda.synchronize()
    qa = nv.quantize(a_dev)  # the chain starts right behind the activation quantizer
    ys = [nv.linear(qa, qw, resident_weights=True) for qw in qws for _ in range(2)]
    torch.cuda.synchronize()
    ra = O.quantize(xa)
    for i, x in enumerate(ws):
        ref = O.gemm(ra, O.quantize(x))
        for y in ys[2 * i:2 * i + 2]:
            assert_gemm_close(to_numpy_f64(y), ref, True, what=f"weight {i}")
    assert nv.sync_status() == 0


def test_linear_degenerate_shapes():
    # through the C ABI: K == 0 is an empty sum, Y = 0 in both output types (for a small-M and
    # a large-M shape); M == 0 or N == 0 leaves nothing to compute and nothing is written
    import ctypes
    from nvfp4_block_scaled_14_b200 import _lib
    L = nv.load()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    for M, N in [(8, 64), (300, 512)]:
        for dt, tdt in [(_lib.NVFP4_BF16, torch.bfloat16), (_lib.NVFP4_F32, torch.float32)]:
            y = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")
            st = L.nvfp4_linear(None, None, None, None, None, None, M, N, 0, dt, ptr(y), None, 0,
                                s)
            torch.cuda.synchronize()
            assert st == _lib.NVFP4_OK
            assert bool((y == 0).all())
    y = torch.full((4, 4), 7.0, dtype=torch.float32, device="cuda")
    for M, N in [(0, 4), (4, 0)]:
        st = L.nvfp4_linear(None, None, None, None, None, None, M, N, 64, _lib.NVFP4_F32, ptr(y),
                            None, 0, s)
        torch.cuda.synchronize()
        assert st == _lib.NVFP4_OK
        assert bool((y == 7.0).all())


def test_linear_rejects_unknown_flag():
    from nvfp4_block_scaled_14_b200 import _lib as L
    qa = gpu_quantize(W.to_bf16_bits(W.normal((4, 64), 1.0, 32, 0)))
    y = torch.zeros((4, 4), dtype=torch.bfloat16, device="cuda")
    st = L.load().nvfp4_linear_ex(qa.codes.data_ptr(), qa.scales_swz.data_ptr(),
                                  qa.global_scale.data_ptr(), qa.codes.data_ptr(),
                                  qa.scales_swz.data_ptr(), qa.global_scale.data_ptr(), 4, 4,
                                  64, L.NVFP4_BF16, y.data_ptr(), None, 0, 2, None)
    assert st == L.NVFP4_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert not y.float().abs().sum().item()


@pytest.mark.parametrize("M,N,K,xkind", [
    (1, 384, 512, "bf16"), (3, 1004, 2048, "f32"), (8, 1536, 3072, "bf16"),
    (16, 640, 1792, "bf16"), (32, 2560, 1024, "f32"), (8, 256, 8192, "bf16"),
    (5, 12288, 4096, "bf16"), (8, 384, 320, "bf16"),
    (64, 512, 1024, "bf16"), (130, 256, 512, "f32"),  # beyond the fused kernel: two steps
])
def test_linear_dynamic_matches_oracle(M, N, K, xkind):
    # activations quantized with their dynamic amax inside the linear call (one kernel for
    # M <= 32): the result is the oracle's quantize-then-GEMM, the reported global scale the
    # oracle's, bit for bit
    xa = W.normal((M, K), 1.0, 36, M + K)
    xa[M // 2, K // 3] = 23.0
    if xkind == "bf16":
        xa = W.to_bf16_bits(xa)
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, 37, N))
    qw = gpu_quantize(xw)
    gs = torch.zeros(1, dtype=torch.float32, device="cuda")
    for resident in (False, True):
        y = nv.linear_dynamic(dev_tensor(xa), qw, x_gs_out=gs, resident_weights=resident)
        torch.cuda.synchronize()
        ra, rw = O.quantize(xa), O.quantize(xw)
        assert_gemm_close(to_numpy_f64(y), O.gemm(ra, rw), True, what=f"resident {resident}")
        assert np.float32(gs.cpu()[0]).tobytes() == np.float32(ra.sg).tobytes()
    assert nv.sync_status() == 0


def test_linear_exact_with_unit_scales():
    # all block scales 1.0 and both global scales 1: 2 * each value is an integer in
    # [-12, 12], the sums are exact in fp32, so the fp32 output must equal the exact product.
    g = np.random.Generator(np.random.PCG64(26))
    for M, N, K in [(64, 256, 512), (200, 300, 1024), (8, 512, 2048)]:
        ac = g.integers(0, 256, (M, K // 2), dtype=np.uint8)
        wc = g.integers(0, 256, (N, K // 2), dtype=np.uint8)

        def swz_ones(rows):
            s = np.zeros(O.swizzled_bytes(rows, K), np.uint8)
            for r in range(rows):
                for b in range(K // 16):
                    s[O.swizzled_offset(r, b, K // 16)] = 0x38
            return s

        ta = nv.NVFP4Tensor(torch.from_numpy(ac).cuda(), torch.from_numpy(swz_ones(M)).cuda(),
                            None, scalar_dev(1.0), M, K)
        tw = nv.NVFP4Tensor(torch.from_numpy(wc).cuda(), torch.from_numpy(swz_ones(N)).cuda(),
                            None, scalar_dev(1.0), N, K)
        y = nv.linear(ta, tw, out_dtype=torch.float32)
        ra = O.Quantized(ac, np.full((M, K // 16), 0x38, np.uint8), None, 1.0, M, K)
        rw = O.Quantized(wc, np.full((N, K // 16), 0x38, np.uint8), None, 1.0, N, K)
        assert np.array_equal(to_numpy_f64(y), O.gemm(ra, rw)), (M, N, K)


@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_linear_large_tile_path(out):
    # enough output tiles that no K split is used: every element against the oracle
    M, N, K = 1280, 2048, 512
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, 27, 1))
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, 27, 2))
    y, ra, rw = _run_linear(xa, xw, torch.bfloat16 if out == "bf16" else torch.float32)
    assert_gemm_close(y, O.gemm(ra, rw), out == "bf16", what=out)


@pytest.mark.parametrize("M,N,K", [
    # CTA-pair kernel (bf16 out, more than 74 tiles of 128 x 256 on 148 SMs)
    (1300, 1960, 512),    # ragged M (a CTA with no valid row) and N (the last 256 x 256 tile
                          # holds 168 columns: one store box lies wholly past the output)
    (1280, 3072, 1024),
    (2000, 2296, 2048),   # ragged M and N, 8 k-tiles
    (4200, 2560, 768),    # two or three tiles per CTA pair (accumulator reuse), ragged M
    # the 5-stage operand ring with one k-tile per tile (every tile starts at a new ring
    # position), 85 tiles on 74 pairs
    (4200, 1280, 256),
])
def test_linear_pair_kernel(M, N, K):
    # every element of the output against the oracle's full product
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, 41, M))
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, 42, N))
    qa, qw = gpu_quantize(xa), gpu_quantize(xw)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nv.linear(qa, qw, out=out)
    torch.cuda.synchronize()
    y = to_numpy_f64(out)
    assert np.isfinite(y).all()  # every element written
    ra, rw = O.quantize(xa), O.quantize(xw)
    assert_quant_equal(qa, ra)
    assert_quant_equal(qw, rw)
    assert_gemm_close(y, O.gemm(ra, rw), True, what=f"pair kernel {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [
    (4200, 1280, 1280),   # exactly as many k-tiles as ring stages, 85 tiles on 74 pairs
    (2560, 3072, 1792),   # 7 k-tiles: the ring wraps inside a tile, 120 tiles on 74 pairs
])
def test_linear_pair_kernel_ring_phases(M, N, K):
    # every 256 x 256 tile checked at its four corners and 12 seeded interior points against the
    # oracle's products computed one by one (a wrong ring phase corrupts whole tiles)
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, 43, M))
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, 44, N))
    qa, qw = gpu_quantize(xa), gpu_quantize(xw)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nv.linear(qa, qw, out=out)
    torch.cuda.synchronize()
    y = to_numpy_f64(out)
    assert np.isfinite(y).all()  # every element written
    ra, rw = O.quantize(xa), O.quantize(xw)
    assert_quant_equal(qa, ra)
    assert_quant_equal(qw, rw)
    rng = np.random.default_rng(45)
    ms, ns = [], []
    for r0 in range(0, M, 256):
        for c0 in range(0, N, 256):
            r1, c1 = min(r0 + 256, M) - 1, min(c0 + 256, N) - 1
            ms += [r0, r0, r1, r1] + list(rng.integers(r0, r1 + 1, 12))
            ns += [c0, c1, c0, c1] + list(rng.integers(c0, c1 + 1, 12))
    ms, ns = np.array(ms, np.int64), np.array(ns, np.int64)
    ref = O.gemm_sampled(ra, rw, ms, ns)
    # the tolerance's max|Y_ref|: over the sample, the oracle's values only
    assert_gemm_close(y[ms, ns], ref, True, tol=gemm_tol(ref), what=f"pair kernel {M}x{N}x{K}")


# ---------------------------------------------------------------------------------------
# calibration percentile
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_calib_percentile_matches_oracle(kind):
    batches = []
    for b in range(5):
        x = W.normal((64, 96 + 32), 1.0, 29, b)
        x.reshape(-1)[::97] *= np.float32(7.0)
        batches.append(W.to_bf16_bits(x) if kind == "bf16" else x)
    f32 = [W.bf16_bits_to_f32(b) if kind == "bf16" else b for b in batches]
    dev = [dev_tensor(b) for b in batches]
    for num, den in [(999, 1000), (1, 2), (1, 1), (1, 1000000)]:
        p, m = nv.calib_percentile_amax(dev, num, den)
        torch.cuda.synchronize()
        rp, rm = O.percentile_abs(f32, num, den)
        assert float(p.cpu()[0]) == rp and float(m.cpu()[0]) == rm, (num, den)


def test_calib_ragged_element_count():
    x = W.normal((1, 1000 + 3), 2.0, 29, 9).ravel()[:1003].copy()
    xs = [x[:1001].copy(), x[1:1002].copy()]
    dev = [torch.from_numpy(a).cuda() for a in xs]
    p, m = nv.calib_percentile_amax(dev)
    torch.cuda.synchronize()
    assert (float(p.cpu()[0]), float(m.cpu()[0])) == O.percentile_abs(xs)


def test_calib_skewed_layout():
    # every 256th 16-byte vector large, the rest small (the large values sit at the same
    # offset of every CTA's range): median and p99.9 still exact
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    nvec = sms * 256
    g = np.random.Generator(np.random.PCG64(35))
    x = (g.random((nvec, 8), dtype=np.float32) * 0.01).astype(np.float32)
    x[::256] = 50.0 + g.random((nvec // 256, 8), dtype=np.float32)
    xb = W.to_bf16_bits(x.reshape(1, -1))
    for num, den in [(1, 2), (999, 1000)]:
        p, m = nv.calib_percentile_amax([dev_tensor(xb), dev_tensor(xb)], num, den)
        torch.cuda.synchronize()
        f = W.bf16_bits_to_f32(xb)
        assert (float(p.cpu()[0]), float(m.cpu()[0])) == O.percentile_abs([f, f], num, den)


def test_sync_status_clean():
    assert nv.sync_status() == 0


# ---------------------------------------------------------------------------------------
# FP8 E4M3 tensorwise layers
# ---------------------------------------------------------------------------------------

def _gpu_e4m3(x: np.ndarray, amax=None):
    q = nv.quantize_e4m3(dev_tensor(x), static_amax=None if amax is None else scalar_dev(amax))
    torch.cuda.synchronize()
    st = nv.sync_status()
    assert st == 0, f"device status {st}"
    return q.codes.cpu().numpy(), float(q.scale.cpu()[0])


@pytest.mark.parametrize("rows,cols", [(1, 8), (3, 37), (1, 5), (64, 3072), (257, 1000),
                                       (4096, 3072), (2050, 3104), (2731, 3072), (2731, 3073)])
@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_quantize_e4m3_matches_oracle(rows, cols, kind):
    # 16 MB and up (n a multiple of 8, within the CTAs' shared memory): the single-pass kernel
    x = W.normal((rows, cols), 1.0, 50, rows * 7 + cols)
    x.reshape(-1)[::101] *= np.float32(40.0)   # a spread of magnitudes, subnormal codes too
    x.reshape(-1)[1::89] *= np.float32(1e-5)
    x.reshape(-1)[2::97] = -0.0
    if kind == "bf16":
        x = W.to_bf16_bits(x)
    codes, s = _gpu_e4m3(x)
    rc, rs = O.quantize_e4m3(x)
    assert s == rs
    assert np.array_equal(codes, rc)


@pytest.mark.parametrize("amax", [0.75, 0.0, 1e-37])
def test_quantize_e4m3_static_amax(amax):
    # values above the static amax saturate at 448; amax 0 gives sign-only codes; a tiny amax
    # makes 1/s overflow (the quotient path must still round correctly)
    x = W.normal((33, 48), 1.0, 51, 1)
    codes, s = _gpu_e4m3(x, amax=amax)
    rc, rs = O.quantize_e4m3(x, amax=amax)
    assert s == rs and np.array_equal(codes, rc)


@pytest.mark.parametrize("shape", [(7, 24), (4096, 3072)])
def test_quantize_e4m3_all_zero(shape):
    x = np.zeros(shape, np.float32)
    x.reshape(-1)[1::3] = -0.0
    codes, s = _gpu_e4m3(W.to_bf16_bits(x))
    assert s == 0.0
    assert np.array_equal(codes, O.quantize_e4m3(W.to_bf16_bits(x))[0])  # sign-only codes


def _e4m3_linear(M, N, K, out_dtype, seed):
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, seed, M))
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, seed + 1, N))
    qa = nv.quantize_e4m3(dev_tensor(xa))
    qw = nv.quantize_e4m3(dev_tensor(xw))
    out = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    nv.linear_e4m3(qa, qw, out=out)
    torch.cuda.synchronize()
    ac, sa = O.quantize_e4m3(xa)
    wc, sw = O.quantize_e4m3(xw)
    assert np.array_equal(qa.codes.cpu().numpy(), ac) and np.array_equal(qw.codes.cpu().numpy(), wc)
    return to_numpy_f64(out), ac, sa, wc, sw


@pytest.mark.parametrize("M,N,K", [
    (1, 256, 128), (5, 384, 512), (300, 520, 1056), (256, 264, 512), (129, 256, 256),
    (130, 1004, 256),   # bf16 rows whose byte stride is not a multiple of 16: direct stores
    (512, 768, 2048),   # several tiles per CTA pair: both accumulators in turn
    (40, 200, 16),      # K of one 16-value step (the rest of the k-tile is zero fill)
])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_linear_e4m3_matches_oracle(M, N, K, out):
    odt = torch.bfloat16 if out == "bf16" else torch.float32
    y, ac, sa, wc, sw = _e4m3_linear(M, N, K, odt, 52)
    assert np.isfinite(y).all()  # every element written
    assert_gemm_close(y, O.gemm_e4m3(ac, sa, wc, sw), out == "bf16", what=f"{M}x{N}x{K} {out}")


def test_linear_e4m3_ragged_pair_tiles():
    # ragged M and N over several 256 x 256 pair tiles: every element against the oracle
    M, N, K = 1300, 1960, 512
    y, ac, sa, wc, sw = _e4m3_linear(M, N, K, torch.bfloat16, 53)
    assert np.isfinite(y).all()
    assert_gemm_close(y, O.gemm_e4m3(ac, sa, wc, sw), True, what="fp8 1300x1960x512")


def test_linear_e4m3_large_sampled():
    M, N, K = 4096, 3072, 3072
    y, ac, sa, wc, sw = _e4m3_linear(M, N, K, torch.bfloat16, 53)
    assert np.isfinite(y).all()
    r = np.random.Generator(np.random.PCG64(54))
    edge = [0, 127, 128, 255, 256, M - 1]
    edge_n = [0, 63, 64, 255, 256, N - 1]
    ms = np.concatenate([r.integers(0, M, 3000), np.repeat(edge, len(edge_n))])
    ns = np.concatenate([r.integers(0, N, 3000), np.tile(edge_n, len(edge))])
    ref = O.gemm_e4m3_sampled(ac, sa, wc, sw, ms, ns)
    # the tolerance from the oracle's sampled values (their max is at most max|Y_ref|)
    assert_gemm_close(y[ms, ns], ref, True, what="fp8 4096x3072x3072 sampled")


def test_linear_e4m3_integer_exact():
    # integer codes with unit scales: every partial sum is an integer below 2^24, so the fp32
    # tensor-core accumulation is exact and equals the oracle bit for bit
    g = np.random.Generator(np.random.PCG64(55))
    M, N, K = 300, 520, 1056
    ints = np.arange(-16, 17).astype(np.float32)
    enc = torch.from_numpy(ints).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ai = g.integers(0, len(ints), (M, K))
    wi = g.integers(0, len(ints), (N, K))
    a = nv.E4M3Tensor(torch.from_numpy(enc[ai]).cuda(), scalar_dev(1.0))
    w = nv.E4M3Tensor(torch.from_numpy(enc[wi]).cuda(), scalar_dev(1.0))
    y = nv.linear_e4m3(a, w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(to_numpy_f64(y), O.gemm_e4m3(enc[ai], 1.0, enc[wi], 1.0))


# ---------------------------------------------------------------------------------------
# linear layer with an NVFP4 output (quantizing epilogue, static amax)
# ---------------------------------------------------------------------------------------

def _unit_scale_operand(rows, K, seed, sg):
    """Random E2M1 codes with every block scale 1.0 (0x38) and a power-of-two global scale:
    all partial sums of the product are exact in fp32. Oracle copy and device copy."""
    g = np.random.Generator(np.random.PCG64(seed))
    codes = g.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    nb = K // 16
    lin = np.full((rows, nb), 0x38, np.uint8)
    swz = np.zeros(O.swizzled_bytes(rows, K), np.uint8)
    for r in range(rows):
        for b in range(nb):
            swz[O.swizzled_offset(r, b, nb)] = 0x38
    q = O.Quantized(codes, lin, swz, sg, rows, K)
    d = nv.NVFP4Tensor(torch.from_numpy(codes).cuda(), torch.from_numpy(swz).cuda(), None,
                       scalar_dev(sg), rows, K)
    return q, d


@pytest.mark.parametrize("M,N,K", [(300, 320, 256), (129, 96, 512), (64, 64, 96),
                                   (1100, 2080, 256), (4100, 544, 128)])
def test_linear_nvfp4_out_exact_identity(M, N, K):
    # exact products: the epilogue's codes, swizzled scales (padding included) and global
    # scale equal the oracle's bit for bit
    qa, da = _unit_scale_operand(M, K, 60 + M, 1.0)
    qw, dw = _unit_scale_operand(N, K, 61 + N, 0.5)
    amax = 0.7 * float(np.abs(O.gemm_sampled(qa, qw, np.arange(M).repeat(4),
                                              np.tile([0, N // 3, N // 2, N - 1], M))).max())
    out = nv.linear_nvfp4_out(da, dw, scalar_dev(amax), "identity")
    torch.cuda.synchronize()
    ref = O.linear_quantize_out(qa, qw, amax, O.ACT_NONE)
    assert float(out.global_scale.cpu()[0]) == ref.sg
    assert np.array_equal(out.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(out.scales_swz.cpu().numpy(), ref.scales_swz)


@pytest.mark.parametrize("act", ["identity", "gelu_tanh"])
@pytest.mark.parametrize("M,N,K", [(500, 640, 1024), (300, 2080, 3072)])
def test_linear_nvfp4_out_within_error_bound(M, N, K, act):
    # realistic operands: the fp32 accumulation (and the fast GELU) move the encoded values by
    # a little, so a code may differ from an exact evaluation where a value sits that close to
    # a rounding boundary. Every block's scale must be the E4M3 rounding of some block maximum
    # within the error bound of the exact one, and every code (with that scale) the E2M1
    # rounding of some value within the bound of the exact value (gpu_helpers).
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, 62, M))
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, 63, N))
    qa_h, qw_h = O.quantize(xa), O.quantize(xw)
    qa, qw = gpu_quantize(xa), gpu_quantize(xw)
    a_act = O.ACT_GELU_TANH if act == "gelu_tanh" else O.ACT_NONE
    y_exact = O.gemm(qa_h, qw_h)
    amax = 0.9 * float(np.abs(O.act_array(y_exact, a_act)).max())  # the largest values saturate
    out = nv.linear_nvfp4_out(qa, qw, scalar_dev(amax), act)
    torch.cuda.synchronize()
    assert_nvfp4_out_valid(out.codes.cpu().numpy(), out.scales_swz.cpu().numpy(),
                           float(out.global_scale.cpu()[0]), qa_h, qw_h, y_exact, a_act, amax)


# ---------------------------------------------------------------------------------------
# linear layer with a BF16 low-rank branch
# ---------------------------------------------------------------------------------------

def _lowrank_case(M, N, K, r, seed, w_std=0.02, lr_std=0.02):
    xb = W.to_bf16_bits(W.normal((M, K), 1.0, 70, seed))
    wb = W.to_bf16_bits(W.normal((N, K), w_std, 71, seed)) if w_std else \
        np.zeros((N, K), np.uint16)
    d = W.to_bf16_bits(W.normal((r, K), lr_std, 72, seed))
    u = W.to_bf16_bits(W.normal((N, r), lr_std, 73, seed))
    return xb, wb, d, u


def _lowrank_per_term(xb, d, t_bits):
    """[rows x r] allowance per unit of |U| for the rows of t_bits (= the rows of xb): each term
    T[m,j] U[n,j] may carry two bf16 roundings (T / alpha on the GPU, T in the oracle: 2^-7 |T|)
    and the fp32 accumulation of T over K (below 2^-12 sum_k |x d|)."""
    x = np.abs(W.bf16_bits_to_f32(xb).astype(np.float64))
    df = np.abs(W.bf16_bits_to_f32(d).astype(np.float64))
    t = np.abs(W.bf16_bits_to_f32(t_bits).astype(np.float64))
    return 2.0 ** -7 * t + 2.0 ** -12 * (x @ df.T)


def _lowrank_bound(xb, d, u, t_bits):
    """Allowance of the branch for every output [M x N]."""
    uf = np.abs(W.bf16_bits_to_f32(u).astype(np.float64))
    return _lowrank_per_term(xb, d, t_bits) @ uf.T


def _assert_lowrank_close(y, ref, branch, bound):
    """Every output within the sound bound (FP4 product's tolerance + the branch's allowance);
    and, since that allowance sums |T U| over the rank, an aggregate check that the error has
    the size of rounding noise: RMS error at most 2^-8 RMS(Y) (bf16 output) + 1 % RMS(branch)
    (its two bf16 roundings leave ~0.3 %) + 1e-4 max|Y| (fp32 accumulation)."""
    assert_gemm_close(y, ref, True, tol=gemm_tol(ref) + bound, what="low-rank layer")
    rms = lambda a: float(np.sqrt(np.mean(np.square(a))))
    limit = 2.0 ** -8 * rms(ref) + 0.01 * rms(branch) + 1e-4 * float(np.abs(ref).max())
    assert rms(y - ref) <= limit, (rms(y - ref), limit)


def _run_lowrank(xb, wb, d, u):
    qa, qw = gpu_quantize(xb), gpu_quantize(wb)
    y = nv.linear_lowrank(qa, qw, dev_tensor(xb), dev_tensor(d), dev_tensor(u))
    torch.cuda.synchronize()
    assert nv.sync_status() == 0
    return to_numpy_f64(y)


@pytest.mark.parametrize("M,N,K,r", [(256, 256, 256, 128), (300, 520, 224, 48),
                                     (130, 264, 512, 256), (512, 768, 3072, 128),
                                     (40, 1032, 96, 16)])
def test_linear_lowrank_matches_oracle(M, N, K, r):
    xb, wb, d, u = _lowrank_case(M, N, K, r, seed=M + N + r)
    y = _run_lowrank(xb, wb, d, u)
    qa_h, qw_h = O.quantize(xb), O.quantize(wb)
    ref = O.linear_lowrank(qa_h, qw_h, xb, d, u)
    bound = _lowrank_bound(xb, d, u, O.lowrank_down(xb, d))
    branch = ref - O.gemm(qa_h, qw_h)
    _assert_lowrank_close(y, ref, branch, bound)
    # the branch is a real part of the output: without it the check fails
    assert np.abs(branch).max() > 0.05 * np.abs(ref).max()
    assert not np.all(gemm_within(y, ref - branch, True, gemm_tol(ref) + bound))


def test_linear_lowrank_zero_up_is_the_linear_layer():
    # a shape nvfp4_linear runs on the same pair kernel (enough tiles for no K split)
    M, N, K, r = 2560, 2048, 1024, 128
    xb, wb, d, _ = _lowrank_case(M, N, K, r, seed=5)
    u = np.zeros((N, r), np.uint16)
    qa, qw = gpu_quantize(xb), gpu_quantize(wb)
    y = nv.linear_lowrank(qa, qw, dev_tensor(xb), dev_tensor(d), dev_tensor(u))
    y0 = nv.linear(qa, qw)
    torch.cuda.synchronize()
    assert torch.equal(y.float(), y0.float())  # adding zero terms leaves the fp32 sums as they are


def test_linear_lowrank_zero_weight_is_the_branch_alone():
    # sgW = 0: the FP4 product vanishes and alpha is taken as 1, so T' is T rounded once
    M, N, K, r = 256, 264, 512, 64
    xb, wb, d, u = _lowrank_case(M, N, K, r, seed=6, w_std=0.0)
    y = _run_lowrank(xb, wb, d, u)
    ref = O.linear_lowrank(O.quantize(xb), O.quantize(wb), xb, d, u)
    bound = _lowrank_bound(xb, d, u, O.lowrank_down(xb, d))
    _assert_lowrank_close(y, ref, ref, bound)


def test_linear_lowrank_full_size_sampled():
    # the attention projection with a rank-128 branch: M4096 N3072 K3072, sampled outputs
    wl = W.attn_proj()
    M, K = wl.X_bf16.shape
    w32 = W.bf16_bits_to_f32(W.to_bf16_bits(W.normal((3072, K), 0.02, 2, 1)))
    wb = W.to_bf16_bits(w32)
    d, u = W.lowrank_factors(N=3072, K=K, r=128)
    y = _run_lowrank(wl.X_bf16, wb, d, u)
    g = np.random.Generator(np.random.PCG64(74))
    ms = np.concatenate([g.integers(0, M, 1500), [0, M - 1, M - 1]])
    ns = np.concatenate([g.integers(0, 3072, 1500), [0, 3071, 0]])
    qa_h, qw_h = O.quantize(wl.X_bf16), O.quantize(wb)
    ref = O.linear_lowrank_sampled(qa_h, qw_h, wl.X_bf16, d, u, ms, ns)
    rows = np.unique(ms)
    per = _lowrank_per_term(wl.X_bf16[rows], d, O.lowrank_down(wl.X_bf16[rows], d))
    uf = np.abs(W.bf16_bits_to_f32(u).astype(np.float64))
    bound = np.einsum("ij,ij->i", per[np.searchsorted(rows, ms)], uf[ns])
    # the tolerance from the oracle's sampled values (their max is at most max|Y_ref|)
    ref_max = float(np.abs(ref).max())
    assert_gemm_close(y[ms, ns], ref, True, tol=gemm_tol(ref) + bound, what="low-rank sampled")
    branch = ref - O.gemm_sampled(qa_h, qw_h, ms, ns)
    rms = lambda a: float(np.sqrt(np.mean(np.square(a))))
    assert rms(y[ms, ns] - ref) <= 2.0 ** -8 * rms(ref) + 0.01 * rms(branch) + 1e-4 * ref_max
