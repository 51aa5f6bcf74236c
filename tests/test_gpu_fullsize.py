"""GPU parity at the workloads' full sizes, in the launch configuration bench.py times:
codes / scales / global scales bit-exact against the oracle over the whole tensors; the
attention projection's GEMM (the CTA-pair kernel) element by element against the oracle's full
product, the other GEMMs on sampled positions (the oracle computes them one by one);
dequantize bit-exact over a whole 12288 x 3072 weight; calibration by the nearest-rank property
that holds at any size."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_14_b200 as nv
import oracle as O
from gpu_helpers import (assert_gemm_close, assert_nvfp4_out_valid, assert_quant_equal,
                         dev_tensor, gpu_quantize, scalar_dev, to_numpy_f64)
from nvfp4_block_scaled_14_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    nv.load()


def _sampled_check(y, ra, rw, n_samples, seed, bf16=True, extra=()):
    Mr, Nr = y.shape
    g = np.random.Generator(np.random.PCG64(seed))
    ms = np.concatenate([g.integers(0, Mr, n_samples), [0, Mr - 1] + [e[0] for e in extra]])
    ns = np.concatenate([g.integers(0, Nr, n_samples), [Nr - 1, 0] + [e[1] for e in extra]])
    ref = O.gemm_sampled(ra, rw, ms, ns)
    # tolerance from the oracle's own values (max over the samples <= max over all of Y)
    assert_gemm_close(y[ms, ns], ref, bf16, what=f"sampled {Mr}x{Nr}")


@pytest.fixture(scope="module")
def attn_proj():
    """The attention projection's operands (W re-quantized from FP8, X bf16 with outlier
    channels), their oracle quantization, and the oracle's full product Y = X W^T in fp64
    (4096 x 3072 x 3072: about a minute on the host cores), shared by the tests below."""
    wl = W.attn_proj()
    rw = O.quantize(wl.W_e4m3, fp8_scale=wl.w_scale)
    rx = O.quantize(wl.X_bf16)
    return wl, rx, rw, O.gemm(rx, rw)


def test_attn_proj_double_quant_full(attn_proj):
    # the bench's workload: both quantizations bit-exact, and every one of the 12.6 M outputs
    # of the CTA-pair GEMM within the tolerance of the oracle's exact product
    wl, rx, rw, ref = attn_proj
    qw = gpu_quantize(wl.W_e4m3, fp8_scale=wl.w_scale)
    qx = gpu_quantize(wl.X_bf16)
    assert_quant_equal(qw, rw)
    assert_quant_equal(qx, rx)
    out = torch.full((4096, 3072), float("nan"), dtype=torch.bfloat16, device="cuda")
    nv.linear(qx, qw, out=out)
    y = to_numpy_f64(out)
    assert np.isfinite(y).all()
    assert_gemm_close(y, ref, True, what="attention projection 4096x3072x3072")


@pytest.mark.parametrize("act", ["identity", "gelu_tanh"])
def test_attn_proj_nvfp4_out_every_block(attn_proj, act):
    # the GEMM with the NVFP4-output epilogue on the same operands: all 786,432 blocks of the
    # 4096 x 3072 output against the exact product's bounds
    wl, rx, rw, ref = attn_proj
    qw = gpu_quantize(wl.W_e4m3, fp8_scale=wl.w_scale)
    qx = gpu_quantize(wl.X_bf16)
    a_act = O.ACT_GELU_TANH if act == "gelu_tanh" else O.ACT_NONE
    amax = 0.9 * float(np.abs(O.act_array(ref, a_act)).max())
    out = nv.linear_nvfp4_out(qx, qw, scalar_dev(amax), act)
    torch.cuda.synchronize()
    assert_nvfp4_out_valid(out.codes.cpu().numpy(), out.scales_swz.cpu().numpy(),
                           float(out.global_scale.cpu()[0]), rx, rw, ref, a_act, amax)


def test_mlp_pair_full():
    mp = W.mlp_pair()
    q1, r1 = gpu_quantize(mp.W1), O.quantize(mp.W1)
    assert_quant_equal(q1, r1)
    qa1, ra1 = gpu_quantize(mp.X1), O.quantize(mp.X1)
    assert_quant_equal(qa1, ra1)
    y1 = to_numpy_f64(nv.linear(qa1, q1))
    _sampled_check(y1, ra1, r1, 1500, 41)
    del q1, qa1, y1
    q2, r2 = gpu_quantize(mp.W2), O.quantize(mp.W2)
    assert_quant_equal(q2, r2)
    qa2, ra2 = gpu_quantize(mp.X2), O.quantize(mp.X2)
    assert_quant_equal(qa2, ra2)
    y2 = to_numpy_f64(nv.linear(qa2, q2))
    _sampled_check(y2, ra2, r2, 1000, 42)


def test_decode_small_m_full():
    dc = W.decode()
    qw, rw = gpu_quantize(dc.W), O.quantize(dc.W)
    assert_quant_equal(qw, rw)
    for m, x in dc.X.items():
        qa, ra = gpu_quantize(x), O.quantize(x)
        assert_quant_equal(qa, ra)
        y = to_numpy_f64(nv.linear(qa, qw))
        if m <= 32:
            assert_gemm_close(y, O.gemm(ra, rw), True, what=f"decode M{m}")
        else:
            _sampled_check(y, ra, rw, 1500, 43 + m)


def test_calibration_full_53_batches():
    nb = 53
    dev_batches, counts_lt, counts_le = [], 0, 0
    host = []
    for b in range(nb):
        xb = W.calib_batch(b)
        dev_batches.append(dev_tensor(xb))
        host.append(xb)
    p, mx = nv.calib_percentile_amax(dev_batches)
    torch.cuda.synchronize()
    p, mx = float(p.cpu()[0]), float(mx.cpu()[0])
    n = nb * 4096 * 3072
    rank = -(-n * 999 // 1000)
    # nearest-rank property: #{|x| < p} < rank <= #{|x| <= p}; max is the largest |x|
    true_max = 0.0
    for xb in host:
        a = np.abs(W.bf16_bits_to_f32(xb))
        counts_lt += int(np.count_nonzero(a < p))
        counts_le += int(np.count_nonzero(a <= p))
        true_max = max(true_max, float(a.max()))
    assert counts_lt < rank <= counts_le
    assert mx == true_max
    # quantize an evaluation batch with the p99.9 static scale and with the max, run the GEMM
    ev = W.calib_batch(53)
    wt = W.calib_weight()
    qw, rw = gpu_quantize(wt), O.quantize(wt)
    assert_quant_equal(qw, rw)
    for amax in (p, mx):
        qa, ra = gpu_quantize(ev, amax=amax), O.quantize(ev, amax=amax)
        assert_quant_equal(qa, ra)
        y = to_numpy_f64(nv.linear(qa, qw))
        _sampled_check(y, ra, rw, 1000, 44)


def test_step_in_cuda_graph_matches_eager():
    # the attention-projection step as the bench replays it: W (FP8) and X quantized in one
    # launch, then the GEMM, captured in a CUDA graph over two input sets (the kernels overlap
    # through programmatic dependent launch) -- bit for bit the eager results
    wl = W.attn_proj()
    w8 = torch.from_numpy(wl.W_e4m3).cuda()
    s8 = torch.tensor([wl.w_scale], dtype=torch.float32, device="cuda")
    xs = [dev_tensor(wl.X_bf16), dev_tensor(W.to_bf16_bits(W.normal((4096, 3072), 1.0, 80, 1)))]
    ws = [w8, w8.clone()]
    ref = []
    for w, x in zip(ws, xs):
        qw, qx = nv.quantize_batch([{"x": w, "fp8_scale": s8}, {"x": x}])
        ref.append(nv.linear(qx, qw).clone())
    qw, qx = nv.quantize_batch([{"x": ws[0], "fp8_scale": s8}, {"x": xs[0]}])
    y = torch.empty_like(ref[0])
    outs = [torch.empty_like(ref[0]) for _ in range(2)]

    def step(i):
        nv.quantize_batch([{"x": ws[i], "fp8_scale": s8, "out": qw}, {"x": xs[i], "out": qx}])
        nv.linear(qx, qw, out=y)
        outs[i].copy_(y)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(0)
        step(1)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(0)
        step(1)
    for _ in range(2):
        outs[0].zero_()
        outs[1].zero_()
        g.replay()
        torch.cuda.synchronize()
        for i in range(2):
            assert torch.equal(outs[i].view(torch.int16), ref[i].view(torch.int16)), i
    del g


def test_mlp_step_in_cuda_graph_matches_eager():
    # the bench's headline step (quantize X1 4096x3072, GEMM1 N12288 K3072, quantize X2
    # 4096x12288, GEMM2 N3072 K12288) for two input sets, captured in one CUDA graph and replayed
    # twice: the single-pass and streamed quantizers take a fresh grid barrier per captured
    # launch, the pair GEMMs run their five-stage ring; every output must match the eager run bit
    # for bit
    mp = W.mlp_pair()
    w1, w2 = nv.quantize(dev_tensor(mp.W1)), nv.quantize(dev_tensor(mp.W2))
    x1s = [dev_tensor(mp.X1), dev_tensor(W.to_bf16_bits(W.normal((4096, 3072), 1.0, 81, 1)))]
    x2s = [dev_tensor(mp.X2), dev_tensor(W.to_bf16_bits(np.abs(W.normal((4096, 12288), 1.0, 82,
                                                                         2))))]
    ref = []
    for x1, x2 in zip(x1s, x2s):
        y1 = nv.linear(nv.quantize(x1), w1)
        y2 = nv.linear(nv.quantize(x2), w2)
        ref.append((y1.clone(), y2.clone()))
    q1, q2 = nv.quantize(x1s[0]), nv.quantize(x2s[0])
    y1 = torch.empty_like(ref[0][0])
    y2 = torch.empty_like(ref[0][1])
    outs = [(torch.empty_like(y1), torch.empty_like(y2)) for _ in range(2)]

    def step(i):
        nv.quantize(x1s[i], out=q1)
        nv.linear(q1, w1, out=y1)
        nv.quantize(x2s[i], out=q2)
        nv.linear(q2, w2, out=y2)
        outs[i][0].copy_(y1)
        outs[i][1].copy_(y2)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(0)
        step(1)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(0)
        step(1)
    for _ in range(2):
        for o in outs:
            o[0].zero_()
            o[1].zero_()
        g.replay()
        torch.cuda.synchronize()
        assert nv.sync_status() == 0
        for i in range(2):
            for k in range(2):
                assert torch.equal(outs[i][k].view(torch.int16), ref[i][k].view(torch.int16)), (i, k)
    del g


def test_decode_chain_in_cuda_graph_matches_eager():
    # back-to-back decode GEMVs (M 8 and M 1, N12288 K4096) with the resident-weights flag, as the
    # bench chains them: each call requests its first weight tiles before waiting for the
    # previous kernel; captured in a CUDA graph and replayed, they match the eager calls bit for
    # bit
    dc = W.decode(Ms=(1, 8))
    wd = dev_tensor(dc.W)
    qws = [nv.quantize(wd), nv.quantize((wd.float() * 0.5).to(torch.bfloat16)),
           nv.quantize((wd.float() * -1.5).to(torch.bfloat16))]
    qas = [nv.quantize(dev_tensor(dc.X[m])) for m in (8, 1)]
    calls = [(qas[i % 2], qws[i % 3]) for i in range(6)]
    ref = [nv.linear(a, w, resident_weights=True).clone() for a, w in calls]
    ys = [torch.empty_like(r) for r in ref]

    def chain():
        for (a, w), y in zip(calls, ys):
            nv.linear(a, w, out=y, resident_weights=True)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        chain()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain()
    for _ in range(3):
        for y in ys:
            y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert nv.sync_status() == 0
        for i, (y, r) in enumerate(zip(ys, ref)):
            assert torch.equal(y.view(torch.int16), r.view(torch.int16)), i
    del g


@pytest.mark.parametrize("offset", [0, 16])
def test_dequantize_full_weight(offset):
    # the MLP's 12288 x 3072 weight, as the bench times it: every warp of the grid takes several
    # grid-stride steps (2.36 M blocks), with the next step's loads in flight; fp32 and bf16,
    # into a 32-byte-aligned output (256-bit stores) and a 16-byte-aligned one (128-bit stores)
    xw = W.mlp_pair(M=8).W1
    rows, cols = xw.shape
    ref = O.quantize(xw)
    q = gpu_quantize(xw)
    assert_quant_equal(q, ref)
    stream = torch.cuda.current_stream().cuda_stream
    for out, esz, code in (("f32", 4, 0), ("bf16", 2, 1)):
        want = O.dequantize(ref, out).view(np.uint8).reshape(-1)
        buf = torch.zeros(rows * cols * esz + 64, dtype=torch.uint8, device="cuda")
        base = buf.data_ptr()
        base += (-base) % 32 + offset
        assert nv.nvfp4_dequantize(q.codes.data_ptr(), q.scales_lin.data_ptr(),
                                   q.global_scale.data_ptr(), rows, cols, code, base,
                                   stream) == 0
        torch.cuda.synchronize()
        start = base - buf.data_ptr()
        got = buf[start:start + rows * cols * esz].cpu().numpy()
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, f"{out}: {bad.size} bytes differ, first at {bad[0]}"
        del buf
