#!/usr/bin/env python
"""Benchmark of the NVFP4 quantized linear layer on B200.

One step = the hot path on the largest single-GPU workload, the diffusion-transformer MLP
pair at a 64x64 latent (4096 tokens, hidden 3072, MLP 12288): quantize the activations X1
(4096x3072 bf16, dynamic per-tensor amax) to NVFP4, GEMM1 Y1 = X1 . W1^T (N 12288, K 3072),
quantize the GELU-like activations X2 (4096x12288 bf16, dynamic amax), GEMM2
Y2 = X2 . W2^T (N 3072, K 12288); bf16 outputs. The weights (bf16 12288x3072 and 3072x12288)
are quantized to NVFP4 once, before timing, as a deployed layer keeps them.

The headline `value` is the step's throughput in TFLOP/s (2*M*N*K of both GEMMs per step
over the whole step, activation quantization included), summed over ranks. Each rank runs its
own independent batch (weak scaling, no collective on the data path). Inputs and outputs rotate
over enough buffer sets that every step reads its inputs cold from HBM and writes to buffers
the previous steps did not leave in L2 (more than 3x the L2 size in flight). Steps are replayed from CUDA graphs (one graph per rotation of the input sets).
Per-op durations come from CUDA events around graph loops of each op alone over the same
rotating inputs, on the launching stream (event nodes inside the step graph would break the
kernels' programmatic dependent launch and add ~15 us per step).

The other rows of the hot path (the double-quant attention projection step, the MLP GEMM with
the NVFP4-output epilogue, the small-M decode GEMV, p99.9 calibration, dequantize, the FP8
and low-rank layers) are measured after the timed region and reported under "rows".

`--impl reference` times the CPU oracle on a bounded sample of the same workload.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# the headline workload: the MLP pair
T, H, F = 4096, 3072, 12288
GEMM_FLOPS = 2.0 * T * F * H          # each of the two GEMMs
FLOPS = 2 * GEMM_FLOPS                # per step
WORKLOAD = "dit_mlp_pair_m4096_h3072_f12288"
# the double-quant attention projection (a row)
M, N, K = 4096, 3072, 3072
A_FLOPS = 2.0 * M * N * K
A_WORKLOAD = "attn_proj_fp8w_m4096_n3072_k3072"
LOWRANK_R = 128  # rank of the BF16 low-rank branch (FP4 layers with rank-128 BF16 branches)
METRIC = "NVFP4 GEMM TFLOPS & quantize GB/s at 1 B200 (fraction of FP4/HBM peak)"
FP4_PER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0  # nominal dense FP8 / BF16 ratio (4.5 / 2.25 PFLOP/s)
# the kernel the linear layer runs for M > 128 with a bf16 output (one 256 x 256 tile per CTA
# pair): the dominant kernel of the step (both GEMMs)
GEMM_KERNEL = "nvfp4_gemm_pair_kernel"
QBYTES_BF16 = 2 + 0.5 + 1 / 16        # quantize: read bf16, write codes and E4M3 scales


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", default=None, choices=sorted(PROFILE_CASES),
                    help="run one op of the hot path --reps times, untimed (for ncu), and exit")
    ap.add_argument("--reps", type=int, default=4)
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        self.gpu = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = time.time()

    def stop(self, t_lo, t_hi):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        self.out.flush()
        rows = []
        for line in open(self.out.name):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(f[1]), float(f[2]), f[3], f[5:9]))
            except ValueError:
                continue
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        inside = [r for r in rows if t_lo - 1.0 <= r[0] <= t_hi + 1.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[4])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

class AttnStep:
    """The double-quant attention projection step over several input sets: W (FP8 source)
    and X (bf16, dynamic amax) quantized in one launch, then the GEMM. Each set has its own
    inputs and its own outputs (quantized W and X, Y)."""

    def __init__(self, nv, wl, n_sets, dev):
        self.nv = nv
        w8 = torch.from_numpy(wl.W_e4m3).to(dev)
        xb = torch.from_numpy(wl.X_bf16.view(np.int16)).to(dev).view(torch.bfloat16)
        s8 = torch.tensor([wl.w_scale], dtype=torch.float32, device=dev)
        self.W = [w8.clone() for _ in range(n_sets)]
        self.X = [xb.clone() for _ in range(n_sets)]
        self.s8 = s8
        self.QW = [nv.quantize_fp8(w, s8) for w in self.W]
        self.QX = [nv.quantize(x) for x in self.X]
        self.Y = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(n_sets)]

    def run(self, i):
        nv = self.nv
        nv.quantize_batch([{"x": self.W[i], "fp8_scale": self.s8, "out": self.QW[i]},
                           {"x": self.X[i], "out": self.QX[i]}])
        nv.linear(self.QX[i], self.QW[i], out=self.Y[i])


def bf16_dev(a, dev):
    return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)


def clone_q(nv, q):
    return nv.NVFP4Tensor(q.codes.clone(), q.scales_swz.clone(), None, q.global_scale.clone(),
                          q.rows, q.cols)


class MlpStep:
    """The MLP pair over several input sets: quantize X1, GEMM1, quantize X2, GEMM2. Each set
    holds its own X1, X2, its own copy of the quantized weights and its own outputs (quantized
    activations, Y1, Y2), so every step reads all of its operands from HBM and writes to
    buffers that the previous steps did not leave in L2."""

    def __init__(self, nv, mp, n_sets, dev):
        self.nv = nv
        x1, x2 = bf16_dev(mp.X1, dev), bf16_dev(mp.X2, dev)
        q1, q2 = nv.quantize(bf16_dev(mp.W1, dev)), nv.quantize(bf16_dev(mp.W2, dev))
        self.X1 = [x1.clone() for _ in range(n_sets)]
        self.X2 = [x2.clone() for _ in range(n_sets)]
        self.Q1 = [clone_q(nv, q1) for _ in range(n_sets)]
        self.Q2 = [clone_q(nv, q2) for _ in range(n_sets)]
        del x1, x2, q1, q2
        self.QX1 = [nv.quantize(x) for x in self.X1]
        self.QX2 = [nv.quantize(x) for x in self.X2]
        self.Y1 = [torch.empty((T, F), dtype=torch.bfloat16, device=dev) for _ in range(n_sets)]
        self.Y2 = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(n_sets)]
        wq = lambda q: q.codes.numel() + q.scales_swz.numel()
        self.set_bytes = ((self.X1[0].numel() + self.X2[0].numel()) * 2 + wq(self.Q1[0]) +
                          wq(self.Q2[0]) + wq(self.QX1[0]) + wq(self.QX2[0]) +
                          (self.Y1[0].numel() + self.Y2[0].numel()) * 2)

    def quantize1(self, i, x=None):
        self.nv.quantize(self.X1[i] if x is None else x, out=self.QX1[i])

    def gemm1(self, i):
        self.nv.linear(self.QX1[i], self.Q1[i], out=self.Y1[i])

    def quantize2(self, i, x=None):
        self.nv.quantize(self.X2[i] if x is None else x, out=self.QX2[i])

    def gemm2(self, i, y=None):
        self.nv.linear(self.QX2[i], self.Q2[i], out=self.Y2[i] if y is None else y)

    def run(self, i):
        self.quantize1(i)
        self.gemm1(i)
        self.quantize2(i)
        self.gemm2(i)


def quantize_launches(nv, nbytes):
    """Kernel launches of one dynamic-amax quantize of a tensor of nbytes: one from 16 MB up
    (the single-pass kernel, or the streamed one beyond shared memory), two (amax, encode)
    below."""
    return 1 if nbytes >= (16 << 20) else 2


def graph_kernel_nodes(fns):
    """Kernel launches of one pass of fns, counted as the kernel nodes of a CUDA graph that
    captures it; None if the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for f in fns:
                f()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            for f in fns:
                f()
        h = rt.cudaGraph_t(init_value=int(g.raw_cuda_graph()))
        err, _, n = rt.cudaGraphGetNodes(h, 0)
        err2, nodes, n = rt.cudaGraphGetNodes(h, n)
        if err != rt.cudaError_t.cudaSuccess or err2 != rt.cudaError_t.cudaSuccess:
            return None
        kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
        count = sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)
        del g
        return count
    except Exception:  # an older torch or cuda-python: the caller falls back to its rule
        return None


def launches_per_step(nv, st=None):
    """Kernel launches of one MLP step: counted in a captured graph of the step when possible,
    else by rule (quantize: quantize_launches; linear: one launch, two when it needs workspace,
    i.e. runs a split-K reduction)."""
    if st is not None:
        n = graph_kernel_nodes([lambda: st.run(0)])
        if n is not None:
            return n
    L = nv.load()
    gemm = lambda m, n, k: 2 if L.nvfp4_workspace_bytes(nv.NVFP4_OP_LINEAR, m, n, k) > 0 else 1
    return (quantize_launches(nv, T * H * 2) + gemm(T, F, H) +
            quantize_launches(nv, T * F * 2) + gemm(T, H, F))


def capture(fns):
    """One CUDA graph that runs every closure in fns in order (warmed up on a side stream)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for f in fns:
            f()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    return g


def replay_ms(graphs, stream):
    """Replay graphs in order; device time between events on the launching stream."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for g in graphs:
        g.replay()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


def op_timer(fns, reps=3):
    """Average device time of one call, over graphs that run every closure in fns (each on
    its own buffer set, so inputs come from HBM), replayed `reps` times."""
    g = capture(fns)
    g.replay()
    torch.cuda.synchronize()
    ms = replay_ms([g] * reps, torch.cuda.current_stream())
    del g
    us = ms * 1e3 / (reps * len(fns))
    return us / 1e3, us / 1e3


def small_m_rows(nv, W, dev, hbm, Ms=(1, 8, 32, 128)):
    """Small-M decode: W 12288x4096 packed (rotating copies larger than L2), per M: back-to-back
    linears (plain), the same with the resident-weights flag (each call starts reading W while
    the previous one finishes), a decode layer that quantizes the activations (dynamic amax)
    then runs the linear, and the same layer in one call (fused for M <= 16)."""
    L2 = torch.cuda.get_device_properties(dev).L2_cache_size
    dc = W.decode(Ms=Ms)
    Wd = bf16_dev(dc.W, dev)
    wbytes = 12288 * 4096 // 2 + 12288 * 4096 // 16
    n_w = max(2, math.ceil(3 * L2 / wbytes))
    qws = [nv.quantize(Wd) for _ in range(n_w)]
    small = {}
    for m, xa in dc.X.items():
        xd = bf16_dev(xa, dev)
        qa = nv.quantize(xd)
        y = torch.empty((m, 12288), dtype=torch.bfloat16, device=dev)
        row = {}
        for key, fns in [
                ("plain", [lambda q=q: nv.linear(qa, q, out=y) for q in qws]),
                ("resident", [lambda q=q: nv.linear(qa, q, out=y, resident_weights=True)
                              for q in qws]),
                ("quantize_x_then_linear", [lambda q=q: (nv.quantize(xd, out=qa),
                                                         nv.linear(qa, q, out=y,
                                                                   resident_weights=True))
                                            for q in qws]),
                ("linear_dynamic", [lambda q=q: nv.linear_dynamic(xd, q, out=y,
                                                                  resident_weights=True)
                                    for q in qws])]:
            avg, med = op_timer(fns)
            gbs = wbytes / (avg * 1e-3) / 1e9
            row[key] = {"us": avg * 1e3, "GB/s_weights": gbs, "frac_hbm": gbs / hbm,
                        "TFLOP/s": 2.0 * m * 12288 * 4096 / (avg * 1e-3) / 1e12}
        small[f"M{m}"] = row
    del qws, Wd
    torch.cuda.empty_cache()
    return small


def extras(nv, W, dev, hbm, fp4_peak, mlp):
    """The other hot-path rows: the attention projection step, the MLP GEMM with the
    NVFP4-output epilogue, small-M decode, calibration, dequantize, FP8 and low-rank layers."""
    rows = {}
    L2 = torch.cuda.get_device_properties(dev).L2_cache_size

    def sets_for(nbytes):
        return max(2, math.ceil(3 * L2 / max(nbytes, 1)))

    t = lambda a: bf16_dev(a, dev)

    # --- the double-quant attention projection: W from FP8 and X in one quantize launch, then
    #     the GEMM, as one step; and each op alone
    wl = W.attn_proj()
    n_a = max(3, math.ceil(3 * L2 / (wl.W_e4m3.nbytes + wl.X_bf16.nbytes)))
    st = AttnStep(nv, wl, n_a, dev)
    step_ms, _ = op_timer([lambda i=i: st.run(i) for i in range(n_a)])
    qw_ms, _ = op_timer([lambda i=i: nv.quantize_fp8(st.W[i], st.s8, out=st.QW[i])
                         for i in range(n_a)])
    qx_ms, _ = op_timer([lambda i=i: nv.quantize(st.X[i], out=st.QX[i]) for i in range(n_a)])
    qb_ms, _ = op_timer([lambda i=i: nv.quantize_batch([{"x": st.W[i], "fp8_scale": st.s8,
                                                         "out": st.QW[i]},
                                                        {"x": st.X[i], "out": st.QX[i]}])
                         for i in range(n_a)])
    g_ms, _ = op_timer([lambda i=i: nv.linear(st.QX[i], st.QW[i], out=st.Y[i])
                        for i in range(n_a)])
    qx_bytes = M * K * QBYTES_BF16 + 4
    qw_bytes = N * K * (1 + 0.5 + 1 / 16) + 4
    g_tf = A_FLOPS / (g_ms * 1e-3) / 1e12
    rows[A_WORKLOAD] = {
        "step_us": step_ms * 1e3, "step_TFLOP/s": A_FLOPS / (step_ms * 1e-3) / 1e12,
        "gemm_us": g_ms * 1e3, "gemm_TFLOP/s": g_tf, "gemm_frac_fp4": g_tf / fp4_peak,
        "quantize_w_fp8_us": qw_ms * 1e3, "quantize_x_bf16_us": qx_ms * 1e3,
        "quantize_batch_w_x_us": qb_ms * 1e3,
        "quantize_x_GB/s": qx_bytes / (qx_ms * 1e-3) / 1e9,
        "quantize_x_frac_hbm": qx_bytes / (qx_ms * 1e-3) / 1e9 / hbm,
        "quantize_batch_GB/s": (qx_bytes + qw_bytes) / (qb_ms * 1e-3) / 1e9,
        "quantize_batch_frac_hbm": (qx_bytes + qw_bytes) / (qb_ms * 1e-3) / 1e9 / hbm}
    del st
    torch.cuda.empty_cache()

    # --- the MLP's GEMM1 writing GEMM2's NVFP4 operand from its epilogue (static amax of the
    #     activation), against GEMM1 in bf16 followed by the static-scale quantize
    amax = torch.tensor([float(mlp.X2[0].float().abs().max())], device=dev)
    n_m = len(mlp.X1)
    sets = list(zip(mlp.QX1, mlp.Q1))
    for i in range(n_m):
        mlp.quantize1(i)
    outs = [nv.linear_nvfp4_out(p[0], p[1], amax) for p in sets]
    row = {}
    for act in ("identity", "gelu_tanh"):
        avg_f, _ = op_timer([lambda p=p, o=o: nv.linear_nvfp4_out(p[0], p[1], amax, act, out=o)
                             for p, o in zip(sets, outs)])
        row[f"nvfp4_out_{act}_us"] = avg_f * 1e3
    avg_q, _ = op_timer([lambda i=i: nv.quantize(mlp.X2[i], static_amax=amax, out=mlp.QX2[i])
                         for i in range(n_m)])
    row["quantize_x2_static_us"] = avg_q * 1e3
    rows["gemm1_m4096_n12288_k3072_nvfp4_out"] = row
    del outs, sets
    torch.cuda.empty_cache()

    # --- small-M decode: W 12288x4096 packed, M in {1, 8, 32, 128}
    rows["small_m_n12288_k4096"] = small_m_rows(nv, W, dev, hbm)

    # --- p99.9 calibration over 53 batches of 4096x3072 bf16 (8 distinct seeded batches,
    #     each read several times; 8 x 25 MB exceeds L2, so every read comes from HBM)
    distinct = [t(W.calib_batch(b)) for b in range(8)]
    batches = [distinct[b % 8] for b in range(53)]
    avg, med = op_timer([lambda: nv.calib_percentile_amax(batches)], reps=5)
    nbytes = 53 * 4096 * 3072 * 2
    gbs = nbytes / (avg * 1e-3) / 1e9
    rows["calib_p999_53x4096x3072_bf16"] = {"us": avg * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm}
    # static input scales from the p99.9 percentile and from the max over the batches, each used
    # to quantize an evaluation batch (the 54th draw) for the GEMM against a 3072x3072 NVFP4
    # weight; error of Y against the fp64 dense product of the unquantized operands on every
    # 64th row
    pct, mx = nv.calib_percentile_amax(batches)
    pct, mx = float(pct.cpu()[0]), float(mx.cpu()[0])
    ev_host, wt_host = W.calib_batch(53), W.calib_weight()
    ev, wt = t(ev_host), t(wt_host)
    qwt = nv.quantize(wt)
    sel = np.arange(0, 4096, 64)
    dense = (W.bf16_bits_to_f32(ev_host)[sel].astype(np.float64)
             @ W.bf16_bits_to_f32(wt_host).astype(np.float64).T)
    cal = {"p999": pct, "max": mx, "p999_over_max": pct / mx, "max_over_p999": mx / pct,
           "batches": "8 distinct seeded batches, each counted 53/8 times"}
    for name, amax in (("p999", pct), ("max", mx)):
        qa = nv.quantize(ev, static_amax=torch.tensor([amax], device=dev))
        y = nv.linear(qa, qwt, out_dtype=torch.float32)[sel].double().cpu().numpy()
        cal[f"rel_err_{name}"] = float(np.linalg.norm(y - dense) / np.linalg.norm(dense))
    rows["calib_p999_53x4096x3072_bf16"]["static_scales"] = cal
    del distinct, batches, ev, wt, qwt

    # --- dequantize 12288x3072 to bf16
    w1 = nv.quantize(t(W.mlp_pair(M=8).W1), linear=True)
    wqs = [nv.NVFP4Tensor(w1.codes.clone(), None, w1.scales_lin.clone(), w1.global_scale,
                          w1.rows, w1.cols) for _ in range(3)]
    # the outputs rotate too (3 x 75.5 MB > L2): every call's writes must reach HBM
    douts = [torch.empty((w1.rows, w1.cols), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    avg, med = op_timer([lambda q=q, o=o: nv.dequantize(q, torch.bfloat16, out=o)
                         for q, o in zip(wqs, douts)])
    elems = 12288 * 3072
    gbs = (elems / 2 + elems / 16 + elems * 2) / (avg * 1e-3) / 1e9
    rows["dequantize_12288x3072_bf16"] = {"us": avg * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm}
    del wqs, w1, douts
    torch.cuda.empty_cache()

    # --- FP8 E4M3 tensorwise W8A8 layers (embed / lm_head path): quantize X, GEMM, both
    fp8_peak = fp4_peak / FP4_PER_BF16 * FP8_PER_BF16
    gen = torch.Generator(device=dev)
    gen.manual_seed(8)
    fp8 = {}
    for name, mm, nn, kk in [("m4096_n3072_k3072", 4096, 3072, 3072),
                             ("m4096_n12288_k3072", 4096, 12288, 3072),
                             ("m4096_n3072_k12288", 4096, 3072, 12288)]:
        nset = sets_for(mm * kk * 2)
        xs = [torch.randn(mm, kk, device=dev, generator=gen).to(torch.bfloat16)
              for _ in range(nset)]
        w8 = nv.quantize_e4m3((torch.randn(nn, kk, device=dev, generator=gen) * 0.02)
                              .to(torch.bfloat16))
        nsw = sets_for(mm * kk + nn * kk)
        a8s = [nv.quantize_e4m3(xs[i % nset]) for i in range(nsw)]
        w8s = [nv.E4M3Tensor(w8.codes.clone(), w8.scale.clone()) for _ in range(nsw)]
        ys = [torch.empty((mm, nn), dtype=torch.bfloat16, device=dev) for _ in range(nsw)]
        avg_q, _ = op_timer([lambda x=x, a=a8s[i % nsw]: nv.quantize_e4m3(x, out=a)
                             for i, x in enumerate(xs)])
        avg_g, _ = op_timer([lambda a=a, w=w, y=y: nv.linear_e4m3(a, w, out=y)
                             for a, w, y in zip(a8s, w8s, ys)])
        avg_l, _ = op_timer([lambda x=x, a=a8s[i], w=w8s[i], y=ys[i]:
                             (nv.quantize_e4m3(x, out=a), nv.linear_e4m3(a, w, out=y))
                             for i, x in enumerate(xs[:nsw] if nsw <= nset else xs)])
        qgbs = mm * kk * 3 / (avg_q * 1e-3) / 1e9
        tf = 2.0 * mm * nn * kk / (avg_g * 1e-3) / 1e12
        fp8[name] = {"quantize_x_us": avg_q * 1e3, "quantize_x_GB/s": qgbs,
                     "quantize_x_frac_hbm": qgbs / hbm, "gemm_us": avg_g * 1e3,
                     "gemm_TFLOP/s": tf, "gemm_frac_fp8": tf / fp8_peak,
                     "quantize_x_then_gemm_us": avg_l * 1e3}
        del xs, a8s, w8s, w8, ys
        torch.cuda.empty_cache()
    rows["fp8_e4m3_w8a8"] = fp8

    # --- FP4 linear with a BF16 rank-128 branch on the attention projection (4096x3072x3072):
    #     the down projection of the bf16 input plus the GEMM with the low-rank k-tiles,
    #     against the plain FP4 linear on the same operands
    wl = W.attn_proj()
    xb = t(wl.X_bf16)
    d_bits, u_bits = W.lowrank_factors(N=N, K=K, r=LOWRANK_R)
    dd, uu = t(d_bits), t(u_bits)
    qw0 = nv.quantize_fp8(torch.from_numpy(wl.W_e4m3).to(dev),
                          torch.tensor([wl.w_scale], dtype=torch.float32, device=dev))
    nset = sets_for(M * K * 2 + N * K // 2)
    xs = [xb.clone() for _ in range(nset)]
    qxs = [nv.quantize(x) for x in xs]
    qws = [clone_q(nv, qw0) for _ in range(nset)]
    ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(nset)]
    avg_p, _ = op_timer([lambda a=a, w=w, y=y: nv.linear(a, w, out=y)
                         for a, w, y in zip(qxs, qws, ys)])
    avg_l, _ = op_timer([lambda a=a, w=w, x=x, y=y: nv.linear_lowrank(a, w, x, dd, uu, out=y)
                         for a, w, x, y in zip(qxs, qws, xs, ys)])
    flops = 2.0 * M * N * K + 2.0 * M * K * LOWRANK_R + 2.0 * M * N * LOWRANK_R
    rows[f"lowrank_r{LOWRANK_R}_m{M}_n{N}_k{K}"] = {
        "linear_us": avg_p * 1e3, "linear_lowrank_us": avg_l * 1e3,
        "branch_extra_us": (avg_l - avg_p) * 1e3,
        "TFLOP/s": flops / (avg_l * 1e-3) / 1e12}
    del xs, qxs, qws, ys, xb, dd, uu, qw0
    torch.cuda.empty_cache()
    return rows


def oracle_threads():
    """Threads the OpenMP oracle runs on: OMP_NUM_THREADS when set, else the CPUs this
    process may run on (libgomp's default), not the machine's total."""
    n = os.environ.get("OMP_NUM_THREADS", "").split(",")[0].strip()
    if n.isdigit() and int(n) > 0:
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_sample(O, W):
    """A bounded sample of the MLP step for the CPU oracle: the weights quantized once (as the
    GPU step keeps them); per call, quantize X1 rows 0..63 and X2 rows 0..15 with their
    whole-tensor amax, and compute Y1[0:64, 0:512] and Y2[0:16, 0:512] in fp64. Returns (one
    call, its GEMM flops, a description)."""
    mp = W.mlp_pair()
    m1, m2, n1 = 64, 16, 512
    amax1 = float(np.abs(W.bf16_bits_to_f32(mp.X1)).max())
    amax2 = float(np.abs(W.bf16_bits_to_f32(mp.X2)).max())
    qw1 = O.quantize(mp.W1[:n1])
    qw2 = O.quantize(mp.W2[:n1])
    x1, x2 = mp.X1[:m1].copy(), mp.X2[:m2].copy()

    def call():
        O.gemm(O.quantize(x1, amax=amax1), qw1)
        O.gemm(O.quantize(x2, amax=amax2), qw2)

    flops = 2.0 * m1 * n1 * H + 2.0 * m2 * n1 * F
    desc = (f"quantize X1[0:{m1}] and X2[0:{m2}] (whole-tensor amax), Y1[0:{m1},0:{n1}] "
            f"(K {H}) and Y2[0:{m2},0:{n1}] (K {F}) in fp64; weight rows 0..{n1 - 1} "
            "quantized once")
    return call, flops, desc


def cpu_baseline(seconds=10.0):
    """The oracle, as it stands, on a bounded sample of the step (oracle_sample), repeated for
    about `seconds`; TFLOP/s of the sample's GEMM part over the whole sample time."""
    import oracle as O
    from nvfp4_block_scaled_14_b200 import workloads as W
    call, flops, desc = oracle_sample(O, W)
    reps, t0 = 0, time.time()
    while True:
        call()
        reps += 1
        if time.time() - t0 >= seconds:
            break
    dt = (time.time() - t0) / reps
    cores = oracle_threads()
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{desc}; {reps} repetitions, {dt:.3f} s each"}


def e2e_pipelined_ms(st, x1_host, x2_host, steps):
    """Device time per step with every step's inputs (X1, X2) copied in from pinned host
    memory and its output Y2 copied back, overlapped across steps as a serving loop would run
    them: step i+1's inputs upload on one stream while step i computes on a second and step
    i-1's output downloads on a third (two device slots for inputs and outputs, events between
    them)."""
    nslot = 2
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    yd = [torch.empty_like(st.Y2[0]) for _ in range(nslot)]
    yh = [torch.empty((T, H), dtype=torch.int16).pin_memory() for _ in range(nslot)]
    ev_in = [torch.cuda.Event() for _ in range(nslot)]
    ev_comp = [torch.cuda.Event() for _ in range(nslot)]
    ev_out = [torch.cuda.Event() for _ in range(nslot)]

    def one(i):
        k = i % nslot
        if i >= nslot:
            s_in.wait_event(ev_comp[k])  # step i-2 has finished reading slot k's inputs
        with torch.cuda.stream(s_in):
            st.X1[k].view(torch.int16).copy_(x1_host, non_blocking=True)
            st.X2[k].view(torch.int16).copy_(x2_host, non_blocking=True)
        ev_in[k].record(s_in)
        s_comp.wait_event(ev_in[k])
        if i >= nslot:
            s_comp.wait_event(ev_out[k])  # step i-2's output has left slot k
        with torch.cuda.stream(s_comp):
            st.quantize1(k)
            st.gemm1(k)
            st.quantize2(k)
            st.gemm2(k, yd[k])
        ev_comp[k].record(s_comp)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            yh[k].copy_(yd[k].view(torch.int16), non_blocking=True)
        ev_out[k].record(s_out)

    for i in range(2 * nslot):  # warm-up, untimed
        one(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        one(i)
    s_in.wait_stream(s_comp)
    s_in.wait_stream(s_out)
    end.record(s_in)
    end.synchronize()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps


def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks (every rank gets it); x itself without a process group."""
    if dist is None:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, ms_per_step: float, flops_per_rank_step: float) -> float:
    """Whole-job throughput: every rank runs its own step on its own inputs (weak scaling), so
    the job does world x the work of one rank in the slowest rank's time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    import nvfp4_block_scaled_14_b200 as nv
    from nvfp4_block_scaled_14_b200 import workloads as W
    nv.load()
    hbm, bf16, peak_kind = peaks()
    fp4_peak = bf16 * FP4_PER_BF16

    # every rank its own activations (its own seed), the same weights
    mp = W.mlp_pair(x_tensor=3 + 100 * rank)
    L2 = torch.cuda.get_device_properties(dev).L2_cache_size
    act_bytes = (mp.X1.nbytes + mp.X2.nbytes)
    n_sets = max(3, math.ceil(3 * L2 / act_bytes))
    st = MlpStep(nv, mp, n_sets, dev)

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        st.run(i % n_sets)
    torch.cuda.synchronize()

    # one graph per rotation of the input sets (n_sets steps, no nodes between the ops),
    # plus one for the remaining steps, so exactly args.steps steps are replayed
    full = capture([lambda i=i: st.run(i) for i in range(n_sets)])
    rem = args.steps % n_sets
    part = capture([lambda i=i: st.run(i) for i in range(rem)]) if rem else None
    plan = [full] * (args.steps // n_sets) + ([part] if part is not None else [])
    for _ in range(max(1, args.warmup // n_sets)):
        full.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_lo = time.time()
    ms = replay_ms(plan, stream)
    t_hi = time.time()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop(t_lo, t_hi)
    del plan, full, part

    # per-op device durations: each op alone, over the rotating input sets
    for i in range(n_sets):
        st.quantize1(i)
    q1_ms, _ = op_timer([lambda i=i: st.quantize1(i) for i in range(n_sets)])
    g1_ms, _ = op_timer([lambda i=i: st.gemm1(i) for i in range(n_sets)])
    q2_ms, _ = op_timer([lambda i=i: st.quantize2(i) for i in range(n_sets)])
    g2_ms, _ = op_timer([lambda i=i: st.gemm2(i) for i in range(n_sets)])

    ms_max = max_over_ranks(ms, dist, dev)

    # e2e: host inputs in pinned memory, copies inside the timed region
    e2e_steps = max(3, min(args.steps, 30))
    x1_host = torch.from_numpy(mp.X1.view(np.int16)).pin_memory()
    x2_host = torch.from_numpy(mp.X2.view(np.int16)).pin_memory()
    y_host = torch.empty((T, H), dtype=torch.int16).pin_memory()

    def e2e_serial_step():
        st.X1[0].view(torch.int16).copy_(x1_host, non_blocking=True)
        st.X2[0].view(torch.int16).copy_(x2_host, non_blocking=True)
        st.run(0)
        y_host.copy_(st.Y2[0].view(torch.int16), non_blocking=True)

    for _ in range(2):
        e2e_serial_step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(e2e_steps):
        e2e_serial_step()
    b.record()
    b.synchronize()
    e2e_serial_ms = a.elapsed_time(b) / e2e_steps
    e2e_mode = "overlapped: step i+1 uploads and step i-1 downloads while step i computes"
    try:
        e2e_local = e2e_pipelined_ms(st, x1_host, x2_host, e2e_steps)
    except Exception as exc:  # measured serially instead; the line says which
        print(f"e2e pipelined measurement failed ({exc}); serial copies reported",
              file=sys.stderr)
        e2e_local, e2e_mode = e2e_serial_ms, "serial: upload, compute, download per step"
    e2e_ms = max_over_ranks(e2e_local, dist, dev)
    e2e_serial_ms = max_over_ranks(e2e_serial_ms, dist, dev)

    rows, small = None, None
    if rank == 0:
        if not args.no_extras:
            rows = extras(nv, W, dev, hbm, fp4_peak, st)
            small = rows["small_m_n12288_k4096"]
        else:
            small = small_m_rows(nv, W, dev, hbm, Ms=(8,))

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    ms_step = ms_max / args.steps
    value = job_tflops(world, ms_step, FLOPS)
    g1_tf = GEMM_FLOPS / (g1_ms * 1e-3) / 1e12
    g2_tf = GEMM_FLOPS / (g2_ms * 1e-3) / 1e12
    gemm_avg_ms = (g1_ms + g2_ms) / 2
    gemm_tf = GEMM_FLOPS / (gemm_avg_ms * 1e-3) / 1e12
    qb1, qb2 = T * H * QBYTES_BF16 + 4, T * F * QBYTES_BF16 + 4
    q1_gbs, q2_gbs = qb1 / (q1_ms * 1e-3) / 1e9, qb2 / (q2_ms * 1e-3) / 1e9
    traffic = None
    tp = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if os.path.exists(tp):
        traffic = json.load(open(tp)).get(GEMM_KERNEL, {}).get(WORKLOAD)
    m8 = small["M8"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp4-e2m1",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": T, "hidden": H, "mlp": F,
                   "gemm1": {"M": T, "N": F, "K": H}, "gemm2": {"M": T, "N": H, "K": F},
                   "weights": "bf16 -> nvfp4 once, before timing",
                   "activations": "bf16, dynamic per-tensor amax, quantized every step",
                   "out": "bf16",
                   "l2": f"inputs and outputs rotate over {n_sets} buffer sets "
                         f"({n_sets * st.set_bytes / 1e6:.0f} MB > 3x L2)",
                   "parallelism": f"{world} independent ranks"},
        "gemm_tflops": {"gemm1": g1_tf, "gemm2": g2_tf},
        "quantize_gbs": {"x1_bf16_4096x3072": q1_gbs, "x2_bf16_4096x12288": q2_gbs},
        "op_us": {"quantize_x1": q1_ms * 1e3, "gemm1": g1_ms * 1e3,
                  "quantize_x2": q2_ms * 1e3, "gemm2": g2_ms * 1e3},
        "roofline": {"bound": "tensor", "kernel": GEMM_KERNEL,
                     "achieved": gemm_tf, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_tf / fp4_peak, "traffic": traffic,
                     "per_launch": "2*4096*12288*3072 flops (both GEMMs) over the mean of the "
                                   "two GEMMs' durations",
                     "peak_note": f"{peak_kind} bf16 burst {bf16} TFLOP/s x {FP4_PER_BF16} "
                                  "(nominal FP4/BF16 ratio)"},
        "roofline_quantize": {
            "bound": "hbm", "unit": "GB/s", "peak": hbm, "peak_note": f"{peak_kind} HBM copy",
            "x1_bf16_4096x3072": {"achieved": q1_gbs, "frac": q1_gbs / hbm, "us": q1_ms * 1e3,
                                  "kernel": "fused_quantize_kernel"},
            "x2_bf16_4096x12288": {"achieved": q2_gbs, "frac": q2_gbs / hbm, "us": q2_ms * 1e3,
                                   "kernel": "stream_quantize_kernel"},
            "bytes": "read 2 B + write 0.5 + 1/16 B per value"},
        # decode: the weights are quantized ahead of time, so the chain of GEMVs runs with the
        # resident-weights flag (each call starts reading its W while the previous call ends);
        # "plain" is the same chain without the flag
        "roofline_small_m": {
            "bound": "hbm", "unit": "GB/s", "peak": hbm, "kernel": "nvfp4_gemm_smallm_kernel",
            "workload": "decode M8 N12288 K4096 (packed weights + scales 28.3 MB), back-to-back "
                        "calls over rotating weights quantized ahead of time",
            "achieved": m8["resident"]["GB/s_weights"], "frac": m8["resident"]["frac_hbm"],
            "us": m8["resident"]["us"], "flags": "NVFP4_LINEAR_RESIDENT_WEIGHTS",
            "plain": {"achieved": m8["plain"]["GB/s_weights"], "frac": m8["plain"]["frac_hbm"],
                      "us": m8["plain"]["us"]}},
        "e2e": {"value": job_tflops(world, e2e_ms, FLOPS), "unit": "TFLOP/s",
                "copies": e2e_mode,
                "serial_value": job_tflops(world, e2e_serial_ms, FLOPS),
                "h2d_bytes_per_step": int(mp.X1.nbytes + mp.X2.nbytes),
                "d2h_bytes_per_step": int(T * H * 2)},
        "gpu_launches": launches_per_step(nv, st) * args.steps,
        "clocks": clk,
    }
    if rows is not None:
        line["rows"] = rows
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


def run_reference(args):
    """The CPU oracle as it stands on a bounded sample of the same workload per step."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle as O
    from nvfp4_block_scaled_14_b200 import workloads as W
    call, flops, desc = oracle_sample(O, W)
    for _ in range(args.warmup):
        call()
    t0 = time.time()
    for _ in range(args.steps):
        call()
    dt = (time.time() - t0) / args.steps
    value = flops / dt / 1e12
    cores = oracle_threads()
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": T, "hidden": H, "mlp": F},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def profile_case(name, reps):
    """One op of the hot path on its workload, run `reps` times over rotating inputs, without
    timing: the program ncu captures. Inputs are a few hundred MB at most."""
    import nvfp4_block_scaled_14_b200 as nv
    from nvfp4_block_scaled_14_b200 import workloads as W
    dev = torch.device("cuda", 0)
    nv.load()
    if name in ("mlp_step", "quantize_x1", "quantize_x2", "gemm1", "gemm2", "nvfp4_out_gelu",
                "nvfp4_out_identity"):
        # one input set (~170 MB on the device): ncu saves and restores device memory around
        # each replay pass of a captured launch, so the case keeps it small
        st = MlpStep(nv, W.mlp_pair(), 1, dev)
        amax = torch.tensor([float(st.X2[0].float().abs().max())], device=dev)
        outs = [nv.linear_nvfp4_out(st.QX1[0], st.Q1[0], amax)] \
            if name.startswith("nvfp4_out") else None
        st.quantize1(0)
        st.quantize2(0)
        torch.cuda.synchronize()
        # the GEMM cases launch only their own GEMM (after the operands' quantize above)
        op3 = {"mlp_step": st.run, "quantize_x1": st.quantize1, "gemm1": st.gemm1,
              "quantize_x2": st.quantize2, "gemm2": st.gemm2,
              "nvfp4_out_gelu": lambda i: nv.linear_nvfp4_out(st.QX1[0], st.Q1[i], amax,
                                                              "gelu_tanh", out=outs[i]),
              "nvfp4_out_identity": lambda i: nv.linear_nvfp4_out(st.QX1[0], st.Q1[i], amax,
                                                                  "identity", out=outs[i])}[name]
        op = lambda i: op3(0)
    elif name in ("smallm_m8", "smallm_m8_resident", "linear_dynamic_m8"):
        dc = W.decode(Ms=(8,))
        wd = bf16_dev(dc.W, dev)
        qws = [nv.quantize(wd) for _ in range(6)]
        xd = bf16_dev(dc.X[8], dev)
        qa = nv.quantize(xd)
        y = torch.empty((8, 12288), dtype=torch.bfloat16, device=dev)
        op = {"smallm_m8": lambda i: nv.linear(qa, qws[i % 6], out=y),
              "smallm_m8_resident": lambda i: nv.linear(qa, qws[i % 6], out=y,
                                                        resident_weights=True),
              "linear_dynamic_m8": lambda i: nv.linear_dynamic(xd, qws[i % 6], out=y,
                                                               resident_weights=True)}[name]
    elif name == "calib":
        distinct = [bf16_dev(W.calib_batch(b), dev) for b in range(8)]
        batches = [distinct[b % 8] for b in range(53)]
        op = lambda i: nv.calib_percentile_amax(batches)
    elif name in ("attn_step", "lowrank"):
        wl = W.attn_proj()
        if name == "attn_step":
            st = AttnStep(nv, wl, 3, dev)
            op = lambda i: st.run(i % 3)
        else:
            xb = bf16_dev(wl.X_bf16, dev)
            d_bits, u_bits = W.lowrank_factors(N=N, K=K, r=LOWRANK_R)
            dd, uu = bf16_dev(d_bits, dev), bf16_dev(u_bits, dev)
            qw = nv.quantize_fp8(torch.from_numpy(wl.W_e4m3).to(dev),
                                 torch.tensor([wl.w_scale], dtype=torch.float32, device=dev))
            xs = [xb.clone() for _ in range(3)]
            qxs = [nv.quantize(x) for x in xs]
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            op = lambda i: nv.linear_lowrank(qxs[i % 3], qw, xs[i % 3], dd, uu, out=y)
    else:
        raise ValueError(name)
    for i in range(reps):
        op(i)
    torch.cuda.synchronize()
    assert nv.sync_status() == 0


PROFILE_CASES = ("mlp_step", "quantize_x1", "quantize_x2", "gemm1", "gemm2", "nvfp4_out_gelu",
                 "nvfp4_out_identity", "smallm_m8", "smallm_m8_resident", "linear_dynamic_m8",
                 "calib", "attn_step", "lowrank")


def main():
    args = parse()
    if args.profile_case:
        profile_case(args.profile_case, args.reps)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
