// api.cu -- the C ABI declared in include/nvfp4.h: argument checks (on the host, before any
// launch), workspace sizing, dispatch to the kernels, status mapping.
#include <cstdio>
#include <cstring>
#include <mutex>
#include <thread>
#include <unordered_map>

#include "grid_exchange.cuh"
#include "nvfp4_internal.cuh"

namespace nvfp4 {

// Library status word (one per device). Kernels whose bounded waits give up write
// NVFP4_ERR_TIMEOUT here; nvfp4_sync_status reads and clears it.
__device__ int g_device_status;

namespace {
constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];
int *g_status_ptr[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

int current_device()
{
    int d = 0;
    cudaGetDevice(&d);
    return d < 0 ? 0 : (d >= kMaxDevices ? kMaxDevices - 1 : d);
}

void init_device(int d)
{
    std::call_once(g_dev_once[d], [d]() {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d);
        g_sms[d] = v > 0 ? v : 1;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) == cudaSuccess)
            g_status_ptr[d] = reinterpret_cast<int *>(p);
    });
}
} // namespace

int num_sms()
{
    const int d = current_device();
    init_device(d);
    return g_sms[d];
}

int *device_status_ptr()
{
    const int d = current_device();
    init_device(d);
    return g_status_ptr[d];
}

// Grid barriers of the single-pass kernels (grid_exchange.cuh): one per stream for launches
// outside graph capture, a fresh one for every launch captured into a graph (round robin over
// the pool). Zero when the library loads.
constexpr int kEagerBarriers = 1024;
constexpr int kCaptureBarriers = 7168;
__device__ GridBarrier g_grid_barriers[kEagerBarriers + kCaptureBarriers];

namespace {
std::mutex g_barrier_mutex;
GridBarrier *g_barrier_base[kMaxDevices];
std::unordered_map<uint64_t, int> g_stream_barrier[kMaxDevices];
int g_next_eager[kMaxDevices];
int g_next_capture[kMaxDevices];

GridBarrier *barrier_base(int d) // with g_barrier_mutex held
{
    if (!g_barrier_base[d]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_grid_barriers) != cudaSuccess)
            return nullptr;
        g_barrier_base[d] = reinterpret_cast<GridBarrier *>(p);
    }
    return g_barrier_base[d];
}
} // namespace

GridBarrier *grid_barrier_for(cudaStream_t s)
{
    const int d = current_device();
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
        (void)cudaGetLastError();
        cs = cudaStreamCaptureStatusNone;
    }
    std::lock_guard<std::mutex> lock(g_barrier_mutex);
    GridBarrier *base = barrier_base(d);
    if (!base)
        return nullptr;
    if (cs == cudaStreamCaptureStatusActive)
        return base + kEagerBarriers + (g_next_capture[d]++ % kCaptureBarriers);
    // the per-thread default stream is a different stream in every host thread
    uint64_t key = reinterpret_cast<uint64_t>(s);
    if (s == cudaStreamPerThread)
        key ^= (uint64_t)std::hash<std::thread::id>()(std::this_thread::get_id()) << 8;
    auto it = g_stream_barrier[d].find(key);
    if (it == g_stream_barrier[d].end())
        it = g_stream_barrier[d].emplace(key, g_next_eager[d]++ % kEagerBarriers).first;
    return base + it->second;
}

cudaError_t reset_grid_barriers()
{
    const int d = current_device();
    std::lock_guard<std::mutex> lock(g_barrier_mutex);
    GridBarrier *base = barrier_base(d);
    if (!base)
        return cudaErrorInvalidValue;
    return cudaMemset(base, 0, sizeof(GridBarrier) * (kEagerBarriers + kCaptureBarriers));
}

} // namespace nvfp4

using namespace nvfp4;

namespace {

constexpr int64_t kMaxDim = (int64_t)1 << 31;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nvfp4_status map_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

nvfp4_status check_device()
{
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return major == 10 ? NVFP4_OK : NVFP4_ERR_UNSUPPORTED;
}

nvfp4_status check_matrix(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0 || rows >= kMaxDim || cols >= kMaxDim)
        return NVFP4_ERR_SHAPE;
    if (cols % 32 != 0)
        return NVFP4_ERR_SHAPE;
    if ((rows / 128 + 1) * (cols / 64 + 1) >= ((int64_t)1 << 31)) // tile indices fit in int32
        return NVFP4_ERR_SHAPE;
    return NVFP4_OK;
}

size_t quantize_ws_bytes() { return quantize_workspace_bytes(); }

// Host-side checks of one quantize call (shared by nvfp4_quantize, _fp8_src and _batch).
nvfp4_status check_quantize(const void *x, int64_t rows, int64_t cols, const float *static_amax,
                            const uint8_t *codes, const uint8_t *scales_swz,
                            const uint8_t *scales_lin, const float *global_scale, const void *ws,
                            size_t ws_bytes)
{
    nvfp4_status st = check_matrix(rows, cols);
    if (st != NVFP4_OK)
        return st;
    const bool empty = rows == 0 || cols == 0;
    if (!global_scale)
        return NVFP4_ERR_INVALID_ARG;
    if (!empty && (!x || !codes || (!scales_swz && !scales_lin)))
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales_swz) || !aligned16(scales_lin) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(static_amax) & 3u) || !aligned16(ws))
        return NVFP4_ERR_ALIGNMENT;
    if (!static_amax && (!ws || ws_bytes < quantize_ws_bytes()))
        return NVFP4_ERR_WORKSPACE;
    return NVFP4_OK;
}

nvfp4_status quantize_common(const void *x, int src_type, const float *fp8_scale, int64_t rows,
                             int64_t cols, const float *static_amax, uint8_t *codes,
                             uint8_t *scales_swz, uint8_t *scales_lin, float *global_scale,
                             void *ws, size_t ws_bytes, cudaStream_t s)
{
    nvfp4_status st = check_quantize(x, rows, cols, static_amax, codes, scales_swz, scales_lin,
                                     global_scale, ws, ws_bytes);
    if (st != NVFP4_OK)
        return st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    return map_cuda(launch_quantize(x, src_type, fp8_scale, rows, cols, static_amax, codes,
                                    scales_swz, scales_lin, global_scale, ws, s));
}

// Workspace of nvfp4_linear_dynamic when it runs as quantize + linear: the quantized
// activations (codes, swizzled scales, global scale), the quantize workspace and the linear
// workspace, each 256-byte aligned. total = 0 when the fused kernel takes the shape.
struct DynWs {
    size_t codes, scales, gs, qws, lws, total;
};

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

DynWs linear_dynamic_ws(int64_t M, int64_t N, int64_t K)
{
    DynWs d{};
    LinearPlan pl;
    if (plan_linear_xq(M, N, K, &pl))
        return d;
    d.codes = 0;
    d.scales = d.codes + align256(nvfp4_codes_bytes(M, K));
    d.gs = d.scales + align256(nvfp4_scales_bytes(M, K, 1));
    d.qws = d.gs + 256;
    d.lws = d.qws + align256(quantize_ws_bytes());
    d.total = d.lws + align256(plan_linear(M, N, K).ws_bytes);
    return d;
}

} // namespace

extern "C" {

const char *nvfp4_status_str(nvfp4_status st)
{
    switch (st) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_SHAPE: return "invalid shape (sizes >= 0, < 2^31, cols a multiple of 32)";
    case NVFP4_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case NVFP4_ERR_WORKSPACE: return "workspace too small";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device-side wait timed out";
    case NVFP4_ERR_UNSUPPORTED: return "device is not sm_100";
    }
    return "unknown status";
}

nvfp4_status nvfp4_quantize_batch(const nvfp4_quant_job *jobs, int njobs, void *ws,
                                  size_t ws_bytes, cudaStream_t stream)
{
    if (!jobs || njobs < 1 || njobs > NVFP4_MAX_QUANT_JOBS)
        return NVFP4_ERR_INVALID_ARG;
    QuantJob jb[NVFP4_MAX_QUANT_JOBS];
    for (int j = 0; j < njobs; ++j) {
        const nvfp4_quant_job &q = jobs[j];
        if (q.src != NVFP4_SRC_F32 && q.src != NVFP4_SRC_BF16 && q.src != NVFP4_SRC_E4M3)
            return NVFP4_ERR_INVALID_ARG;
        if (q.src == NVFP4_SRC_E4M3 && (reinterpret_cast<uintptr_t>(q.fp8_scale) & 3u))
            return NVFP4_ERR_ALIGNMENT;
        const nvfp4_status st =
            check_quantize(q.x, q.rows, q.cols, q.static_amax, q.codes, q.scales_swz,
                           q.scales_lin, q.global_scale, ws, ws_bytes);
        if (st != NVFP4_OK)
            return st;
        jb[j] = QuantJob{q.x,          q.src,   q.src == NVFP4_SRC_E4M3 ? q.fp8_scale : nullptr,
                         q.rows,       q.cols,  q.static_amax,
                         q.codes,      q.scales_swz,
                         q.scales_lin, q.global_scale};
    }
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    return map_cuda(launch_quantize_batch(jb, njobs, ws, stream));
}

size_t nvfp4_codes_bytes(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0)
        return 0;
    return (size_t)(rows * (cols / 2));
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int swizzled)
{
    if (rows < 0 || cols < 0)
        return 0;
    const int64_t nb = cols / 16;
    if (!swizzled)
        return (size_t)(rows * nb);
    return (size_t)(((rows + 127) / 128) * 128 * ((nb + 3) / 4) * 4);
}

size_t nvfp4_workspace_bytes(int op, int64_t m, int64_t n, int64_t k)
{
    switch (op) {
    case NVFP4_OP_QUANTIZE: return quantize_ws_bytes();
    case NVFP4_OP_LINEAR:
        if (m <= 0 || n <= 0 || k <= 0)
            return 0;
        return plan_linear(m, n, k).ws_bytes;
    case NVFP4_OP_LINEAR_DYNAMIC:
        if (m <= 0 || n <= 0 || k <= 0)
            return 0;
        return linear_dynamic_ws(m, n, k).total;
    case NVFP4_OP_QUANTIZE_E4M3: return quantize_ws_bytes();
    case NVFP4_OP_LINEAR_LOWRANK:
        if (m <= 0 || n <= 0 || m >= kMaxDim || n > 256)
            return 0;
        return (size_t)m * (size_t)n * 2;
    case NVFP4_OP_CALIB_BF16: return calib_workspace_bytes(1);
    case NVFP4_OP_CALIB_F32: return calib_workspace_bytes(0);
    }
    return 0;
}

nvfp4_status nvfp4_quantize(const void *x, nvfp4_dtype dt, int64_t rows, int64_t cols,
                            const float *static_amax, uint8_t *codes, uint8_t *scales_swz,
                            uint8_t *scales_lin, float *global_scale, void *ws, size_t ws_bytes,
                            cudaStream_t stream)
{
    if (dt != NVFP4_F32 && dt != NVFP4_BF16)
        return NVFP4_ERR_INVALID_ARG;
    return quantize_common(x, dt == NVFP4_F32 ? kSrcF32 : kSrcBF16, nullptr, rows, cols,
                           static_amax, codes, scales_swz, scales_lin, global_scale, ws,
                           ws_bytes, stream);
}

nvfp4_status nvfp4_quantize_fp8_src(const uint8_t *x_e4m3, const float *fp8_scale, int64_t rows,
                                    int64_t cols, const float *static_amax, uint8_t *codes,
                                    uint8_t *scales_swz, uint8_t *scales_lin,
                                    float *global_scale, void *ws, size_t ws_bytes,
                                    cudaStream_t stream)
{
    if (reinterpret_cast<uintptr_t>(fp8_scale) & 3u)
        return NVFP4_ERR_ALIGNMENT;
    return quantize_common(x_e4m3, kSrcE4M3, fp8_scale, rows, cols, static_amax, codes,
                           scales_swz, scales_lin, global_scale, ws, ws_bytes, stream);
}

nvfp4_status nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales_lin,
                              const float *global_scale, int64_t rows, int64_t cols,
                              nvfp4_dtype out_dt, void *out, cudaStream_t stream)
{
    nvfp4_status st = check_matrix(rows, cols);
    if (st != NVFP4_OK)
        return st;
    if (out_dt != NVFP4_F32 && out_dt != NVFP4_BF16)
        return NVFP4_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0)
        return NVFP4_OK;
    if (!codes || !scales_lin || !global_scale || !out)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(out) || (reinterpret_cast<uintptr_t>(global_scale) & 3u))
        return NVFP4_ERR_ALIGNMENT;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    return map_cuda(launch_dequantize(codes, scales_lin, global_scale, rows, cols,
                                      out_dt == NVFP4_BF16, out, stream));
}

nvfp4_status nvfp4_linear(const uint8_t *a_codes, const uint8_t *a_scales_swz, const float *a_gs,
                          const uint8_t *w_codes, const uint8_t *w_scales_swz, const float *w_gs,
                          int64_t M, int64_t N, int64_t K, nvfp4_dtype out_dt, void *y, void *ws,
                          size_t ws_bytes, cudaStream_t stream)
{
    return nvfp4_linear_ex(a_codes, a_scales_swz, a_gs, w_codes, w_scales_swz, w_gs, M, N, K,
                           out_dt, y, ws, ws_bytes, 0u, stream);
}

nvfp4_status nvfp4_linear_dynamic(const void *x, nvfp4_dtype x_dt, const uint8_t *w_codes,
                                  const uint8_t *w_scales_swz, const float *w_gs, int64_t M,
                                  int64_t N, int64_t K, nvfp4_dtype out_dt, void *y,
                                  float *x_gs_out, void *ws, size_t ws_bytes, uint32_t flags,
                                  cudaStream_t stream)
{
    if (flags & ~(uint32_t)NVFP4_LINEAR_RESIDENT_WEIGHTS)
        return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || K % 32 != 0)
        return NVFP4_ERR_SHAPE;
    if ((out_dt != NVFP4_F32 && out_dt != NVFP4_BF16) ||
        (x_dt != NVFP4_F32 && x_dt != NVFP4_BF16))
        return NVFP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (!y)
        return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    const size_t esz = out_dt == NVFP4_BF16 ? 2 : 4;
    if (K == 0)
        return map_cuda(cudaMemsetAsync(y, 0, (size_t)M * N * esz, stream));
    if (!x || !w_codes || !w_scales_swz || !w_gs)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales_swz) || !aligned16(y) ||
        !aligned16(ws) || (reinterpret_cast<uintptr_t>(w_gs) & 3u) ||
        (reinterpret_cast<uintptr_t>(x_gs_out) & 3u))
        return NVFP4_ERR_ALIGNMENT;
    LinearPlan pl;
    if (plan_linear_xq(M, N, K, &pl)) {
        st = NVFP4_OK;
        const cudaError_t e =
            launch_linear_xq(pl, x, x_dt == NVFP4_BF16, w_codes, w_scales_swz, w_gs, M, N, K,
                             out_dt == NVFP4_BF16, y, x_gs_out, flags, stream, &st);
        return st != NVFP4_OK ? st : map_cuda(e);
    }
    // quantize + linear, the quantized activations in ws
    const DynWs d = linear_dynamic_ws(M, N, K);
    if (!ws || ws_bytes < d.total)
        return NVFP4_ERR_WORKSPACE;
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    float *gs = x_gs_out ? x_gs_out : reinterpret_cast<float *>(w + d.gs);
    st = quantize_common(x, x_dt == NVFP4_BF16 ? kSrcBF16 : kSrcF32, nullptr, M, K, nullptr,
                         w + d.codes, w + d.scales, nullptr, gs, w + d.qws,
                         quantize_ws_bytes(), stream);
    if (st != NVFP4_OK)
        return st;
    return nvfp4_linear_ex(w + d.codes, w + d.scales, gs, w_codes, w_scales_swz, w_gs, M, N, K,
                           out_dt, y, w + d.lws, ws_bytes - d.lws, flags, stream);
}

nvfp4_status nvfp4_linear_ex(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                             const float *a_gs, const uint8_t *w_codes,
                             const uint8_t *w_scales_swz, const float *w_gs, int64_t M,
                             int64_t N, int64_t K, nvfp4_dtype out_dt, void *y, void *ws,
                             size_t ws_bytes, uint32_t flags, cudaStream_t stream)
{
    if (flags & ~(uint32_t)NVFP4_LINEAR_RESIDENT_WEIGHTS)
        return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || K % 32 != 0)
        return NVFP4_ERR_SHAPE;
    if (out_dt != NVFP4_F32 && out_dt != NVFP4_BF16)
        return NVFP4_ERR_INVALID_ARG;
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (!y)
        return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    const size_t esz = out_dt == NVFP4_BF16 ? 2 : 4;
    if (K == 0)
        return map_cuda(cudaMemsetAsync(y, 0, (size_t)M * N * esz, stream));
    if (!a_codes || !a_scales_swz || !a_gs || !w_codes || !w_scales_swz || !w_gs)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_scales_swz) || !aligned16(w_codes) ||
        !aligned16(w_scales_swz) || !aligned16(y) || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(a_gs) & 3u) || (reinterpret_cast<uintptr_t>(w_gs) & 3u))
        return NVFP4_ERR_ALIGNMENT;
    const LinearPlan pl = plan_linear(M, N, K, flags);
    if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes))
        return NVFP4_ERR_WORKSPACE;
    st = NVFP4_OK;
    cudaError_t e = launch_linear(pl, a_codes, a_scales_swz, a_gs, w_codes, w_scales_swz, w_gs,
                                  M, N, K, out_dt == NVFP4_BF16, y, ws, flags, stream, &st);
    if (st != NVFP4_OK)
        return st;
    return map_cuda(e);
}

nvfp4_status nvfp4_calib_percentile_amax(const void *const *batches, int num_batches,
                                         int64_t elems_per_batch, nvfp4_dtype dt,
                                         uint32_t pct_num, uint32_t pct_den, float *out_pct,
                                         float *out_max, void *ws, size_t ws_bytes,
                                         cudaStream_t stream)
{
    if (dt != NVFP4_F32 && dt != NVFP4_BF16)
        return NVFP4_ERR_INVALID_ARG;
    if (!batches || num_batches <= 0 || !out_pct || !out_max)
        return NVFP4_ERR_INVALID_ARG;
    if (pct_den == 0 || pct_num == 0 || pct_num > pct_den)
        return NVFP4_ERR_INVALID_ARG;
    if (elems_per_batch <= 0 || elems_per_batch >= kMaxDim)
        return NVFP4_ERR_SHAPE;
    for (int i = 0; i < num_batches; ++i) {
        if (!batches[i])
            return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(batches[i]))
            return NVFP4_ERR_ALIGNMENT;
    }
    if (!aligned16(ws) || (reinterpret_cast<uintptr_t>(out_pct) & 3u) ||
        (reinterpret_cast<uintptr_t>(out_max) & 3u))
        return NVFP4_ERR_ALIGNMENT;
    const int bf16 = dt == NVFP4_BF16;
    if (!ws || ws_bytes < calib_workspace_bytes(bf16))
        return NVFP4_ERR_WORKSPACE;
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    const unsigned __int128 n = (unsigned __int128)num_batches * (uint64_t)elems_per_batch;
    unsigned __int128 rank = (n * pct_num + pct_den - 1) / pct_den;
    if (rank < 1)
        rank = 1;
    return map_cuda(launch_calib(batches, num_batches, elems_per_batch, bf16, (uint64_t)rank,
                                 out_pct, out_max, ws, stream));
}

nvfp4_status nvfp4_linear_nvfp4_out(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                                    const float *a_gs, const uint8_t *w_codes,
                                    const uint8_t *w_scales_swz, const float *w_gs, int64_t M,
                                    int64_t N, int64_t K, int act, const float *static_amax,
                                    uint8_t *y_codes, uint8_t *y_scales_swz, float *y_gs,
                                    cudaStream_t stream)
{
    if (act != NVFP4_ACT_IDENTITY && act != NVFP4_ACT_GELU_TANH)
        return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st;
    if ((st = check_matrix(M, K)) != NVFP4_OK || (st = check_matrix(N, K)) != NVFP4_OK ||
        (st = check_matrix(M, N)) != NVFP4_OK)
        return st;
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (K == 0)
        return NVFP4_ERR_SHAPE;
    if (!a_codes || !a_scales_swz || !a_gs || !w_codes || !w_scales_swz || !w_gs ||
        !static_amax || !y_codes || !y_scales_swz || !y_gs)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_scales_swz) || !aligned16(w_codes) ||
        !aligned16(w_scales_swz) || !aligned16(y_codes) || !aligned16(y_scales_swz) ||
        (reinterpret_cast<uintptr_t>(a_gs) & 3u) || (reinterpret_cast<uintptr_t>(w_gs) & 3u) ||
        (reinterpret_cast<uintptr_t>(static_amax) & 3u) || (reinterpret_cast<uintptr_t>(y_gs) & 3u))
        return NVFP4_ERR_ALIGNMENT;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    st = NVFP4_OK;
    const cudaError_t e =
        launch_linear_nvfp4_out(a_codes, a_scales_swz, a_gs, w_codes, w_scales_swz, w_gs, M, N, K,
                                act, static_amax, y_codes, y_scales_swz, y_gs, stream, &st);
    return st != NVFP4_OK ? st : map_cuda(e);
}

nvfp4_status nvfp4_linear_lowrank(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                                  const float *a_gs, const uint8_t *w_codes,
                                  const uint8_t *w_scales_swz, const float *w_gs,
                                  const void *x_bf16, const void *lr_down, const void *lr_up,
                                  int64_t M, int64_t N, int64_t K, int64_t rank, void *y,
                                  void *ws, size_t ws_bytes, cudaStream_t stream)
{
    nvfp4_status st;
    if ((st = check_matrix(M, K)) != NVFP4_OK || (st = check_matrix(N, K)) != NVFP4_OK)
        return st;
    if (K == 0 || N % 8 != 0 || rank < 16 || rank > 256 || rank % 16 != 0)
        return NVFP4_ERR_SHAPE;
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (!a_codes || !a_scales_swz || !a_gs || !w_codes || !w_scales_swz || !w_gs || !x_bf16 ||
        !lr_down || !lr_up || !y)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_scales_swz) || !aligned16(w_codes) ||
        !aligned16(w_scales_swz) || !aligned16(x_bf16) || !aligned16(lr_down) ||
        !aligned16(lr_up) || !aligned16(y) || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(a_gs) & 3u) || (reinterpret_cast<uintptr_t>(w_gs) & 3u))
        return NVFP4_ERR_ALIGNMENT;
    if (!ws || ws_bytes < (size_t)M * (size_t)rank * 2)
        return NVFP4_ERR_WORKSPACE;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    st = NVFP4_OK;
    const cudaError_t e =
        launch_linear_lowrank(a_codes, a_scales_swz, a_gs, w_codes, w_scales_swz, w_gs, x_bf16,
                              lr_down, lr_up, M, N, K, (int)rank, y, ws, stream, &st);
    return st != NVFP4_OK ? st : map_cuda(e);
}

nvfp4_status nvfp4_quantize_e4m3(const void *x, nvfp4_dtype dt, int64_t rows, int64_t cols,
                                 const float *static_amax, uint8_t *codes, float *scale, void *ws,
                                 size_t ws_bytes, cudaStream_t stream)
{
    if (dt != NVFP4_F32 && dt != NVFP4_BF16)
        return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || rows >= kMaxDim || cols >= kMaxDim)
        return NVFP4_ERR_SHAPE;
    const int64_t n = rows * cols;
    if (!scale || (n > 0 && (!x || !codes)))
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(scale) & 3u) || (reinterpret_cast<uintptr_t>(static_amax) & 3u))
        return NVFP4_ERR_ALIGNMENT;
    if (!static_amax && (!ws || ws_bytes < quantize_ws_bytes()))
        return NVFP4_ERR_WORKSPACE;
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    return map_cuda(launch_quantize_e4m3(x, dt == NVFP4_F32 ? kSrcF32 : kSrcBF16, n, static_amax,
                                         codes, scale, ws, stream));
}

nvfp4_status nvfp4_linear_e4m3(const uint8_t *a, const float *a_scale, const uint8_t *w,
                               const float *w_scale, int64_t M, int64_t N, int64_t K,
                               nvfp4_dtype out_dt, void *y, cudaStream_t stream)
{
    if (out_dt != NVFP4_F32 && out_dt != NVFP4_BF16)
        return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K <= 0 || M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || K % 16 != 0)
        return NVFP4_ERR_SHAPE;
    if (M == 0 || N == 0)
        return NVFP4_OK;
    if (!a || !w || !a_scale || !w_scale || !y)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(w) || (reinterpret_cast<uintptr_t>(a_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(w_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(y) & (out_dt == NVFP4_F32 ? 3u : 1u)))
        return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    return map_cuda(launch_linear_e4m3(a, a_scale, w, w_scale, M, N, K, out_dt == NVFP4_BF16, y,
                                       stream));
}

nvfp4_status nvfp4_selftest_wait_timeout(cudaStream_t stream)
{
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    return map_cuda(launch_wait_timeout_selftest(stream));
}

nvfp4_status nvfp4_selftest_grid_exchange(int nblk, const float *vals, int skip_cta,
                                          int late_cta, uint32_t late_ns, uint32_t poll_limit,
                                          float *out, void *ws, size_t ws_bytes,
                                          cudaStream_t stream)
{
    nvfp4_status st;
    if ((st = check_device()) != NVFP4_OK)
        return st;
    if (nblk < 1 || nblk > 160 || !vals || !out || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(vals) & 3u) || (reinterpret_cast<uintptr_t>(out) & 3u))
        return NVFP4_ERR_INVALID_ARG;
    if (!ws || ws_bytes < quantize_ws_bytes())
        return NVFP4_ERR_WORKSPACE;
    return map_cuda(launch_exchange_selftest(nblk, vals, skip_cta, late_cta, late_ns, poll_limit,
                                             out, ws, stream));
}

nvfp4_status nvfp4_sync_status(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    int *p = device_status_ptr();
    if (!p)
        return NVFP4_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    }
    // a grid barrier that gave up is left unbalanced: start every barrier afresh
    if (v == NVFP4_ERR_TIMEOUT && reset_grid_barriers() != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return (nvfp4_status)v;
}

} // extern "C"
