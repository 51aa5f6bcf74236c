// nvfp4_internal.cuh -- declarations shared by the library's translation units.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "nvfp4.h"

namespace nvfp4 {

// Source element types of the quantizer.
enum SrcType : int { kSrcF32 = 0, kSrcBF16 = 1, kSrcE4M3 = 2 };

// Byte offset of the scale of (row, block) in the tensor-core scale layout: atoms of
// 128 rows x 4 blocks (512 B), atoms of a 128-row band consecutive along the blocks.
__host__ __device__ __forceinline__ int64_t swz_offset(int64_t row, int64_t blk,
                                                       int64_t atoms_per_band)
{
    return ((row >> 7) * atoms_per_band + (blk >> 2)) * 512 + ((row & 31) << 4) +
           (((row >> 5) & 3) << 2) + (blk & 3);
}

// Device-side status word of the current device (bounded waits that give up write
// NVFP4_ERR_TIMEOUT here). Resolved once per device.
int *device_status_ptr();

int num_sms();

// ---- quantize.cu --------------------------------------------------------------------
// Per-CTA maxima the quantizer's workspace holds (one amax CTA per SM).
constexpr int kAmaxPartials = 1024;
size_t quantize_workspace_bytes();

// One tensor of a batched quantize (the fields of nvfp4_quant_job).
struct QuantJob {
    const void *x;
    int src; // SrcType
    const float *fp8_scale;
    int64_t rows, cols;
    const float *static_amax;
    uint8_t *codes, *scales_swz, *scales_lin;
    float *global_scale;
};
cudaError_t launch_quantize_batch(const QuantJob *jobs, int njobs, void *ws, cudaStream_t s);

// Launches a kernel whose bounded wait cannot complete (selftest.cu).
cudaError_t launch_wait_timeout_selftest(cudaStream_t s);
// Runs the quantizers' grid-wide exchange alone (selftest.cu).
cudaError_t launch_exchange_selftest(int nblk, const float *vals, int skip, int late,
                                     uint32_t late_ns, uint32_t limit, float *out, void *ws,
                                     cudaStream_t s);

// FP8 E4M3 tensorwise quantize of n values (fp32 or bf16, 16-byte aligned) into codes (16-byte
// aligned) and the tensor scale (device fp32); ws as for launch_quantize.
cudaError_t launch_quantize_e4m3(const void *x, int src_type, int64_t n, const float *static_amax,
                                 uint8_t *codes, float *scale_out, void *ws, cudaStream_t s);
// Block-scaled GEMM whose epilogue applies act (0 identity, 1 tanh-form GELU) and quantizes
// the [M x N] result to NVFP4 with the static amax: codes, swizzled scales, global scale.
cudaError_t launch_linear_nvfp4_out(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gs,
                                    const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gs,
                                    int64_t M, int64_t N, int64_t K, int act,
                                    const float *static_amax, uint8_t *y_codes, uint8_t *y_sf,
                                    float *y_gs, cudaStream_t s, nvfp4_status *st);
// FP8 E4M3 tensorwise W8A8 GEMM: Y = (a_scale * w_scale) * A . W^T, A [M x K], W [N x K].
cudaError_t launch_linear_e4m3(const uint8_t *a, const float *a_scale, const uint8_t *w,
                               const float *w_scale, int64_t M, int64_t N, int64_t K, int out_bf16,
                               void *y, cudaStream_t s);
cudaError_t launch_quantize(const void *x, int src_type, const float *fp8_scale, int64_t rows,
                            int64_t cols, const float *static_amax, uint8_t *codes,
                            uint8_t *scales_swz, uint8_t *scales_lin, float *global_scale,
                            void *ws, cudaStream_t s);

// ---- dequantize.cu ------------------------------------------------------------------
cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scales_lin,
                              const float *global_scale, int64_t rows, int64_t cols,
                              int out_bf16, void *out, cudaStream_t s);

// ---- calib.cu -----------------------------------------------------------------------
size_t calib_workspace_bytes(int is_bf16);
cudaError_t launch_calib(const void *const *batches, int num_batches, int64_t elems_per_batch,
                         int is_bf16, uint64_t rank, float *out_pct, float *out_max, void *ws,
                         cudaStream_t s);

// ---- gemm_sm100.cu ------------------------------------------------------------------
struct LinearPlan {
    bool swap_ab;       // operand "A" of the MMA is W (rows N), "B" is the activations
    int bn;             // MMA N (tile width on the B side)
    int64_t rows_a;     // rows of the MMA A operand
    int64_t rows_b;     // rows of the MMA B operand
    int64_t tiles_a;    // ceil(rows_a / 128)
    int64_t tiles_b;    // ceil(rows_b / bn)
    int kt;             // k-tiles of 256 elements
    int splits;         // split-K factor (1 = no split)
    int kt_per_split;
    int csplit;         // small M: K split over a thread-block cluster of csplit CTAs (0 = the
                        // persistent kernel runs the shape)
    size_t ws_bytes;    // workspace for split-K partials
};
// flags: nvfp4_linear_flags (they change the small-M launch shape, never the workspace)
LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, unsigned flags = 0);
cudaError_t launch_linear(const LinearPlan &p, const uint8_t *a_codes, const uint8_t *a_sf,
                          const float *a_gs, const uint8_t *w_codes, const uint8_t *w_sf,
                          const float *w_gs, int64_t M, int64_t N, int64_t K, int out_bf16,
                          void *y, void *ws, unsigned flags, cudaStream_t s, nvfp4_status *st);

// Fused dynamic-activation linear for M <= 32 (gemm_sm100.cu): plan (false if the shape does
// not fit the fused kernel) and launch.
bool plan_linear_xq(int64_t M, int64_t N, int64_t K, LinearPlan *out);
cudaError_t launch_linear_xq(const LinearPlan &pl, const void *x, int x_bf16,
                             const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gs,
                             int64_t M, int64_t N, int64_t K, int out_bf16, void *y,
                             float *x_gs_out, unsigned flags, cudaStream_t s, nvfp4_status *st);

// ---- lowrank_sm100.cu ----------------------------------------------------------------
// bf16 [rows x cols] row-major tensor map: box 64 columns x box_rows rows, 128B swizzle.
bool make_bf16_kmajor_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                          int box_rows);
// T' [M x r] = bf16((x . D^T) * RN(1 / alpha)), alpha = sgA * sgW (1 if that is 0); x [M x K] and
// D [r x K] bf16, r a multiple of 16 in 16..256, K > 0.
cudaError_t launch_lowrank_down(const void *x, const void *d, int64_t M, int64_t K, int r,
                                const float *a_gs, const float *w_gs, void *t, cudaStream_t s,
                                nvfp4_status *st);
// Y = FP4 product + T . U^T (bf16 out): launch_lowrank_down into t_ws (M x rank bf16), then the
// pair GEMM with the low-rank k-tiles.
cudaError_t launch_linear_lowrank(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gs,
                                  const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gs,
                                  const void *x, const void *lr_down, const void *lr_up,
                                  int64_t M, int64_t N, int64_t K, int rank, void *y, void *t_ws,
                                  cudaStream_t s, nvfp4_status *st);

} // namespace nvfp4
