/*
 * nvfp4.h -- C ABI of the NVFP4 quantized linear layer for NVIDIA B200 (sm_100a).
 *
 * The format (from "Qwen-Image NVFP4 on a 16 GB Ada GPU", section "What NVFP4 is and how it
 * differs from NF4", and the figure "First NVFP4 block, as stored in the file"):
 *   - each value is a 4-bit E2M1 code: sign, two exponent bits, one mantissa bit;
 *     magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6};
 *   - each block of 16 consecutive values of a row carries one FP8 E4M3 scale;
 *   - each tensor carries one FP32 global scale;
 *   - value = E2M1(code) x block scale x global scale;
 *   - two codes per byte, the first (even-index) code in the low nibble.
 *
 * Conventions for every call:
 *   - Matrices are row-major. A quantized matrix of [rows x cols] values has
 *       codes      : rows x cols/2 bytes, row-major;
 *       scales_lin : rows x cols/16 bytes (E4M3 bit patterns), row-major ("linear" layout);
 *       scales_swz : nvfp4_scales_bytes(rows, cols, 1) bytes, the tensor-core operand layout:
 *                    the [rows x cols/16] scale matrix cut into atoms of 128 rows x 4 blocks,
 *                    512 bytes each; atoms of one 128-row band are stored one after another
 *                    along the blocks, bands one after another; inside an atom, (r, b) sits at
 *                    byte 16*(r%32) + 4*((r%128)/32) + b%4. Padding rows / blocks are zero;
 *       global_scale: one fp32 in device memory.
 *   - Blocks run along cols (the GEMM's K dimension). cols must be a multiple of 32.
 *   - The caller owns every buffer; the library never allocates or frees memory. Every
 *     pointer is a device pointer unless stated otherwise: arrays 16-byte aligned, pointers
 *     to a single fp32 (global scales, static amax, fp8 scales, percentile outputs) 4-byte
 *     aligned (NVFP4_ERR_ALIGNMENT otherwise).
 *   - Every call is asynchronous on the given stream. Argument checks run on the host before
 *     any launch and return an error without touching memory.
 *   - Numbers of rows, cols, M, N, K are >= 0 and < 2^31. Empty inputs are allowed.
 *   - Inputs must be finite; a NaN or Inf input gives unspecified codes.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1, /* NULL pointer, bad enum, bad ratio */
    NVFP4_ERR_SHAPE = 2,       /* negative or too large size, cols not a multiple of 32 */
    NVFP4_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
    NVFP4_ERR_WORKSPACE = 4,   /* workspace smaller than nvfp4_workspace_bytes() */
    NVFP4_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed */
    NVFP4_ERR_TIMEOUT = 6,     /* a device-side wait gave up (reported by nvfp4_sync_status) */
    NVFP4_ERR_UNSUPPORTED = 7  /* the device is not sm_100 */
} nvfp4_status;

typedef enum { NVFP4_F32 = 0, NVFP4_BF16 = 1 } nvfp4_dtype;

/* Operations whose workspace can be queried with nvfp4_workspace_bytes. */
typedef enum {
    NVFP4_OP_QUANTIZE = 0,   /* m = rows, k = cols (n ignored) */
    NVFP4_OP_LINEAR = 1,     /* m = M, n = N, k = K */
    NVFP4_OP_CALIB_BF16 = 2, /* m, n, k ignored */
    NVFP4_OP_CALIB_F32 = 3,  /* m, n, k ignored */
    NVFP4_OP_LINEAR_DYNAMIC = 4, /* m = M, n = N, k = K of nvfp4_linear_dynamic */
    NVFP4_OP_QUANTIZE_E4M3 = 5,  /* nvfp4_quantize_e4m3 (m, n, k ignored) */
    NVFP4_OP_LINEAR_LOWRANK = 6  /* nvfp4_linear_lowrank: m = M, n = rank (k ignored) */
} nvfp4_op;

/* Human-readable name of a status. Never NULL. */
const char *nvfp4_status_str(nvfp4_status st);

/* Bytes of the packed codes of a rows x cols matrix: rows * cols / 2. */
size_t nvfp4_codes_bytes(int64_t rows, int64_t cols);

/* Bytes of its scales: linear rows * cols/16 (swizzled = 0), or the swizzled layout padded to
 * whole 128 x 4 atoms (swizzled = 1). */
size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int swizzled);

/* Device workspace the call needs (0 if none). Returns 0 for an unknown op. A workspace holds
 * the call's state (partial maxima, split-K partials) from the launch until its kernels have
 * finished: calls that may run at the same time (on different streams or host threads) need
 * different workspaces; calls on one stream may reuse one. */
size_t nvfp4_workspace_bytes(int op, int64_t m, int64_t n, int64_t k);

/*
 * Quantize a fp32 or bf16 matrix x [rows x cols] to NVFP4.
 *
 * Global scale: sg = amax / (6 * 448) where amax is either the dynamic per-tensor max |x|
 * (static_amax == NULL; "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details":
 * activations quantized at runtime from the per-tensor amax) or the calibrated value that
 * static_amax points to (device fp32; "Qwen-Rapid-AIO FP8 -> NVFP4", "Recommended Model":
 * p99.9 input scales). Values above a static amax saturate to +-6 x 448 x sg.
 * Block scale: sb = E4M3(bmax / (6 * sg)), round to nearest even, saturating at 448.
 * Code: E2M1(x * (1 / (sb * sg))), round to nearest even, saturating at 6, sign kept.
 * All code-deciding arithmetic is IEEE fp32 round-to-nearest in that order; sg == 0 or
 * sb == 0 gives all-zero codes for the block.
 *
 * Outputs: codes (required); scales_swz and / or scales_lin (at least one non-NULL; padding of
 * scales_swz is written with zeros); global_scale (required, device fp32).
 * ws: device workspace of nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, 0, cols) bytes
 * (may be NULL when static_amax is given).
 */
nvfp4_status nvfp4_quantize(const void *x, nvfp4_dtype dt, int64_t rows, int64_t cols,
                            const float *static_amax, uint8_t *codes, uint8_t *scales_swz,
                            uint8_t *scales_lin, float *global_scale, void *ws, size_t ws_bytes,
                            cudaStream_t stream);

/*
 * Double quantization ("Qwen-Rapid-AIO FP8 -> NVFP4", "Why This Exists" and
 * "1. Double Quantization"): x_e4m3 holds FP8 E4M3 bit patterns; each value is upcast to
 * fp32 as e4m3 * (*fp8_scale) (one fp32 multiply; fp8_scale is a device fp32, or NULL for
 * layers that ship without a weight_scale, read as 1.0) and then quantized exactly as
 * nvfp4_quantize does. Same outputs, workspace and rules as nvfp4_quantize.
 */
nvfp4_status nvfp4_quantize_fp8_src(const uint8_t *x_e4m3, const float *fp8_scale, int64_t rows,
                                    int64_t cols, const float *static_amax, uint8_t *codes,
                                    uint8_t *scales_swz, uint8_t *scales_lin,
                                    float *global_scale, void *ws, size_t ws_bytes,
                                    cudaStream_t stream);

/* Source element type of a batched quantize job. */
typedef enum { NVFP4_SRC_F32 = 0, NVFP4_SRC_BF16 = 1, NVFP4_SRC_E4M3 = 2 } nvfp4_src;

/* One tensor of nvfp4_quantize_batch: the arguments of nvfp4_quantize (F32 / BF16 source) or
 * nvfp4_quantize_fp8_src (E4M3 source; fp8_scale ignored for the other types). */
typedef struct {
    const void *x;
    int src; /* nvfp4_src */
    const float *fp8_scale;
    int64_t rows, cols;
    const float *static_amax;
    uint8_t *codes, *scales_swz, *scales_lin;
    float *global_scale;
} nvfp4_quant_job;

#define NVFP4_MAX_QUANT_JOBS 8

/*
 * Several quantizations in one pass: job i gets exactly the outputs that nvfp4_quantize /
 * nvfp4_quantize_fp8_src give for its arguments (its own amax and global scale). No
 * counterpart in the paper: the per-tensor method above, batched so that the tensors share one
 * amax launch and one encode launch (CTAs split in proportion to the bytes) and their memory
 * traffic overlaps, e.g. a weight re-quantized from FP8 and the activations of the same layer.
 * Two tensors whose larger fits the CTAs' shared memory (up to about 28 MB) and whose smaller
 * fits their registers (up to about 9.7 MB) are quantized in a single launch instead, each read
 * from HBM once.
 * jobs: HOST array of njobs (1 .. NVFP4_MAX_QUANT_JOBS) descriptors, each checked as its own
 * call would be (first failure returned, nothing launched). ws: one workspace of
 * nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, ...) bytes serves the whole batch.
 */
nvfp4_status nvfp4_quantize_batch(const nvfp4_quant_job *jobs, int njobs, void *ws,
                                  size_t ws_bytes, cudaStream_t stream);

/*
 * Dequantize ("Qwen-Image NVFP4 on a 16 GB Ada GPU", worked example under "First NVFP4
 * block, as stored in the file": weight = E2M1 x block scale x global scale).
 * out[r, k] = (E2M1(code) * sb) * sg in fp32 (two round-to-nearest multiplies in that order);
 * for NVFP4_BF16 output, that fp32 value rounded to nearest even. Reads linear scales.
 * out: rows x cols of out_dt. No workspace.
 */
nvfp4_status nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales_lin,
                              const float *global_scale, int64_t rows, int64_t cols,
                              nvfp4_dtype out_dt, void *out, cudaStream_t stream);

/*
 * Block-scaled W4A4 linear layer Y = dequant(A) . dequant(W)^T on the FP4 tensor cores
 * ("Qwen-Image NVFP4 on a 16 GB Ada GPU", "What NVFP4 is...": on Blackwell the tensor cores
 * multiply in FP4 with weights and activations both in 4 bits).
 *   A: M x K (activations: a_codes, a_scales_swz, a_gs), W: N x K (weights, nn.Linear layout).
 *   Y[m, n] = (sgA * sgW) * sum_b sA[m,b] * sW[n,b] * sum_{k in b} eA[m,k] * eW[n,k],
 *   accumulated in fp32 by the tensor cores, scaled by sgA * sgW (fp32), then stored as out_dt
 *   (bf16 rounded to nearest even). y: M x N of out_dt.
 * K must be a multiple of 32. ws: nvfp4_workspace_bytes(NVFP4_OP_LINEAR, M, N, K) bytes.
 */
nvfp4_status nvfp4_linear(const uint8_t *a_codes, const uint8_t *a_scales_swz, const float *a_gs,
                          const uint8_t *w_codes, const uint8_t *w_scales_swz, const float *w_gs,
                          int64_t M, int64_t N, int64_t K, nvfp4_dtype out_dt, void *y, void *ws,
                          size_t ws_bytes, cudaStream_t stream);

/* Flags of nvfp4_linear_ex (bitwise or). */
typedef enum {
    NVFP4_LINEAR_DEFAULT = 0,
    /* The weight operand (w_codes, w_scales_swz, w_gs) is resident: nothing that may still be
     * running on the stream when this call's kernel starts writes it (model weights loaded or
     * quantized ahead of time and only read since). The small-M (M <= 128) kernel then starts
     * reading W while the previous kernel of the stream is still finishing (programmatic
     * dependent launch), so consecutive decode-size layers stream weights back to back; the
     * activations, the global scales' product and y still wait for that kernel. Ignored for
     * M > 128. Results are identical with and without the flag. */
    NVFP4_LINEAR_RESIDENT_WEIGHTS = 1
} nvfp4_linear_flags;

/*
 * nvfp4_linear with flags (nvfp4_linear_flags). No counterpart in the paper: the flag is a
 * scheduling hint about the caller's stream, the result is the one nvfp4_linear defines.
 * An unknown flag bit gives NVFP4_ERR_INVALID_ARG.
 */
nvfp4_status nvfp4_linear_ex(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                             const float *a_gs, const uint8_t *w_codes,
                             const uint8_t *w_scales_swz, const float *w_gs, int64_t M,
                             int64_t N, int64_t K, nvfp4_dtype out_dt, void *y, void *ws,
                             size_t ws_bytes, uint32_t flags, cudaStream_t stream);

/*
 * Linear layer on unquantized activations: Y = dequant(Q(x)) . dequant(W)^T, where Q(x) is
 * exactly what nvfp4_quantize(x, dynamic per-tensor amax) gives ("Qwen3-VL-8B-Instruct-
 * heretic-NVFP4", "Quantization Details": activations quantized at runtime from the per-tensor
 * amax), and the product is nvfp4_linear's. x: M x K of x_dt (NVFP4_F32 or NVFP4_BF16),
 * row-major, 16-byte aligned; W as in nvfp4_linear. x_gs_out (device fp32, may be NULL)
 * receives the activations' global scale.
 * For M <= 16 (decode) one kernel does both: every thread-block cluster takes the tensor amax
 * itself, each CTA encodes its K range of x straight into the tensor-core operand in shared
 * memory, and the weights stream as in nvfp4_linear (flags as in nvfp4_linear_ex), so the
 * quantized activations never go to HBM and no quantize kernels run before the GEMV. Other
 * shapes run nvfp4_quantize and nvfp4_linear, with the quantized activations in ws.
 * ws: nvfp4_workspace_bytes(NVFP4_OP_LINEAR_DYNAMIC, M, N, K) bytes (0 for the fused case).
 */
nvfp4_status nvfp4_linear_dynamic(const void *x, nvfp4_dtype x_dt, const uint8_t *w_codes,
                                  const uint8_t *w_scales_swz, const float *w_gs, int64_t M,
                                  int64_t N, int64_t K, nvfp4_dtype out_dt, void *y,
                                  float *x_gs_out, void *ws, size_t ws_bytes, uint32_t flags,
                                  cudaStream_t stream);

/*
 * nvfp4_linear without a caller-supplied workspace. No counterpart in the paper: it exists for
 * callers that cannot call cudaMalloc or lend a device buffer, e.g. code that runs inside an
 * engine or plugin host that owns all device memory, latency-critical loops where an
 * allocation (which may synchronize the device) is not allowed, or callers with no buffer to
 * spare. Same arguments, result and checks as nvfp4_linear minus ws / ws_bytes.
 * Scratch: the split-K partial sums go to a 4 MiB array that the library keeps in device
 * memory (every GPU that loads the library holds it until the process exits). Shapes whose
 * partial sums need more than 4 MiB (nvfp4_workspace_bytes(NVFP4_OP_LINEAR, M, N, K) >
 * 4 MiB) are rejected with NVFP4_ERR_WORKSPACE before any launch; shapes that need no partial
 * sums (workspace 0) never touch the array. The call allocates nothing.
 * The array is shared by every call on the device and keeps the last call's contents; each
 * call writes every partial it later reads, so nothing needs clearing. Calls whose GPU work
 * overlaps (other streams, or concurrent host threads) race on the array: serialize them.
 * The first call on each device that needs the scratch resolves its address
 * (cudaGetSymbolAddress) with that device current; make that first call before any stream
 * capture. A lookup that fails returns NVFP4_ERR_CUDA and is tried again by the next call.
 */
nvfp4_status nvfp4_linear_noalloc(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                                  const float *a_gs, const uint8_t *w_codes,
                                  const uint8_t *w_scales_swz, const float *w_gs, int64_t M,
                                  int64_t N, int64_t K, nvfp4_dtype out_dt, void *y,
                                  cudaStream_t stream);

/*
 * Static-scale calibration ("Qwen-Rapid-AIO FP8 -> NVFP4", "Recommended Model": p99.9
 * percentile aggregation over calibration generations instead of max aggregation).
 * Over the union of num_batches device arrays (batches is a HOST array of device pointers),
 * each of elems_per_batch values of dt, computes exactly:
 *   *out_pct = the nearest-rank pct_num/pct_den percentile of |x|: the rank-th smallest |x|
 *              with rank = ceil(n * pct_num / pct_den) (1-based, at least 1), n = all values;
 *   *out_max = max |x|.
 * out_pct / out_max are device fp32; either may be used as the static_amax of nvfp4_quantize.
 * Requires 0 < pct_num <= pct_den and n > 0.
 * ws: nvfp4_workspace_bytes(NVFP4_OP_CALIB_BF16 or _F32, 0, 0, 0) bytes.
 */
nvfp4_status nvfp4_calib_percentile_amax(const void *const *batches, int num_batches,
                                         int64_t elems_per_batch, nvfp4_dtype dt,
                                         uint32_t pct_num, uint32_t pct_den, float *out_pct,
                                         float *out_max, void *ws, size_t ws_bytes,
                                         cudaStream_t stream);

/* Activation of nvfp4_linear_nvfp4_out. */
typedef enum {
    NVFP4_ACT_IDENTITY = 0,
    NVFP4_ACT_GELU_TANH = 1 /* 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))) */
} nvfp4_act;

/*
 * Linear layer whose output is the next layer's NVFP4 operand: Y as nvfp4_linear defines it
 * (fp32 tensor-core accumulation, scaled by sgA * sgW in fp32), V = act(Y), then V quantized
 * exactly as nvfp4_quantize(V, static_amax) would quantize an fp32 V, inside the GEMM's
 * epilogue, so V never goes to memory in bf16 ("Qwen-Rapid-AIO FP8 -> NVFP4", "Recommended
 * Model": static input scales from calibration; e.g. the first GEMM of an MLP writing the
 * second one's activations). act: nvfp4_act; NVFP4_ACT_GELU_TANH uses the hardware's fast
 * exponential and division (relative error ~1e-6 against the exact formula), so codes can
 * differ from an exact evaluation only where V lies that close to a rounding boundary.
 * A: M x K, W: N x K as in nvfp4_linear (swizzled scales). static_amax: device fp32.
 * Outputs (device, 16-byte aligned): y_codes M x N/2 bytes, y_scales_swz
 * nvfp4_scales_bytes(M, N, 1) bytes (padding written as zero), y_gs one fp32 (the global scale,
 * static_amax / 2688). K and N must be multiples of 32. No workspace.
 */
nvfp4_status nvfp4_linear_nvfp4_out(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                                    const float *a_gs, const uint8_t *w_codes,
                                    const uint8_t *w_scales_swz, const float *w_gs, int64_t M,
                                    int64_t N, int64_t K, int act, const float *static_amax,
                                    uint8_t *y_codes, uint8_t *y_scales_swz, float *y_gs,
                                    cudaStream_t stream);

/*
 * Linear layer with a BF16 low-rank branch ("Qwen Image 2.1: INT4 + FP4", section "What I
 * quantized": the transformer's layers run in native FP4 on Blackwell with BF16 rank-128
 * branches):
 *   Y = dequant(A) . dequant(W)^T + (x . D^T) . U^T
 * A, W, a_gs, w_gs: the FP4 operands as in nvfp4_linear (A is normally nvfp4_quantize(x)).
 * x: M x K bf16, the layer's unquantized input. lr_down D: rank x K bf16; lr_up U: N x rank
 * bf16; all row-major, 16-byte aligned. y: M x N bf16.
 * How it is computed: one kernel forms T' = bf16((x . D^T) * RN(1 / alpha)) with fp32 tensor-core
 * accumulation, alpha = sgA * sgW in fp32 (1 when that product is 0), into ws; the FP4 GEMM
 * then adds T' . U^T (bf16 tensor-core MMAs) into the same fp32 accumulator as the FP4
 * product, and its epilogue multiplies by alpha and rounds to bf16. Against the branch taken
 * exactly with its intermediate rounded once to bf16 (bf16(x . D^T) . U^T), each term
 * T[m,j] U[n,j] can differ by up to 2^-7 |T[m,j] U[n,j]| (two bf16 roundings instead of one),
 * on top of nvfp4_linear's fp32 accumulation. |x . D^T| / alpha must stay below the bf16
 * range (3.4e38).
 * K: multiple of 32, > 0. N: multiple of 8. rank: multiple of 16, 16..256.
 * ws: nvfp4_workspace_bytes(NVFP4_OP_LINEAR_LOWRANK, M, rank, 0) bytes (M * rank * 2).
 */
nvfp4_status nvfp4_linear_lowrank(const uint8_t *a_codes, const uint8_t *a_scales_swz,
                                  const float *a_gs, const uint8_t *w_codes,
                                  const uint8_t *w_scales_swz, const float *w_gs,
                                  const void *x_bf16, const void *lr_down, const void *lr_up,
                                  int64_t M, int64_t N, int64_t K, int64_t rank, void *y,
                                  void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * FP8 E4M3 tensorwise quantization ("Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization
 * Details" and "Layer breakdown": embed_tokens and lm_head in float8_e4m3fn, tensorwise,
 * round-to-nearest). One fp32 scale per tensor and one E4M3 code per value:
 *   s = amax / 448 (fp32 division; amax = max |x| of the tensor, or *static_amax),
 *   code = sign(x) | E4M3(|x| / s): the IEEE fp32 quotient rounded to the nearest E4M3 value,
 *   ties to the even code, saturating at 448; s == 0 gives sign-only codes.
 * Decode: x ~= E4M3(code) * s.
 * x: rows x cols of dt (NVFP4_F32 or NVFP4_BF16), row-major and contiguous, 16-byte aligned.
 * codes: rows x cols bytes (device, 16-byte aligned), written. scale: device fp32, written.
 * static_amax: device fp32 or NULL (dynamic). Values must be finite.
 * ws: nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE_E4M3, 0, 0, 0) bytes, unused with static_amax.
 * Asynchronous on stream. The caller owns every buffer.
 */
nvfp4_status nvfp4_quantize_e4m3(const void *x, nvfp4_dtype dt, int64_t rows, int64_t cols,
                                 const float *static_amax, uint8_t *codes, float *scale, void *ws,
                                 size_t ws_bytes, cudaStream_t stream);

/*
 * FP8 E4M3 tensorwise W8A8 linear layer on the FP8 tensor cores ("Qwen3-VL-8B-Instruct-
 * heretic-NVFP4", "Runtime / hardware": FP8 layers run as native FP8 on Blackwell; "Qwen-Rapid-
 * AIO FP8 -> NVFP4", "Solution": FP8 layers stay FP8, so E4M3 weights with their scale are used
 * as they are):
 *   Y[m, n] = (sA * sW) * sum_k E4M3(a[m, k]) * E4M3(w[n, k]),
 * accumulated in fp32 by the tensor cores, scaled by sA * sW (fp32), stored as out_dt (bf16
 * rounded to nearest even).
 * a: M x K codes (activations, e.g. from nvfp4_quantize_e4m3), w: N x K codes (nn.Linear
 * layout), both row-major and 16-byte aligned; a_scale / w_scale: device fp32.
 * y: M x N of out_dt, row-major. K must be a positive multiple of 16. No workspace.
 */
nvfp4_status nvfp4_linear_e4m3(const uint8_t *a, const float *a_scale, const uint8_t *w,
                               const float *w_scale, int64_t M, int64_t N, int64_t K,
                               nvfp4_dtype out_dt, void *y, cudaStream_t stream);

/*
 * Test of the failure-detection path. No counterpart in the paper. Launches one small kernel
 * whose bounded wait cannot complete (an mbarrier that nothing arrives on); it gives up after
 * a short poll limit and records NVFP4_ERR_TIMEOUT in the device-side status word, exactly as
 * a library kernel does when one of its waits runs out, and returns normally (no fault, the
 * context stays usable). The next nvfp4_sync_status on the stream reports NVFP4_ERR_TIMEOUT.
 * Returns the launch status.
 */
nvfp4_status nvfp4_selftest_wait_timeout(cudaStream_t stream);

/*
 * Test of the single-pass quantizers' grid-wide exchange. No counterpart in the paper. Those
 * kernels (nvfp4_quantize of 16 MB and more with a dynamic amax, the two-tensor
 * nvfp4_quantize_batch, nvfp4_quantize_e4m3) meet once all their CTAs have folded their
 * share of the tensor: each CTA writes its partial maxima into an 8-byte slot of the
 * workspace and adds once to a barrier counter in library memory (one per stream, a fresh one
 * per launch captured into a CUDA graph) whose top bit flips at the last arrival; every CTA
 * polls for the flip for a bounded number of rounds, then reads all the slots. This call runs
 * the exchange alone, on a cooperative grid of nblk
 * (1..160) CTAs of one warp: CTA i contributes vals[i] (device fp32; and vals[i] / 2 as the
 * second value); CTA skip_cta (-1: none) never arrives; CTA late_cta (-1: none) arrives after
 * spinning late_ns nanoseconds; poll_limit bounds the rounds. If every CTA arrived, out[0..1]
 * (device fp32) get max vals and max vals / 2; otherwise the waiting CTAs give up after
 * poll_limit rounds, record NVFP4_ERR_TIMEOUT in the status word (see nvfp4_sync_status) and
 * return, leaving out untouched. ws: nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, ...) bytes,
 * any contents. Returns the launch status.
 */
nvfp4_status nvfp4_selftest_grid_exchange(int nblk, const float *vals, int skip_cta,
                                          int late_cta, uint32_t late_ns, uint32_t poll_limit,
                                          float *out, void *ws, size_t ws_bytes,
                                          cudaStream_t stream);

/*
 * Synchronize the stream, then report and clear the library's device-side status word
 * (set by a kernel whose bounded wait gave up: NVFP4_ERR_TIMEOUT). After a timeout it also
 * resets the library's grid-barrier counters, which an exchange that gave up leaves
 * unbalanced. Returns NVFP4_ERR_CUDA if the synchronization itself failed.
 */
nvfp4_status nvfp4_sync_status(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
