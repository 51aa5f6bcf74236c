/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the NVFP4 quantized linear layer.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU-baseline leg load
 * this file. The CUDA library never links, includes or calls it, and it shares no code, table
 * or header with the CUDA sources.
 *
 * Every step below is written from the definitions on these pages:
 *   [QI]  "Qwen-Image NVFP4 on a 16 GB Ada GPU" (efraingaray.com), section
 *         "What NVFP4 is and how it differs from NF4": E2M1 codes (sign, two exponent bits,
 *         one mantissa bit, values 0..6), one FP8 scale per 16-weight block, one FP32 global
 *         scale per matrix.
 *   [QIb] same page, figure "First NVFP4 block, as stored in the file" and the worked
 *         example under it: weight = E2M1 x block scale x global scale; two codes per byte,
 *         the low nibble holds the first code; 4 bits + 8 bits of scale per 16 = 4.5 bits.
 *   [QR]  "Qwen-Rapid-AIO FP8 -> NVFP4" model card, "Why This Exists" and
 *         "1. Double Quantization": FP8 E4M3 weights are upcast to FP32 (times their
 *         weight_scale, which some layers lack) and then re-quantized to NVFP4.
 *   [QV]  "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details": activations are
 *         quantized dynamically from the per-tensor amax.
 *   [QRc] the Qwen-Rapid-AIO card, "Recommended Model": static input scales from the p99.9
 *         percentile of calibration activations instead of their max.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - global scale sg = amax / (6 * 448): the block holding amax gets the largest finite E4M3
 *     scale. The stored sg is the decode multiplier of [QIb].
 *   - block scale sb = E4M3(bmax / (sg * 6)), round-to-nearest-even, saturating at 448,
 *     subnormals kept.
 *   - element code = E2M1(x * (1 / (float(sb) * sg))), round-to-nearest-even, saturating at 6,
 *     sign kept (a negative value that rounds to zero magnitude gives code 0b1000).
 *   - sg == 0 or sb == 0: every code of the block is 0.
 *   - all arithmetic that decides a code is IEEE fp32 with round-to-nearest, in the order
 *     written; this file must be compiled without FMA contraction (-ffp-contract=off).
 *   - percentile: nearest rank, rank = ceil(n * num / den) (1-based) over |x|.
 *
 * Layouts: values are row-major [rows x cols]; blocks run along cols. Codes are
 * [rows x cols/2] bytes. "Linear" scales are [rows x cols/16]. "Swizzled" scales are the
 * tensor-core operand layout: 128-row x 4-block atoms of 512 bytes, atoms of one 128-row band
 * contiguous along the blocks, zero padding (see ora_swizzled_offset).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* Scalar codecs                                                                               */
/* ------------------------------------------------------------------------------------------ */

/* E2M1 magnitude of a 3-bit magnitude code: exponent bits e (bias 1), mantissa bit m.
 * e == 0 is the subnormal range (m * 0.5); otherwise 2^(e-1) * (1 + m/2). [QI] */
static double e2m1_magnitude(int mag_code)
{
    int e = (mag_code >> 1) & 3;
    int m = mag_code & 1;
    if (e == 0)
        return 0.5 * m;
    return ldexp(1.0 + 0.5 * m, e - 1);
}

/* Signed value of a 4-bit code: bit 3 is the sign. [QI], [QIb] */
double ora_e2m1_decode(int code)
{
    double v = e2m1_magnitude(code & 7);
    return (code & 8) ? -v : v;
}

/* FP8 E4M3 (bias 7, 3 mantissa bits, subnormals, 0x7F / 0xFF are NaN, no infinities). */
double ora_e4m3_decode(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7)
        return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return s ? -v : v;
}

/* Nearest code on a grid of non-negative magnitudes listed in increasing code order,
 * ties to the even code, saturating at the largest magnitude. v must be >= 0 and not NaN.
 * The midpoint test compares 2v with lo + hi: both sides are exact in double. */
static int nearest_code_rne(double v, const double *mag, int n)
{
    if (v >= mag[n - 1])
        return n - 1;
    int i = 0;
    while (mag[i + 1] <= v)
        i++;
    double twice = 2.0 * v, sum = mag[i] + mag[i + 1];
    if (twice < sum)
        return i;
    if (twice > sum)
        return i + 1;
    return (i % 2 == 0) ? i : i + 1;
}

static double g_e2m1_mag[8];
static double g_e4m3_mag[127];
static int g_tables_ready = 0;

static void init_tables(void)
{
    if (g_tables_ready)
        return;
    for (int c = 0; c < 8; c++)
        g_e2m1_mag[c] = e2m1_magnitude(c);
    for (int c = 0; c < 127; c++)
        g_e4m3_mag[c] = ora_e4m3_decode((uint8_t)c);
    g_tables_ready = 1;
}

/* E2M1 code of y: sign bit from y, magnitude rounded to nearest (ties to even code),
 * saturating at 6. */
int ora_e2m1_encode(float y)
{
    init_tables();
    int sign = signbit(y) ? 8 : 0;
    return sign | nearest_code_rne(fabs((double)y), g_e2m1_mag, 8);
}

/* E4M3 code of a non-negative v: round to nearest, ties to even, saturate at 448 (0x7E). */
uint8_t ora_e4m3_encode_nonneg(float v)
{
    init_tables();
    if (!(v > 0.0f))
        return 0;
    return (uint8_t)nearest_code_rne((double)v, g_e4m3_mag, 127);
}

/* Array forms of the two encoders, for exhaustive checks. */
void ora_e2m1_encode_array(const float *y, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)ora_e2m1_encode(y[i]);
}

void ora_e4m3_encode_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = ora_e4m3_encode_nonneg(v[i]);
}

float ora_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest even (finite inputs). */
uint16_t ora_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1;
    u += 0x7FFF + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------------------------ */
/* Layout helpers                                                                              */
/* ------------------------------------------------------------------------------------------ */

/* Byte offset of the scale of (row, block) in the swizzled layout. The layout tiles the
 * [rows x nblocks] scale matrix into atoms of 128 rows x 4 blocks (512 bytes). Atoms are
 * ordered band by band (a band = 128 rows), and along the blocks inside a band. Inside an
 * atom, row r sits at 16 * (r % 32) + 4 * ((r % 128) / 32) and block b at b % 4. */
int64_t ora_swizzled_offset(int64_t row, int64_t block, int64_t nblocks)
{
    int64_t atoms_per_band = (nblocks + 3) / 4;
    int64_t atom = (row / 128) * atoms_per_band + block / 4;
    int64_t inner = 16 * (row % 32) + 4 * ((row % 128) / 32) + (block % 4);
    return atom * 512 + inner;
}

int64_t ora_swizzled_bytes(int64_t rows, int64_t cols)
{
    int64_t nblocks = cols / 16;
    return ((rows + 127) / 128) * 128 * (((nblocks + 3) / 4) * 4);
}

/* ------------------------------------------------------------------------------------------ */
/* Source upcast                                                                               */
/* ------------------------------------------------------------------------------------------ */

/* dtype: 0 = fp32, 1 = bf16, 2 = FP8 E4M3 multiplied by *fp8_scale (NULL -> 1.0, [QR]:
 * layers without weight_scale). The fp8 upcast is one fp32 multiply. */
void ora_source_to_f32(const void *src, int dtype, const float *fp8_scale, int64_t n, float *out)
{
    if (dtype == 0) {
        memcpy(out, src, (size_t)n * 4);
    } else if (dtype == 1) {
        const uint16_t *s = (const uint16_t *)src;
        for (int64_t i = 0; i < n; i++)
            out[i] = ora_bf16_to_f32(s[i]);
    } else {
        const uint8_t *s = (const uint8_t *)src;
        float s8 = fp8_scale ? *fp8_scale : 1.0f;
        for (int64_t i = 0; i < n; i++) {
            float e = (float)ora_e4m3_decode(s[i]);
            out[i] = e * s8;
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Quantize / dequantize                                                                       */
/* ------------------------------------------------------------------------------------------ */

float ora_amax(const float *x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(x[i]);
        if (a > m)
            m = a;
    }
    return m;
}

/* Quantize a fp32 matrix to NVFP4. amax_in: NULL -> dynamic amax of x [QV]; otherwise the
 * static calibrated amax [QRc] (values above it saturate). Writes codes [rows x cols/2],
 * linear scales [rows x cols/16], optionally swizzled scales (zero padded), and sg.
 * Returns 0, or -1 if cols is not a multiple of 16. */
int ora_quantize_f32(const float *x, int64_t rows, int64_t cols, const float *amax_in,
                     uint8_t *codes, uint8_t *scales_lin, uint8_t *scales_swz, float *sg_out)
{
    if (cols % 16 != 0 || rows < 0)
        return -1;
    int64_t nb = cols / 16;
    float amax = amax_in ? *amax_in : ora_amax(x, rows * cols);
    float sg = amax / 2688.0f; /* 2688 = 6 * 448 */
    float t = sg * 6.0f;
    *sg_out = sg;
    if (scales_swz)
        memset(scales_swz, 0, (size_t)ora_swizzled_bytes(rows, cols));
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < nb; b++) {
            const float *blk = x + r * cols + b * 16;
            float bmax = 0.0f;
            for (int j = 0; j < 16; j++) {
                float a = fabsf(blk[j]);
                if (a > bmax)
                    bmax = a;
            }
            uint8_t sb = 0;
            if (sg > 0.0f) {
                float sraw = bmax / t;
                sb = ora_e4m3_encode_nonneg(sraw);
            }
            scales_lin[r * nb + b] = sb;
            if (scales_swz)
                scales_swz[ora_swizzled_offset(r, b, nb)] = sb;
            int c[16];
            float fsb = (float)ora_e4m3_decode(sb);
            if (fsb == 0.0f) {
                for (int j = 0; j < 16; j++)
                    c[j] = 0;
            } else {
                float d = fsb * sg;
                float rcp = 1.0f / d;
                for (int j = 0; j < 16; j++) {
                    float y = blk[j] * rcp;
                    c[j] = ora_e2m1_encode(y);
                }
            }
            uint8_t *out = codes + r * (cols / 2) + b * 8;
            for (int j = 0; j < 8; j++)
                out[j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
    }
    return 0;
}

/* Quantize from any source dtype (see ora_source_to_f32). */
int ora_quantize(const void *src, int dtype, const float *fp8_scale, int64_t rows, int64_t cols,
                 const float *amax_in, uint8_t *codes, uint8_t *scales_lin, uint8_t *scales_swz,
                 float *sg_out)
{
    float *x = (float *)malloc((size_t)(rows * cols > 0 ? rows * cols : 1) * 4);
    if (!x)
        return -2;
    ora_source_to_f32(src, dtype, fp8_scale, rows * cols, x);
    int rc = ora_quantize_f32(x, rows, cols, amax_in, codes, scales_lin, scales_swz, sg_out);
    free(x);
    return rc;
}

/* weight = E2M1 x block scale x global scale [QIb], in fp32, multiplied in that order. */
void ora_dequantize_f32(const uint8_t *codes, const uint8_t *scales_lin, float sg, int64_t rows,
                        int64_t cols, float *out)
{
    int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t k = 0; k < cols; k++) {
            uint8_t byte = codes[r * (cols / 2) + k / 2];
            int code = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
            float e = (float)ora_e2m1_decode(code);
            float s = (float)ora_e4m3_decode(scales_lin[r * nb + k / 16]);
            float es = e * s;
            out[r * cols + k] = es * sg;
        }
    }
}

void ora_dequantize_bf16(const uint8_t *codes, const uint8_t *scales_lin, float sg, int64_t rows,
                         int64_t cols, uint16_t *out)
{
    float *tmp = (float *)malloc((size_t)(rows * cols > 0 ? rows * cols : 1) * 4);
    ora_dequantize_f32(codes, scales_lin, sg, rows, cols, tmp);
    for (int64_t i = 0; i < rows * cols; i++)
        out[i] = ora_f32_to_bf16(tmp[i]);
    free(tmp);
}

/* ------------------------------------------------------------------------------------------ */
/* GEMM over decoded values, fp64                                                              */
/* ------------------------------------------------------------------------------------------ */

/* One output of Y = dequant(A) . dequant(W)^T: decode both rows exactly and accumulate in
 * fp64: Y[m,n] = sgA*sgW * sum_b sA[m,b]*sW[n,b] * sum_{k in b} eA[m,k]*eW[n,k]. */
static double gemm_one(const uint8_t *a_codes, const uint8_t *a_sc, float a_sg,
                       const uint8_t *w_codes, const uint8_t *w_sc, float w_sg,
                       int64_t m, int64_t n, int64_t K)
{
    int64_t nb = K / 16;
    double acc = 0.0;
    for (int64_t b = 0; b < nb; b++) {
        double inner = 0.0;
        for (int64_t j = 0; j < 16; j++) {
            int64_t k = b * 16 + j;
            uint8_t ab = a_codes[m * (K / 2) + k / 2];
            uint8_t wb = w_codes[n * (K / 2) + k / 2];
            int ac = (k % 2 == 0) ? (ab & 15) : (ab >> 4);
            int wc = (k % 2 == 0) ? (wb & 15) : (wb >> 4);
            inner += ora_e2m1_decode(ac) * ora_e2m1_decode(wc);
        }
        acc += ora_e4m3_decode(a_sc[m * nb + b]) * ora_e4m3_decode(w_sc[n * nb + b]) * inner;
    }
    return (double)a_sg * (double)w_sg * acc;
}

/* Full product, out [M x N] row-major. */
void ora_gemm_f64(const uint8_t *a_codes, const uint8_t *a_scales_lin, float a_sg,
                  const uint8_t *w_codes, const uint8_t *w_scales_lin, float w_sg,
                  int64_t M, int64_t N, int64_t K, double *out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++)
            out[m * N + n] = gemm_one(a_codes, a_scales_lin, a_sg, w_codes, w_scales_lin, w_sg,
                                      m, n, K);
}

/* Selected outputs (ms[i], ns[i]) only, for checks at sizes where the full product is slow. */
void ora_gemm_f64_sampled(const uint8_t *a_codes, const uint8_t *a_scales_lin, float a_sg,
                          const uint8_t *w_codes, const uint8_t *w_scales_lin, float w_sg,
                          int64_t K, const int64_t *ms, const int64_t *ns, int64_t count,
                          double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++)
        out[i] = gemm_one(a_codes, a_scales_lin, a_sg, w_codes, w_scales_lin, w_sg, ms[i], ns[i],
                          K);
}

/* ------------------------------------------------------------------------------------------ */
/* Linear layer with an NVFP4 output (a producer epilogue)                                     */
/* ------------------------------------------------------------------------------------------ */
/* [QRc] "Recommended Model": with static input scales from calibration, the next layer's input
 * can be quantized where it is produced. Readings where the pages are silent (design notes):
 *   - acc = sum_b sA[m,b] sW[n,b] sum_k eA eW (exact), y = RN32(RN32(acc) * RN32(sgA * sgW)):
 *     the fp32 product the tensor cores accumulate, scaled as the linear layer's epilogue does;
 *   - activation act: 0 identity; 1 GELU in its tanh form,
 *     gelu(y) = 0.5 y (1 + tanh(u)) = y / (1 + exp(-2 u)), u = sqrt(2/pi) (y + 0.044715 y^3),
 *     evaluated in fp64 (the second form: no cancellation for negative y) and rounded to fp32;
 *   - the activation output is NVFP4-quantized with the static amax (ora_quantize_f32). */

double ora_gelu_tanh_f64(double y)
{
    double u = 0.7978845608028654 * (y + 0.044715 * y * y * y);
    return y / (1.0 + exp(-2.0 * u));
}

static double act_f64(double y, int act) { return act == 1 ? ora_gelu_tanh_f64(y) : y; }

/* acc without the global scales (see gemm_one). */
static double block_sum(const uint8_t *a_codes, const uint8_t *a_sc, const uint8_t *w_codes,
                        const uint8_t *w_sc, int64_t m, int64_t n, int64_t K)
{
    return gemm_one(a_codes, a_sc, 1.0f, w_codes, w_sc, 1.0f, m, n, K);
}

/* fp64 activation of the exact product sgA sgW acc: the value the fused layer approximates. */
void ora_linear_act_f64_sampled(const uint8_t *a_codes, const uint8_t *a_sc, float a_sg,
                                const uint8_t *w_codes, const uint8_t *w_sc, float w_sg,
                                int64_t K, int act, const int64_t *ms, const int64_t *ns,
                                int64_t count, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++)
        out[i] = act_f64((double)a_sg * (double)w_sg *
                             block_sum(a_codes, a_sc, w_codes, w_sc, ms[i], ns[i], K),
                         act);
}

/* act applied in fp64 to each of n values (y = an exact product from ora_gemm_f64, whose
 * scaling sgA * sgW * acc is the same expression as above). */
void ora_act_f64_array(const double *y, int64_t n, int act, double *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = act_f64(y[i], act);
}

/* The fused layer's NVFP4 output [M x N]: y as above, v = act(y) in fp32, quantized with the
 * static amax. Returns 0, or -1 if N is not a multiple of 16, -2 on allocation failure. */
int ora_linear_quantize_out(const uint8_t *a_codes, const uint8_t *a_sc, float a_sg,
                            const uint8_t *w_codes, const uint8_t *w_sc, float w_sg, int64_t M,
                            int64_t N, int64_t K, float static_amax, int act, uint8_t *codes,
                            uint8_t *scales_lin, uint8_t *scales_swz, float *sg_out)
{
    if (N % 16 != 0)
        return -1;
    float *v = (float *)malloc((size_t)(M * N > 0 ? M * N : 1) * sizeof(float));
    if (!v)
        return -2;
    const float alpha = a_sg * w_sg;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            float acc = (float)block_sum(a_codes, a_sc, w_codes, w_sc, m, n, K);
            float y = acc * alpha;
            v[m * N + n] = act == 1 ? (float)ora_gelu_tanh_f64((double)y) : y;
        }
    int rc = ora_quantize_f32(v, M, N, &static_amax, codes, scales_lin, scales_swz, sg_out);
    free(v);
    return rc;
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 E4M3 tensorwise layers                                                                  */
/* ------------------------------------------------------------------------------------------ */
/* [QVf] "Qwen3-VL-8B-Instruct-heretic-NVFP4", "Quantization Details" and "Layer breakdown":
 *       embed_tokens and lm_head are float8_e4m3fn, tensorwise, round-to-nearest; "Runtime /
 *       hardware": FP8 layers run as native FP8 on Blackwell.
 * [QRp] "Qwen-Rapid-AIO FP8 -> NVFP4", the "Solution" table and the paragraph under it: layers
 *       that are FP8 stay FP8 (no re-quantization through fp32).
 * Readings where the pages are silent (also in the design notes):
 *   - one fp32 scale per tensor, s = amax / 448 (fp32 division): the largest |x| maps to the
 *     largest finite E4M3 value; amax is the tensor's own (dynamic) or a static value, above
 *     which values saturate.
 *   - code = sign(x) | E4M3(|x| / s): the quotient is an IEEE fp32 division, rounded to the
 *     nearest E4M3 value, ties to the even code, saturating at 448; s == 0 gives sign-only codes.
 *   - the linear layer is W8A8: activations quantized the same way from their dynamic amax, and
 *     Y[m,n] = sA * sW * sum_k eA[m,k] * eW[n,k].
 */

/* E4M3 codes of n fp32 values with one tensor scale; returns s. */
float ora_quantize_e4m3_f32(const float *x, int64_t n, const float *amax_in, uint8_t *codes)
{
    float amax = amax_in ? *amax_in : ora_amax(x, n);
    float s = amax / 448.0f;
    for (int64_t i = 0; i < n; i++) {
        uint8_t sign = signbit(x[i]) ? 0x80 : 0x00;
        uint8_t mag = (s > 0.0f) ? ora_e4m3_encode_nonneg(fabsf(x[i]) / s) : 0;
        codes[i] = (uint8_t)(sign | mag);
    }
    return s;
}

/* Source of dtype 0 (fp32) or 1 (bf16 bits); returns 0, or -1 for another dtype. */
int ora_quantize_e4m3(const void *src, int dtype, int64_t n, const float *amax_in,
                      uint8_t *codes, float *scale_out)
{
    if (dtype != 0 && dtype != 1)
        return -1;
    float *x = (float *)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!x)
        return -2;
    ora_source_to_f32(src, dtype, NULL, n, x);
    *scale_out = ora_quantize_e4m3_f32(x, n, amax_in, codes);
    free(x);
    return 0;
}

/* One output of the W8A8 product: exact decodes, fp64 accumulation. */
static double gemm_e4m3_one(const uint8_t *a, float sa, const uint8_t *w, float sw, int64_t m,
                            int64_t n, int64_t K)
{
    double acc = 0.0;
    for (int64_t k = 0; k < K; k++)
        acc += ora_e4m3_decode(a[m * K + k]) * ora_e4m3_decode(w[n * K + k]);
    return (double)sa * (double)sw * acc;
}

/* Y [M x N] row-major from A codes [M x K] and W codes [N x K] (nn.Linear layout). */
void ora_gemm_e4m3_f64(const uint8_t *a, float sa, const uint8_t *w, float sw, int64_t M,
                       int64_t N, int64_t K, double *out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++)
            out[m * N + n] = gemm_e4m3_one(a, sa, w, sw, m, n, K);
}

void ora_gemm_e4m3_f64_sampled(const uint8_t *a, float sa, const uint8_t *w, float sw, int64_t K,
                               const int64_t *ms, const int64_t *ns, int64_t count, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++)
        out[i] = gemm_e4m3_one(a, sa, w, sw, ms[i], ns[i], K);
}

/* ------------------------------------------------------------------------------------------ */
/* Percentile calibration                                                                      */
/* ------------------------------------------------------------------------------------------ */

static int cmp_float(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

/* Nearest-rank percentile of |x| over the union of the given fp32 arrays, plus the max.
 * rank = ceil(n * num / den), at least 1. Returns -1 on an empty input or bad ratio. */
int ora_percentile_abs(const float *const *arrays, const int64_t *lengths, int count,
                       uint32_t num, uint32_t den, float *pct, float *mx)
{
    int64_t n = 0;
    for (int i = 0; i < count; i++)
        n += lengths[i];
    if (n <= 0 || den == 0 || num > den)
        return -1;
    float *v = (float *)malloc((size_t)n * 4);
    if (!v)
        return -2;
    int64_t p = 0;
    for (int i = 0; i < count; i++)
        for (int64_t j = 0; j < lengths[i]; j++)
            v[p++] = fabsf(arrays[i][j]);
    qsort(v, (size_t)n, 4, cmp_float);
    uint64_t rank = ((uint64_t)n * num + den - 1) / den;
    if (rank < 1)
        rank = 1;
    *pct = v[rank - 1];
    *mx = v[n - 1];
    free(v);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Linear layer with a BF16 low-rank branch                                                    */
/* ------------------------------------------------------------------------------------------ */
/* "Qwen Image 2.1: INT4 + FP4", section "What I quantized": the transformer's linear layers
 * run in native FP4 on Blackwell together with BF16 rank-128 branches. Readings where the
 * page is silent (each also listed in the design notes):
 *   - a branch is a rank-r factorization U . D of a correction to the layer's weight, applied
 *     to the layer's unquantized bf16 input x:
 *       Y = dequant(A) . dequant(W)^T + (x . D^T) . U^T,  D [r x K] ("down"), U [N x r] ("up");
 *   - the branch runs in BF16: its intermediate T = x . D^T is a bf16 tensor, each element the
 *     exact sum rounded once to the nearest bf16 (ties to even);
 *   - the up product T . U^T and its sum with the FP4 product are exact (fp64) here; the
 *     tensor cores approximate them with fp32 accumulation. The caller rounds Y. */

/* fp64 -> nearest bf16 (ties to even) in one rounding, as bits. Finite inputs whose rounded
 * magnitude is below 2^128. bf16 keeps 8 significant bits; below 2^-126 the spacing stays
 * 2^-133 (subnormals). */
uint16_t ora_f64_to_bf16(double v)
{
    if (v == 0.0)
        return signbit(v) ? 0x8000u : 0u;
    int e;
    frexp(v, &e); /* |v| in [2^(e-1), 2^e) */
    if (e < -125)
        e = -125;
    double q = rint(ldexp(v, 8 - e)); /* round to a multiple of 2^(e-8); default mode: ties even */
    float f = (float)ldexp(q, e - 8);  /* exact: at most 9 significant bits, in range */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* T [M x r] (bf16 bits) = RNE_bf16(sum_k x[m,k] * d[j,k]), x [M x K], d [r x K] bf16 bits. */
static uint16_t lowrank_t(const uint16_t *x, const uint16_t *d, int64_t K, int64_t m, int64_t j)
{
    double s = 0.0;
    for (int64_t k = 0; k < K; k++)
        s += (double)ora_bf16_to_f32(x[m * K + k]) * (double)ora_bf16_to_f32(d[j * K + k]);
    return ora_f64_to_bf16(s);
}

void ora_lowrank_down_bf16(const uint16_t *x, const uint16_t *d, int64_t M, int64_t K,
                           int64_t r, uint16_t *t)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t j = 0; j < r; j++)
            t[m * r + j] = lowrank_t(x, d, K, m, j);
}

/* One output: the FP4 product (gemm_one) plus sum_j T[m,j] * U[n,j], T from row t_row. */
static double lowrank_one(const uint8_t *a_codes, const uint8_t *a_sc, float a_sg,
                          const uint8_t *w_codes, const uint8_t *w_sc, float w_sg,
                          const uint16_t *t_row, const uint16_t *u, int64_t m, int64_t n,
                          int64_t K, int64_t r)
{
    double lr = 0.0;
    for (int64_t j = 0; j < r; j++)
        lr += (double)ora_bf16_to_f32(t_row[j]) * (double)ora_bf16_to_f32(u[n * r + j]);
    return gemm_one(a_codes, a_sc, a_sg, w_codes, w_sc, w_sg, m, n, K) + lr;
}

/* Full output Y [M x N] in fp64. Returns 0, or -2 on allocation failure. */
int ora_linear_lowrank_f64(const uint8_t *a_codes, const uint8_t *a_sc, float a_sg,
                           const uint8_t *w_codes, const uint8_t *w_sc, float w_sg,
                           const uint16_t *x, const uint16_t *d, const uint16_t *u, int64_t M,
                           int64_t N, int64_t K, int64_t r, double *out)
{
    uint16_t *t = (uint16_t *)malloc((size_t)(M * r > 0 ? M * r : 1) * 2);
    if (!t)
        return -2;
    ora_lowrank_down_bf16(x, d, M, K, r, t);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++)
            out[m * N + n] = lowrank_one(a_codes, a_sc, a_sg, w_codes, w_sc, w_sg, t + m * r, u,
                                         m, n, K, r);
    free(t);
    return 0;
}

/* Selected outputs (ms[i], ns[i]); the needed row of T is recomputed per output. */
int ora_linear_lowrank_f64_sampled(const uint8_t *a_codes, const uint8_t *a_sc, float a_sg,
                                   const uint8_t *w_codes, const uint8_t *w_sc, float w_sg,
                                   const uint16_t *x, const uint16_t *d, const uint16_t *u,
                                   int64_t K, int64_t r, const int64_t *ms, const int64_t *ns,
                                   int64_t count, double *out)
{
    int err = 0;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++) {
        uint16_t *t_row = (uint16_t *)malloc((size_t)(r > 0 ? r : 1) * 2);
        if (!t_row) {
            err = -2;
            continue;
        }
        for (int64_t j = 0; j < r; j++)
            t_row[j] = lowrank_t(x, d, K, ms[i], j);
        out[i] = lowrank_one(a_codes, a_sc, a_sg, w_codes, w_sc, w_sg, t_row, u, ms[i], ns[i],
                             K, r);
        free(t_row);
    }
    return err;
}
