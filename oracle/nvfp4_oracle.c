/*
 * CPU oracle for NVFP4 two-level microblock quantization and the
 * block-scaled FP4 GEMM.  TEST INFRASTRUCTURE ONLY: it is used by tests/,
 * the smoke check and the CPU-baseline leg of bench.py, never by the
 * product path.  It shares no code with the CUDA library.
 *
 * What it follows:
 *  - "英伟达B200狂飙10.2倍！AI绘图告别龟速！" (nmedialink), section
 *    "NVFP4量化：在精度与速度之间寻得最佳平衡": NVFP4 uses two-level
 *    microblock scaling — one FP32 scale per tensor (static or dynamic)
 *    and one scale per block of 16 elements computed dynamically.
 *  - "Scaling NVFP4 Inference for FLUX.2 on NVIDIA Blackwell Data Center
 *    GPUs" (engineering.fyi), section "Key Questions Answered": the same
 *    two-level scaling with dynamic quantization.
 * The pages name neither the element nor the block-scale format; this
 * library uses the standard NVFP4 encoding: E2M1 elements and unsigned E4M3
 * block scales.  Every step the pages leave open is a stated reading:
 *   S_enc = 2688 / amax   (2688 = 6 * 448: E2M1 max times E4M3 max);
 *           amax == 0 -> 1; a non-finite result -> FLT_MAX
 *   per block: s = (a_b / 6) * S_enc  (two fp32 round-to-nearest ops)
 *              sf = E4M3(s), round to nearest, ties to even, saturating
 *              inv = (sf == 0) ? 0 : S_enc / sf, clamped to FLT_MAX if it
 *                    overflows (tensors with amax below ~1e-35)
 *              q_i = E2M1(x_i * inv), round to nearest even, saturating,
 *                    sign kept (a negative value that rounds to 0 is -0)
 *   packing: byte j of a row holds element 2j in the low nibble
 *   scale layout: 128x4 tiles of 512 bytes (see ref_sf_offset)
 *   dequantization and the GEMM are evaluated in fp64.
 *
 * All fp32 steps are single IEEE operations: build with -ffp-contract=off.
 * Encoders search the format's value table (no bit tricks) so that they can
 * be checked against the definitions by eye.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#pragma STDC FP_CONTRACT OFF

/* ---------------- element and scale formats ---------------- */

/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit, no inf/NaN.
 * Magnitudes of codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double ref_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? m * 0.5 : (1.0 + m * 0.5) * ldexp(1.0, e - 1);
    return s ? -mag : mag;
}

/* E4M3 "fn": 1 sign, 4 exponent (bias 7), 3 mantissa bits, no inf,
 * S.1111.111 is NaN, max finite 448, min subnormal 2^-9. */
double ref_e4m3_value(uint8_t code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? m * ldexp(1.0, -9) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return s ? -mag : mag;
}

/* Round a non-negative magnitude to the code of the nearest entry of an
 * ascending table of magnitudes (codes 0..n-1); ties go to the even code;
 * anything at or above the largest entry saturates to it. */
static uint8_t round_to_table(double v, const double *table, int n)
{
    if (!(v < table[n - 1])) return (uint8_t)(n - 1);   /* also +inf */
    int i = 0;
    while (table[i + 1] <= v) i++;                       /* table[i] <= v < table[i+1] */
    double mid = 0.5 * (table[i] + table[i + 1]);        /* exact in fp64 */
    if (v < mid) return (uint8_t)i;
    if (v > mid) return (uint8_t)(i + 1);
    return (uint8_t)((i % 2 == 0) ? i : i + 1);
}

static double g_e2m1_mag[8];
static double g_e4m3_mag[127];  /* codes 0x00..0x7E */
static int g_tables_ready = 0;

static void init_tables(void)
{
    if (g_tables_ready) return;
    for (int c = 0; c < 8; c++) g_e2m1_mag[c] = ref_e2m1_value((uint8_t)c);
    for (int c = 0; c < 127; c++) g_e4m3_mag[c] = ref_e4m3_value((uint8_t)c);
    g_tables_ready = 1;
}

uint8_t ref_e2m1_encode(float v)
{
    init_tables();
    int neg = signbit(v) ? 1 : 0;
    uint8_t c = round_to_table(fabs((double)v), g_e2m1_mag, 8);
    return (uint8_t)(c | (neg << 3));
}

uint8_t ref_e4m3_encode(float v)
{
    init_tables();
    int neg = signbit(v) ? 1 : 0;
    uint8_t c = round_to_table(fabs((double)v), g_e4m3_mag, 127);
    return (uint8_t)(c | (neg << 7));
}

/* ---------------- tensor-level scale ---------------- */

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* amax = max_i |x_i| over a bfloat16 tensor (exact). */
float ref_tensor_amax(const uint16_t *x, int64_t n)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float v = fabsf(bf16_to_float(x[i]));
        if (v > a) a = v;
    }
    return a;
}

/* Per-tensor encode scale S_enc = (6 * 448) / amax. */
float ref_tensor_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    float s = 2688.0f / amax;
    if (!isfinite(s)) s = FLT_MAX;
    return s;
}

/* Per-tensor decode scale S_dec = 1 / S_enc. */
float ref_decode_scale(float s_enc)
{
    return 1.0f / s_enc;
}

/* ---------------- scale-factor layout ---------------- */

int64_t ref_sf_bytes(int64_t rows, int64_t cols)
{
    int64_t kb = cols / 16;
    return ((rows + 127) / 128 * 128) * ((kb + 3) / 4 * 4);
}

/* Byte offset of the scale of (row r, block c) when a row has kb blocks:
 * 128-row x 4-block tiles of 512 bytes, tiles ordered row-block-major;
 * inside a tile, row r sits in 16-byte line r%32 at 4-byte slot (r/32)%4,
 * and block c at byte c%4 of that slot. */
int64_t ref_sf_offset(int64_t r, int64_t c, int64_t kb)
{
    int64_t kb4 = (kb + 3) / 4;
    int64_t tile = (r / 128) * kb4 + c / 4;
    return tile * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);
}

/* ---------------- quantization ---------------- */

/* Quantize one block of 16 values; returns the E4M3 scale code and writes
 * 16 E2M1 codes. */
static uint8_t quantize_block(const float *x, float s_enc, uint8_t *codes)
{
    float a = 0.0f;
    for (int i = 0; i < 16; i++) {
        float v = fabsf(x[i]);
        if (v > a) a = v;
    }
    float s = a / 6.0f;
    s = s * s_enc;
    uint8_t sf = ref_e4m3_encode(s);
    float sfv = (float)ref_e4m3_value(sf);
    float inv = (sfv == 0.0f) ? 0.0f : s_enc / sfv;
    if (!isfinite(inv)) inv = FLT_MAX;   /* only when S_enc is near FLT_MAX */
    for (int i = 0; i < 16; i++) codes[i] = ref_e2m1_encode(x[i] * inv);
    return sf;
}

/* x: bfloat16 [rows, cols] row-major, cols % 16 == 0.
 * q: [rows, cols/2] packed, low nibble = even element.
 * sf: ref_sf_bytes(rows, cols) bytes in the tiled layout, padding zero. */
void ref_quantize(const uint16_t *x, int64_t rows, int64_t cols, float s_enc,
                  uint8_t *q, uint8_t *sf)
{
    init_tables();
    int64_t kb = cols / 16;
    memset(sf, 0, (size_t)ref_sf_bytes(rows, cols));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float blk[16];
        uint8_t codes[16];
        for (int64_t c = 0; c < kb; c++) {
            for (int i = 0; i < 16; i++) blk[i] = bf16_to_float(x[r * cols + c * 16 + i]);
            sf[ref_sf_offset(r, c, kb)] = quantize_block(blk, s_enc, codes);
            for (int j = 0; j < 8; j++)
                q[r * (cols / 2) + c * 8 + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
    }
}

/* ---------------- dequantization and GEMM ---------------- */

/* x_hat[r,k] = e2m1(q) * e4m3(sf) * s_dec, in fp64, for the listed rows
 * (row_idx == NULL: all rows). */
void ref_dequantize(const uint8_t *q, const uint8_t *sf, float s_dec,
                    int64_t rows, int64_t cols, const int64_t *row_idx,
                    int64_t n_idx, double *out)
{
    init_tables();
    int64_t kb = cols / 16;
    int64_t n = row_idx ? n_idx : rows;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        int64_t r = row_idx ? row_idx[i] : i;
        for (int64_t k = 0; k < cols; k++) {
            uint8_t byte = q[r * (cols / 2) + k / 2];
            uint8_t code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double scale = ref_e4m3_value(sf[ref_sf_offset(r, k / 16, kb)]);
            out[i * cols + k] = ref_e2m1_value(code) * scale * (double)s_dec;
        }
    }
}

/* Brute-force y[m,n] = sum_k a[m,k] * b[n,k] in fp64, k ascending. */
void ref_gemm_naive(const double *a, const double *b, int64_t M, int64_t N,
                    int64_t K, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) acc += a[m * K + k] * b[n * K + k];
            y[m * N + n] = acc;
        }
}

/* ---------------- FP8 (E4M3) variant with one FP32 per-tensor scale ----------------
 * The pages select an FP8 mode beside NVFP4 ("NVIDIA показала, как
 * сократить генерацию FLUX 3 Image Klein с 22 до 6 секунд", section "2.
 * Запуск генерации изображения": --variant fp8r) without describing its
 * scaling; the reading taken is the plainest one: E4M3 elements with one
 * FP32 scale per tensor, S_enc = 448 / amax (the E4M3 maximum over the tensor
 * amax; 1 if amax == 0, FLT_MAX if not finite), q = E4M3_rn_satfinite(x * S_enc)
 * with the sign kept, S_dec = 1 / S_enc. */
float ref_fp8_tensor_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    float s = 448.0f / amax;
    if (!isfinite(s)) s = FLT_MAX;
    return s;
}

void ref_quantize_fp8(const uint16_t *x, int64_t n, float s_enc, uint8_t *q)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        float v = bf16_to_float(x[i]) * s_enc;
        q[i] = ref_e4m3_encode(v);
    }
}

int ref_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
