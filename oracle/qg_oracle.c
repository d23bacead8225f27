/*
 * qg_oracle.c -- plain, slow CPU oracle for the quantized-GEMM hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may include, link or call this file.  Only the tests,
 * the smoke check and the benchmark's CPU-baseline leg use it.  It shares no
 * code, header, table or helper with the CUDA path.
 *
 * Every routine is the plain definition written out: per-element loops in the
 * order the pages state them, integer products accumulated in int64, floating
 * products accumulated in fp64.  The only concession to speed is an OpenMP
 * "parallel for" over independent output rows, which does not change any
 * result (each output element is still produced by one thread, in loop order).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 * (no fused multiply-add contraction, no fast-math: the quantizers must be
 * IEEE-754 binary32 operations with round-to-nearest-even, as written).
 *
 * Sources (web pages on INT8/INT4 quantized GEMM):
 *  - "量化算法的本质 / per_channel_quant_int8" (hotelren.com/news/2718779):
 *    symmetric per-row quant: absmax.clamp_min(1e-10), x*(127/absmax), round;
 *    W8A8: Y = (x_scale*X) @ (w_scale*W) + bias; X row-major [M,K],
 *    W column-major [K,N] with stride [1,K]; GPTQ group quant clamp 1e-5.
 *  - "量化与多精度算子" (quant67.com, §二 §四 §六): q = round(x/s)+z,
 *    x ~= s(q-z); symmetric range [-127,127]; INT32 accumulation; clamp.
 *  - "从零实现大语言模型 INT8 量化" (zingnex.cn, 第一步/第二步): block of 64,
 *    scale = (max-min)/(levels-1), zero = round(-min/scale),
 *    q = round(w/scale) + zero.
 *  - "INT4/FP16混合精度GEMM" (xdnf.cn, §3.2 §4.2): unpack (w >> 4i) & 0xF,
 *    dequant (q - zp) * scale, FP16 matmul with FP32 accumulate.
 *  - "Ascend C per-channel INT8 GEMM" (2048ai.net, §五 5.4): int32 accumulate,
 *    multiply by the per-column scale at write-back.
 *
 * Readings where the pages are silent or disagree (round half to even; the
 * symmetric multiply order x*(127/a); fp16 scale used for quantizing; 8 nibbles
 * per 32-bit word, low nibble first; scale/zero laid out [K/group, N]) are the
 * ones listed with the design notes of this repository.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16 / bfloat16 codecs, written from the bit layouts.        */
/* ------------------------------------------------------------------------ */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Normal: (1024 + frac) * 2^(exp - 25); subnormal: frac * 2^-24. */
double oracle_f16_bits_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

float oracle_f16_bits_to_f32(uint16_t h) { return (float)oracle_f16_bits_to_f64(h); }

/* bfloat16: the upper 16 bits of a binary32. */
double oracle_bf16_bits_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a finite double to p significand bits with minimum normal exponent
 * emin, ties to even.  Below 2^emin the quantum stays 2^(emin-p+1)
 * (gradual underflow).  Scaling by a power of two is exact, and nearbyint()
 * rounds to nearest-even in the default rounding mode. */
static double round_to_precision(double a, int p, int emin)
{
    if (a == 0.0 || !isfinite(a))
        return a;
    int e2;
    (void)frexp(fabs(a), &e2);   /* |a| = f * 2^e2, f in [0.5, 1) */
    int ea = e2 - 1;             /* exponent of the leading bit */
    int qe = (ea < emin ? emin : ea) - (p - 1);
    double r = nearbyint(ldexp(fabs(a), -qe));
    return copysign(ldexp(r, qe), a);
}

/* Encode a double as binary16, rounding to nearest even. */
uint16_t oracle_f64_to_f16_bits(double a)
{
    if (isnan(a))
        return 0x7E00;
    uint16_t sign = signbit(a) ? 0x8000 : 0;
    double r = fabs(round_to_precision(a, 11, -14));
    if (r > 65504.0)
        return sign | 0x7C00; /* overflow to infinity */
    if (r < ldexp(1.0, -14))  /* subnormal (or zero): count of 2^-24 quanta */
        return sign | (uint16_t)ldexp(r, 24);
    int e2;
    (void)frexp(r, &e2);
    int ea = e2 - 1;
    uint16_t frac = (uint16_t)(ldexp(r, 10 - ea) - 1024.0);
    return sign | (uint16_t)((ea + 15) << 10) | frac;
}

uint16_t oracle_f32_to_f16_bits(float f) { return oracle_f64_to_f16_bits((double)f); }

/* Encode a double as bfloat16 (8 significand bits, binary32 exponent range). */
uint16_t oracle_f64_to_bf16_bits(double a)
{
    if (isnan(a))
        return 0x7FC0;
    double r = round_to_precision(a, 8, -126);
    double maxf = ldexp(255.0, 127 - 7); /* (2 - 2^-7) * 2^127 */
    if (fabs(r) > maxf)
        return signbit(a) ? 0xFF80 : 0x7F80;
    float f = (float)r; /* exact: r has 8 significand bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* a1 / a2: symmetric per-row int8 quantization.                             */
/* ------------------------------------------------------------------------ */

/* For every row m of X (fp16, row-major, leading dimension ldx):
 *   a       = max_k |x[m,k]|, then a = max(a, 1e-10)         (clamp_min)
 *   inv     = 127 / a                                         (binary32 division)
 *   q[m,k]  = clamp(round_half_even(x[m,k] * inv), -127, 127) (binary32 product)
 *   scale[m]= a / 127                                          (binary32 division)
 * Applied to the [N,K] storage of a column-major weight it is the per-output-
 * column weight quantizer (one scale per column n). */
void ref_quantize_rowwise_int8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                               int8_t *q, int64_t ldq, float *scale)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t *row = x + m * ldx;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(oracle_f16_bits_to_f32(row[k]));
            if (v > a)
                a = v;
        }
        if (a < 1e-10f)
            a = 1e-10f;
        float inv = 127.0f / a;
        for (int64_t k = 0; k < K; ++k) {
            float t = oracle_f16_bits_to_f32(row[k]) * inv;
            float r = rintf(t);
            if (r > 127.0f)
                r = 127.0f;
            if (r < -127.0f)
                r = -127.0f;
            q[m * ldq + k] = (int8_t)r;
        }
        scale[m] = a / 127.0f;
    }
}

/* ------------------------------------------------------------------------ */
/* a2: block-wise asymmetric 4-bit weight quantization and packing.          */
/* ------------------------------------------------------------------------ */

/* W is the [N,K] storage of a column-major [K,N] fp16 weight (ldw >= K).
 * For every column n and every block b of `group` consecutive k:
 *   mn, mx  = min and max of the block
 *   s32     = max((mx - mn) / 15, 1e-5)           (binary32)
 *   s       = fp16(s32) (stored; quantizing uses this rounded value)
 *   z       = clamp(round_half_even(-mn / s), 0, 15), stored as fp16
 *   q[n,k]  = clamp(round_half_even(w / s) + z, 0, 15)
 * Packing: qweight[n, p] holds k = 8p .. 8p+7, nibble j at bits 4j..4j+3.
 * scale and zero are [K/group, N] row-major.  q_out (nullable) receives the
 * unpacked codes [N,K]. */
void ref_quantize_block_asym4(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int64_t group,
                              uint32_t *qweight, uint16_t *scale, uint16_t *zero, uint8_t *q_out)
{
    int64_t nblk = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * ldw;
        for (int64_t p = 0; p < K / 8; ++p)
            qweight[n * (K / 8) + p] = 0u;
        for (int64_t b = 0; b < nblk; ++b) {
            float mn = INFINITY, mx = -INFINITY;
            for (int64_t k = b * group; k < (b + 1) * group; ++k) {
                float v = oracle_f16_bits_to_f32(row[k]);
                if (v < mn)
                    mn = v;
                if (v > mx)
                    mx = v;
            }
            float s32 = (mx - mn) / 15.0f;
            if (s32 < 1e-5f)
                s32 = 1e-5f;
            uint16_t sh = oracle_f32_to_f16_bits(s32);
            float s = oracle_f16_bits_to_f32(sh);
            float zr = rintf(-mn / s);
            int zi = zr < 0.0f ? 0 : (zr > 15.0f ? 15 : (int)zr); /* integer code 0..15 */
            float z = (float)zi;
            scale[b * N + n] = sh;
            zero[b * N + n] = oracle_f32_to_f16_bits(z);
            for (int64_t k = b * group; k < (b + 1) * group; ++k) {
                float v = oracle_f16_bits_to_f32(row[k]);
                float t = rintf(v / s) + z;
                if (t < 0.0f)
                    t = 0.0f;
                if (t > 15.0f)
                    t = 15.0f;
                uint32_t code = (uint32_t)t;
                qweight[n * (K / 8) + k / 8] |= code << (4 * (k % 8));
                if (q_out)
                    q_out[n * K + k] = (uint8_t)code;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a3: integer GEMM with int64 accumulation.                                 */
/* ------------------------------------------------------------------------ */

/* acc[m,n] = sum_k xq[m,k] * wq[k,n]; xq row-major [M,K] (ldx), wq column-major
 * [K,N] stored as [N,K] (ldw).  acc is [M,N] row-major int64. */
void ref_gemm_i8_i64(const int8_t *xq, int64_t ldx, const int8_t *wq, int64_t ldw,
                     int64_t M, int64_t N, int64_t K, int64_t *acc)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)xq[m * ldx + k] * (int64_t)wq[n * ldw + k];
            acc[m * N + n] = s;
        }
}

/* a4: the W8A8 epilogue in fp64:
 * y[m,n] = acc[m,n] * x_scale[m] * w_scale[n] + bias[n]   (bias nullable). */
void ref_w8a8_epilogue_f64(const int64_t *acc, const float *x_scale, const float *w_scale,
                           const float *bias, int64_t M, int64_t N, double *y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double v = (double)acc[m * N + n] * (double)x_scale[m] * (double)w_scale[n];
            if (bias)
                v += (double)bias[n];
            y[m * N + n] = v;
        }
}

/* a3+a4 in one call (what the CPU baseline times): int64 accumulate, then the
 * fp64 epilogue, one output row at a time. */
void ref_w8a8_f64(const int8_t *xq, int64_t ldx, const int8_t *wq, int64_t ldw,
                  const float *x_scale, const float *w_scale, const float *bias,
                  int64_t M, int64_t N, int64_t K, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)xq[m * ldx + k] * (int64_t)wq[n * ldw + k];
            double v = (double)s * (double)x_scale[m] * (double)w_scale[n];
            if (bias)
                v += (double)bias[n];
            y[m * N + n] = v;
        }
}

/* ------------------------------------------------------------------------ */
/* NEXT-2: asymmetric per-row int8 and the zero-point W8A8 product.           */
/* ------------------------------------------------------------------------ */

/* Asymmetric per-row int8 quantization.  The affine form of page
 * "量化与多精度算子" §二: x ~= s (q - z), q = round(x / s) + z, with the int8
 * range [-128, 127]; page "量化算法的本质" gives, for the asymmetric case of its
 * per-row quantizer, the step s = (max - min) / 255 over the row, the floor 1e-8
 * on s, and a zero point that places the row minimum at code -128 (z = -min/s
 * - 128, not rounded to an integer).  Readings of this library where the pages
 * leave the binary32 details open: every step is one binary32 operation; the
 * offset is added before rounding, q = round_half_even(x / s + z) (so a real z
 * shifts the rounding grid instead of being rounded itself); codes are clamped
 * to [-128, 127].  For an empty row min = max = 0, so s = 1e-8 and z = -128.
 * qsum[m] = sum_k q[m,k] (the row sum of the codes, exact), used by the
 * zero-point GEMM's correction terms. */
void ref_quantize_rowwise_asym_int8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                                    int8_t *q, int64_t ldq, float *scale, float *zero,
                                    int32_t *qsum)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t *row = x + m * ldx;
        float mn = 0.0f, mx = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = oracle_f16_bits_to_f32(row[k]);
            if (k == 0 || v < mn)
                mn = v;
            if (k == 0 || v > mx)
                mx = v;
        }
        float s = (mx - mn) / 255.0f;
        if (s < 1e-8f)
            s = 1e-8f;
        float z = -mn / s - 128.0f;
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            float t = oracle_f16_bits_to_f32(row[k]) / s + z;
            float r = rintf(t);
            if (r > 127.0f)
                r = 127.0f;
            if (r < -128.0f)
                r = -128.0f;
            q[m * ldq + k] = (int8_t)r;
            sum += (int64_t)r;
        }
        scale[m] = s;
        zero[m] = z;
        if (qsum)
            qsum[m] = (int32_t)sum;
    }
}

/* Zero-point W8A8 (page "量化与多精度算子" §二: x ~= s_x (q_x - z_x),
 * w ~= s_w (q_w - z_w), and the product of the two), straight from the
 * definition: dequantize both operands in fp64 and sum the products.
 *   y[m,n] = sum_k x_scale[m] (xq[m,k] - x_zero[m]) * w_scale[n] (wq[k,n] - w_zero[n]) + bias[n]
 * x_zero / w_zero may be NULL (a symmetric operand, z = 0); bias nullable.
 * wq is the [N,K] storage of the column-major [K,N] weight. */
void ref_w8a8_zp_f64(const int8_t *xq, int64_t ldx, const float *x_scale, const float *x_zero,
                     const int8_t *wq, int64_t ldw, const float *w_scale, const float *w_zero,
                     const float *bias, int64_t M, int64_t N, int64_t K, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const double xs = x_scale[m], ws = w_scale[n];
            const double xz = x_zero ? (double)x_zero[m] : 0.0;
            const double wz = w_zero ? (double)w_zero[n] : 0.0;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double xv = xs * ((double)xq[m * ldx + k] - xz);
                double wv = ws * ((double)wq[n * ldw + k] - wz);
                s += xv * wv;
            }
            if (bias)
                s += (double)bias[n];
            y[m * N + n] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* NEXT-3: symmetric int4 weights (page "INT4/FP16混合精度GEMM" §5.1:        */
/* scale = max|w| / 7, q = round(w / scale), int4 range [-8, 7]) and the     */
/* int4-into-int8 product (page "Ascend C per-channel INT8 GEMM" §9.1:       */
/* unpack int4 to int8, then the int8 matmul).                               */
/* ------------------------------------------------------------------------ */

/* Two's-complement nibble of an int4 code (bits 0..3). */
static uint32_t nibble_of(int q) { return (uint32_t)q & 0xFu; }

/* Sign-extended int4 code of nibble j (bits 4j..4j+3) of a packed word. */
static int code_of(uint32_t word, int j)
{
    int v = (int)((word >> (4 * j)) & 0xFu);
    return v >= 8 ? v - 16 : v;
}

/* Block-wise symmetric int4 (blocks of `group` consecutive k of one column):
 *   s32 = max(max|w| / 7, 1e-5)     (binary32; the 1e-5 floor as in the
 *                                    asymmetric block quantizer)
 *   s   = fp16(s32), stored; quantizing uses this rounded value
 *   q   = clamp(round_half_even(w / s), -8, 7)
 * Packing: qweight[n, p] holds k = 8p..8p+7, nibble j (two's complement) at
 * bits 4j.  scale is [K/group, N] fp16.  q_out (nullable): codes [N,K]. */
void ref_quantize_block_sym4(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int64_t group,
                             uint32_t *qweight, uint16_t *scale, int8_t *q_out)
{
    int64_t nblk = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * ldw;
        for (int64_t p = 0; p < K / 8; ++p)
            qweight[n * (K / 8) + p] = 0u;
        for (int64_t b = 0; b < nblk; ++b) {
            float a = 0.0f;
            for (int64_t k = b * group; k < (b + 1) * group; ++k) {
                float v = fabsf(oracle_f16_bits_to_f32(row[k]));
                if (v > a)
                    a = v;
            }
            float s32 = a / 7.0f;
            if (s32 < 1e-5f)
                s32 = 1e-5f;
            uint16_t sh = oracle_f32_to_f16_bits(s32);
            float s = oracle_f16_bits_to_f32(sh);
            scale[b * N + n] = sh;
            for (int64_t k = b * group; k < (b + 1) * group; ++k) {
                float t = rintf(oracle_f16_bits_to_f32(row[k]) / s);
                if (t < -8.0f)
                    t = -8.0f;
                if (t > 7.0f)
                    t = 7.0f;
                qweight[n * (K / 8) + k / 8] |= nibble_of((int)t) << (4 * (k % 8));
                if (q_out)
                    q_out[n * K + k] = (int8_t)t;
            }
        }
    }
}

/* Per-output-column symmetric int4 for the int8 tensor path:
 *   a = max(max_k |w[n,k]|, 1e-10);  s = a / 7   (binary32, kept in fp32)
 *   q = clamp(round_half_even(w / s), -8, 7)     (binary32 division)
 * Same packing as above; scale is float32 [N]. */
void ref_quantize_channel_sym4(const uint16_t *w, int64_t N, int64_t K, int64_t ldw,
                               uint32_t *qweight, float *scale, int8_t *q_out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * ldw;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(oracle_f16_bits_to_f32(row[k]));
            if (v > a)
                a = v;
        }
        if (a < 1e-10f)
            a = 1e-10f;
        float s = a / 7.0f;
        scale[n] = s;
        for (int64_t p = 0; p < K / 8; ++p)
            qweight[n * (K / 8) + p] = 0u;
        for (int64_t k = 0; k < K; ++k) {
            float t = rintf(oracle_f16_bits_to_f32(row[k]) / s);
            if (t < -8.0f)
                t = -8.0f;
            if (t > 7.0f)
                t = 7.0f;
            qweight[n * (K / 8) + k / 8] |= nibble_of((int)t) << (4 * (k % 8));
            if (q_out)
                q_out[n * K + k] = (int8_t)t;
        }
    }
}

/* W4A8: y[m,n] = x_scale[m] * w_scale[n] * sum_k xq[m,k] * q4[k,n] + bias[n],
 * q4 the sign-extended nibbles (the unpacked int8 codes); int64 accumulation,
 * fp64 epilogue. */
void ref_w4a8_f64(const int8_t *xq, int64_t ldx, const uint32_t *qweight, const float *x_scale,
                  const float *w_scale, const float *bias, int64_t M, int64_t N, int64_t K, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k)
                acc += (int64_t)xq[m * ldx + k] * (int64_t)code_of(qweight[n * (K / 8) + k / 8], (int)(k % 8));
            double v = (double)acc * (double)x_scale[m] * (double)w_scale[n];
            if (bias)
                v += (double)bias[n];
            y[m * N + n] = v;
        }
}

/* Symmetric group-int4 W4A16: y[m,n] = sum_k x[m,k] * q4[k,n] * s[k/group, n] + bias[n]
 * (fp64; s the stored fp16 scale). */
void ref_w4a16_sym_f64(const uint16_t *x, int64_t ldx, const uint32_t *qweight, const uint16_t *scale,
                       int64_t group, const float *bias, int64_t M, int64_t N, int64_t K, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double wv = (double)code_of(qweight[n * (K / 8) + k / 8], (int)(k % 8)) *
                            oracle_f16_bits_to_f64(scale[(k / group) * N + n]);
                s += oracle_f16_bits_to_f64(x[m * ldx + k]) * wv;
            }
            if (bias)
                s += (double)bias[n];
            y[m * N + n] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* NEXT-4: activation after the GEMM (page "INT4/FP16混合精度GEMM" §8,        */
/* fused linear_gelu: y = GEMM(...), then gelu(y) without writing y back).   */
/* ------------------------------------------------------------------------ */

/* GELU from its definition, y * Phi(y) with Phi the standard normal CDF:
 *   gelu(y) = 0.5 * y * (1 + erf(y / sqrt(2)))     (fp64, C99 erf) */
void ref_gelu_f64(const double *y, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = 0.5 * y[i] * (1.0 + erf(y[i] / sqrt(2.0)));
}

/* ------------------------------------------------------------------------ */
/* a5: weight-only int8 (W8A16): fp64 product with the dequantized weights.  */
/* ------------------------------------------------------------------------ */

/* y[m,n] = sum_k x[m,k] * (w_scale[n] * wq[k,n]) + bias[n]; x fp16 row-major. */
void ref_w8a16_f64(const uint16_t *x, int64_t ldx, const int8_t *wq, int64_t ldw,
                   const float *w_scale, const float *bias, int64_t M, int64_t N, int64_t K, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double wdq = (double)w_scale[n] * (double)wq[n * ldw + k];
                s += oracle_f16_bits_to_f64(x[m * ldx + k]) * wdq;
            }
            if (bias)
                s += (double)bias[n];
            y[m * N + n] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* a6: weight-only 4-bit block-asymmetric (W4A16).                          */
/* ------------------------------------------------------------------------ */

/* Dequantized weight of (k, n): w = (q - z) * s with b = k / group,
 * q = (qweight[n, k/8] >> 4*(k%8)) & 0xF, s = scale[b, n], z = zero[b, n]. */
double ref_w4_dequant(const uint32_t *qweight, const uint16_t *scale, const uint16_t *zero,
                      int64_t N, int64_t K, int64_t group, int64_t k, int64_t n)
{
    uint32_t word = qweight[n * (K / 8) + k / 8];
    double q = (double)((word >> (4 * (k % 8))) & 0xFu);
    int64_t b = k / group;
    double s = oracle_f16_bits_to_f64(scale[b * N + n]);
    double z = oracle_f16_bits_to_f64(zero[b * N + n]);
    return (q - z) * s;
}

/* y[m,n] = sum_k x[m,k] * w(k,n) + bias[n], all in fp64. */
void ref_w4a16_f64(const uint16_t *x, int64_t ldx, const uint32_t *qweight, const uint16_t *scale,
                   const uint16_t *zero, int64_t group, const float *bias,
                   int64_t M, int64_t N, int64_t K, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += oracle_f16_bits_to_f64(x[m * ldx + k]) *
                     ref_w4_dequant(qweight, scale, zero, N, K, group, k, n);
            if (bias)
                s += (double)bias[n];
            y[m * N + n] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* Output rounding and threading helpers.                                    */
/* ------------------------------------------------------------------------ */

/* Round an fp64 array to fp16 / bf16 bit patterns (nearest even). */
void ref_round_f16(const double *y, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f64_to_f16_bits(y[i]);
}

void ref_round_bf16(const double *y, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f64_to_bf16_bits(y[i]);
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Array forms of the codecs (used by the oracle's own self-tests). */
void oracle_f16_decode_array(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f16_bits_to_f64(h[i]);
}

void oracle_f32_to_f16_array(const float *f, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_f16_bits(f[i]);
}

void oracle_bf16_decode_array(const uint16_t *b, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_bits_to_f64(b[i]);
}
