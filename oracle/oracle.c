/*
 * oracle.c -- plain, slow, obviously correct CPU oracle for the BitNet b1.58
 * W2A8 BitLinear path (ternary weights x int8 activations -> int32 -> bf16).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load or call this library. The CUDA path
 * shares no code with it: no headers, helpers, tables or constants.
 *
 * Pages cited (title, address):
 *   [WIN]  "Windows 上跑通 BitNet b1.58：Flash Attention 与 CUDA sm_86 部署实录"
 *          (hmyw.cn/news/146226)
 *   [CPU]  "微软BitNet：1-bit量化大模型CPU部署实践" (m.mzlw.cn/news/189456)
 *   [GEMV] "如何编译 BitNet W2A8 CUDA 内核并用 test.py 运行 GEMV 加速测试？"
 *          (pwwt.cn/news/4591536)
 *
 * Every function is a direct transcription of a definition: loops in the
 * definition's order, fp64 where the pages fix no precision, fp32 where a
 * floating-point value decides an integer (both sides decide in fp32).
 * Readings taken where the pages are silent are stated next to each function.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Exact widening of a bf16 bit pattern to fp32 (bf16 is the top half of an
 * fp32 word). */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int oracle_abi_version(void) { return 1; }

/* ---------------------------------------------------------------------------
 * Absmean scale.  [WIN] §3.1 (BitLinear 层的三值权重逻辑): the scale is the mean
 * absolute value over the WHOLE weight matrix.  [CPU] §6.3 (模型微调) computes
 * the same quantity as the mean of |weights|.
 * Reading: sum in fp64 in row-major order, divide by N*K in fp64, round once
 * to fp32.  An empty matrix has scale 0.
 */
float oracle_absmean(const uint16_t *W, int64_t N, int64_t K)
{
    if (N <= 0 || K <= 0)
        return 0.0f;
    double sum = 0.0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            sum += fabs((double)bf16_to_f32(W[n * K + k]));
    return (float)(sum / ((double)N * (double)K));
}

/* ---------------------------------------------------------------------------
 * Ternarisation with a given scale.  [WIN] §3.1: divide each weight by the
 * scale and round to one of -1, 0, +1.  [CPU] §6.3: round(W / scale), then
 * clamp to [-1, 1].
 * Readings: fp32 IEEE division W/gamma; round half to even (the rounding of
 * the code on [CPU] §6.3); clamp to [-1, 1].  gamma == 0 (all-zero matrix) or a
 * non-positive / NaN gamma gives all zeros.  A NaN ratio gives 0.
 */
void oracle_ternarize(const uint16_t *W, int64_t N, int64_t K, float gamma,
                      int8_t *Wt)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int8_t t = 0;
            if (gamma > 0.0f) {
                float r = bf16_to_f32(W[n * K + k]) / gamma;
                if (r == r) {           /* not NaN */
                    float v = rintf(r); /* default mode: nearest, ties to even */
                    if (v > 1.0f) v = 1.0f;
                    if (v < -1.0f) v = -1.0f;
                    t = (int8_t)v;
                }
            }
            Wt[n * K + k] = t;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Per-token absmax int8 activation quantisation.  [GEMV] opening paragraph:
 * W2A8 means 2-bit weights against 8-bit activations.  The pages give no
 * formula; reading taken: for token m,
 *     amax_m = max_k |x[m,k]|                    (fp32, exact)
 *     s_m    = 127 / max(amax_m, 1e-5)           (fp32 IEEE division)
 *     q[m,k] = clamp(rne(x[m,k] * s_m), -128, 127)   (fp32 multiply)
 *     rowsum_m = sum_k q[m,k]                    (exact integer)
 * rowsum may be NULL.
 */
void oracle_quant_act(const uint16_t *x, int64_t M, int64_t K, int8_t *q,
                      float *s, int32_t *rowsum)
{
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_f32(x[m * K + k]));
            if (a > amax)
                amax = a;
        }
        float den = amax > 1e-5f ? amax : 1e-5f;
        float sc = 127.0f / den;
        s[m] = sc;
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_f32(x[m * K + k]) * sc;
            float r = rintf(v);
            if (!(r == r))
                r = 0.0f;
            if (r > 127.0f) r = 127.0f;
            if (r < -128.0f) r = -128.0f;
            int8_t qi = (int8_t)r;
            q[m * K + k] = qi;
            sum += qi;
        }
        if (rowsum)
            rowsum[m] = (int32_t)sum;
    }
}

/* ---------------------------------------------------------------------------
 * The W2A8 contraction.  [GEMV] section "运行 test.py 做 GEMV 基准测试": the
 * kernel's result must equal an int32 matrix product of the int8 activations
 * with the ternary weights, element by element.  [CPU] §2.1: with weights in
 * {-1, 0, 1} the product reduces to signed accumulation.
 *     y[m,n] = sum_k q[m,k] * W_t[n,k]    (W_t stored [N, K], out x in)
 * Accumulated in int64; returns 1 if any result leaves the int32 range (the
 * stored value is then the int64 result truncated), else 0.
 * Rows of the output are independent; they are split across OpenMP threads
 * when the library is built with OpenMP.  No blocking or reordering inside a
 * dot product.
 */
int oracle_gemm_i32(const int8_t *q, const int8_t *Wt, int64_t M, int64_t N,
                    int64_t K, int32_t *y)
{
    int overflow = 0;
    int64_t MN = M * N;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t idx = 0; idx < MN; ++idx) {
        int64_t m = idx / N, n = idx % N;
        const int8_t *qr = q + m * K;
        const int8_t *wr = Wt + n * K;
        int64_t acc = 0;
        for (int64_t k = 0; k < K; ++k)
            acc += (int64_t)qr[k] * (int64_t)wr[k];
        if (acc > INT32_MAX || acc < INT32_MIN)
            overflow = 1;
        y[idx] = (int32_t)acc;
    }
    return overflow;
}

/* Same contraction for a chosen list of output elements (m_i, n_i): used to
 * check full-size outputs on a sample. */
void oracle_gemm_i32_sampled(const int8_t *q, const int8_t *Wt, int64_t K,
                             const int64_t *ms, const int64_t *ns,
                             int64_t count, int32_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        const int8_t *qr = q + ms[i] * K;
        const int8_t *wr = Wt + ns[i] * K;
        int64_t acc = 0;
        for (int64_t k = 0; k < K; ++k)
            acc += (int64_t)qr[k] * (int64_t)wr[k];
        out[i] = (int32_t)acc;
    }
}

/* ---------------------------------------------------------------------------
 * Rescale.  [WIN] §3.1: the ternary product is multiplied back by the weight
 * scale; with int8 activations quantised by s_m = 127/amax_m the activation
 * scale is divided out as well:
 *     y[m,n] = acc[m,n] * gamma / s_m          (fp64)
 */
void oracle_rescale(const int32_t *acc, int64_t M, int64_t N, float gamma,
                    const float *s, double *y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (double)acc[m * N + n] * (double)gamma / (double)s[m];
}

/* ---------------------------------------------------------------------------
 * Full BitLinear: quantise x, contract with W_t, rescale.  q, s and acc are
 * caller-provided scratch ([M,K], [M], [M,N]).  Returns the contraction's
 * overflow flag.
 */
int oracle_bitlinear(const uint16_t *x, const int8_t *Wt, float gamma,
                     int64_t M, int64_t N, int64_t K, int8_t *q, float *s,
                     int32_t *acc, double *y)
{
    oracle_quant_act(x, M, K, q, s, (int32_t *)0);
    int of = oracle_gemm_i32(q, Wt, M, N, K, acc);
    oracle_rescale(acc, M, N, gamma, s, y);
    return of;
}

/* ---------------------------------------------------------------------------
 * 2-bit codes.  [CPU] §2.1 (1.58-bit量化原理): -1 -> 00, 0 -> 01, +1 -> 10, i.e.
 * code = w + 1; 11 is unused.  [CPU] §2.2: four ternary values per byte
 * (eight per two bytes).
 *
 * Canonical (reading) layout: row-major, ceil(K/4) bytes per row, value k of a
 * row in byte k/4 at bits 2*(k%4); unused high fields of a row's last byte
 * hold code 01.
 */
int64_t oracle_canonical_packed_bytes(int64_t N, int64_t K)
{
    return N * ((K + 3) / 4);
}

void oracle_pack_canonical(const int8_t *Wt, int64_t N, int64_t K, uint8_t *out)
{
    int64_t rb = (K + 3) / 4;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < rb; ++b) {
            unsigned byte = 0;
            for (int64_t j = 0; j < 4; ++j) {
                int64_t k = 4 * b + j;
                unsigned code = 1u;
                if (k < K)
                    code = (unsigned)(Wt[n * K + k] + 1);
                byte |= code << (2 * j);
            }
            out[n * rb + b] = (uint8_t)byte;
        }
    }
}

void oracle_unpack_canonical(const uint8_t *in, int64_t N, int64_t K, int8_t *Wt)
{
    int64_t rb = (K + 3) / 4;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            unsigned code = (in[n * rb + k / 4] >> (2 * (k % 4))) & 3u;
            Wt[n * K + k] = (int8_t)((int)code - 1);
        }
}

/* ---------------------------------------------------------------------------
 * The device layout (layout version 1), written from its specification:
 *   K_pad      = 128 * ceil(K / 128)
 *   row stride = K_pad / 4 bytes, rows in order n = 0 .. N-1
 *   value k of a row: byte 4*floor(k/16) + (k mod 4), bits 2*floor((k mod 16)/4)
 *   codes as above; positions K <= k < K_pad hold code 01 (zero weight).
 * Packing counts inputs outside {-1, 0, 1}; they are stored as code 01.
 */
int64_t oracle_device_packed_bytes(int64_t N, int64_t K)
{
    int64_t kpad = ((K + 127) / 128) * 128;
    return N * (kpad / 4);
}

int64_t oracle_pack_device(const int8_t *Wt, int64_t N, int64_t K, uint8_t *out)
{
    int64_t kpad = ((K + 127) / 128) * 128;
    int64_t stride = kpad / 4;
    int64_t invalid = 0;
    for (int64_t n = 0; n < N; ++n) {
        uint8_t *row = out + n * stride;
        for (int64_t b = 0; b < stride; ++b)
            row[b] = 0;
        for (int64_t k = 0; k < kpad; ++k) {
            unsigned code = 1u;
            if (k < K) {
                int w = Wt[n * K + k];
                if (w >= -1 && w <= 1)
                    code = (unsigned)(w + 1);
                else
                    ++invalid;
            }
            int64_t byte = 4 * (k / 16) + (k % 4);
            int shift = 2 * (int)((k % 16) / 4);
            row[byte] = (uint8_t)(row[byte] | (code << shift));
        }
    }
    return invalid;
}

/* Decodes the device layout back to ternary values; returns the number of
 * fields (inside [0, K)) holding the unused code 11, which decode to 0. */
int64_t oracle_unpack_device(const uint8_t *in, int64_t N, int64_t K, int8_t *Wt)
{
    int64_t kpad = ((K + 127) / 128) * 128;
    int64_t stride = kpad / 4;
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int64_t byte = 4 * (k / 16) + (k % 4);
            int shift = 2 * (int)((k % 16) / 4);
            unsigned code = (in[n * stride + byte] >> shift) & 3u;
            if (code == 3u) {
                ++bad;
                code = 1u;
            }
            Wt[n * K + k] = (int8_t)((int)code - 1);
        }
    return bad;
}
