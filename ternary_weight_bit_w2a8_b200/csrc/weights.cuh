// weights.cuh -- offline weight preparation: absmean scale, ternarisation and
// packing into layout v1.
//
// Absmean and ternarisation follow page "Windows 上跑通 BitNet b1.58：Flash
// Attention 与 CUDA sm_86 部署实录" §3.1 (scale = mean |W| over the whole matrix,
// W / scale rounded into {-1, 0, 1}) and page "微软BitNet：1-bit量化大模型CPU部署
// 实践" §6.3 (round, then clamp to [-1, 1]).  Codes follow §2.1 of the latter
// page (-1 -> 00, 0 -> 01, +1 -> 10), four per byte (§2.2).
#pragma once

#include "common.cuh"

namespace bitnet {

// ---------------------------------------------------------------- absmean
// Two passes with a fixed summation order for a given element count: pass 1
// gives each of `nblk` CTAs a contiguous range and sums |w| in fp64 per thread
// (strided), then across the CTA; pass 2 sums the CTA partials in index order.

constexpr int kAbsmeanMaxBlocks = 1024;

__host__ __forceinline__ int absmean_blocks(int64_t total) {
    int64_t b = ceil_div(total, 8192);
    if (b < 1) b = 1;
    if (b > kAbsmeanMaxBlocks) b = kAbsmeanMaxBlocks;
    return (int)b;
}

__global__ void __launch_bounds__(kThreads) absmean_partial_kernel(const uint16_t *__restrict__ W,
                                                                   int64_t total,
                                                                   double *__restrict__ partial) {
    __shared__ double scratch[32];
    const int64_t per = ceil_div(total, gridDim.x);
    const int64_t lo = (int64_t)blockIdx.x * per;
    const int64_t hi = lo + per < total ? lo + per : total;
    double acc = 0.0;
    for (int64_t i = lo + threadIdx.x; i < hi; i += kThreads)
        acc += fabs((double)bf16_bits_to_float(W[i]));
    double s = block_reduce(acc, [](double a, double b) { return a + b; }, scratch);
    if (threadIdx.x == 0) partial[blockIdx.x] = s;
}

__global__ void __launch_bounds__(kThreads) absmean_final_kernel(const double *__restrict__ partial,
                                                                 int nblk, int64_t total,
                                                                 float *__restrict__ gamma) {
    __shared__ double scratch[32];
    double acc = 0.0;
    for (int i = threadIdx.x; i < nblk; i += kThreads) acc += partial[i];
    double s = block_reduce(acc, [](double a, double b) { return a + b; }, scratch);
    if (threadIdx.x == 0) *gamma = total > 0 ? (float)(s / (double)total) : 0.0f;
}

// ---------------------------------------------------------------- ternarise
__device__ __forceinline__ int8_t ternarize_one(uint16_t w, float gamma) {
    if (!(gamma > 0.0f)) return 0;
    float r = __fdiv_rn(bf16_bits_to_float(w), gamma);  // IEEE fp32 division
    if (r != r) return 0;
    float v = rintf(r);  // nearest, ties to even
    v = v > 1.0f ? 1.0f : v;
    v = v < -1.0f ? -1.0f : v;
    return (int8_t)v;
}

__global__ void __launch_bounds__(kThreads) ternarize_kernel(const uint16_t *__restrict__ W,
                                                             int64_t total,
                                                             const float *__restrict__ gamma_p,
                                                             int8_t *__restrict__ Wt) {
    const float gamma = *gamma_p;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total; i += stride)
        Wt[i] = ternarize_one(W[i], gamma);
}

// ---------------------------------------------------------------- pack (layout v1)
// One thread writes one 32-bit word = 16 consecutive k of a row: value
// k0 + 4j + b goes to bits 8b + 2j.  Values outside {-1, 0, 1} are counted and
// stored as code 01.
__global__ void __launch_bounds__(kThreads) pack_v1_kernel(const int8_t *__restrict__ Wt, int64_t N,
                                                           int64_t K, int64_t words_per_row,
                                                           uint32_t *__restrict__ out,
                                                           int32_t *__restrict__ invalid) {
    const int64_t total = N * words_per_row;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int bad = 0;
    for (int64_t idx = (int64_t)blockIdx.x * kThreads + threadIdx.x; idx < total; idx += stride) {
        const int64_t n = idx / words_per_row;
        const int64_t k0 = (idx - n * words_per_row) * 16;
        const int8_t *src = Wt + n * K + k0;
        uint32_t word = 0;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            uint32_t code = 1u;
            if (k0 + t < K) {
                const int v = src[t];
                if (v >= -1 && v <= 1)
                    code = (uint32_t)(v + 1);
                else
                    ++bad;
            }
            word |= code << (8 * (t & 3) + 2 * (t >> 2));
        }
        out[idx] = word;
    }
    if (invalid != nullptr) {
        bad = __reduce_add_sync(0xffffffffu, bad);
        if ((threadIdx.x & 31) == 0 && bad) atomicAdd(invalid, bad);
    }
}

}  // namespace bitnet
