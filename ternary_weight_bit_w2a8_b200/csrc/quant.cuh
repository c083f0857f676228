// quant.cuh -- per-token absmax int8 activation quantisation.
//
// Page "如何编译 BitNet W2A8 CUDA 内核并用 test.py 运行 GEMV 加速测试？" (opening
// paragraph) fixes 8-bit activations against 2-bit weights; the pages give no
// formula, so this library reads it as the per-token absmax scale:
//   s_m = 127 / max(max_k |x[m,k]|, 1e-5),  q = clamp(rne(x * s_m), -128, 127)
// with fp32 division and multiplication (IEEE round-to-nearest, no FMA).
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr float kQuantEps = 1e-5f;

__device__ __forceinline__ int8_t quant_one(float x, float sc) {
    float r = rintf(__fmul_rn(x, sc));
    if (r != r) r = 0.0f;
    r = r > 127.0f ? 127.0f : r;
    r = r < -128.0f ? -128.0f : r;
    return (int8_t)r;
}

// One CTA per token.  Writes q with row stride ldq (>= K); positions
// K <= k < ldq are written as 0 when zero_pad is set.
__global__ void __launch_bounds__(kThreads) quant_act_kernel(const uint16_t *__restrict__ x, int64_t K,
                                                             int8_t *__restrict__ q, int64_t ldq,
                                                             bool zero_pad, float *__restrict__ s,
                                                             int32_t *__restrict__ rowsum) {
    __shared__ float fscratch[32];
    __shared__ int iscratch[32];
    // a dependent kernel may start its own independent work (weight loads) now;
    // it waits for this grid to complete before it reads q or s
    pdl_launch_dependents();
    const int64_t m = blockIdx.x;
    const uint16_t *xr = x + m * K;
    int8_t *qr = q + m * ldq;
    const bool vec = ((reinterpret_cast<uintptr_t>(xr) & 15) == 0);
    const int64_t K8 = vec ? (K / 8) * 8 : 0;
    const bool qvec = vec && ((reinterpret_cast<uintptr_t>(qr) & 7) == 0);

    float amax = 0.0f;
    for (int64_t k = threadIdx.x * 8; k < K8; k += kThreads * 8) {
        uint4 v = *reinterpret_cast<const uint4 *>(xr + k);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xffff0000u)));
        }
    }
    for (int64_t k = K8 + threadIdx.x; k < K; k += kThreads) amax = fmaxf(amax, fabsf(bf16_bits_to_float(xr[k])));
    amax = block_reduce(amax, [](float a, float b) { return fmaxf(a, b); }, fscratch);

    const float sc = __fdiv_rn(127.0f, amax > kQuantEps ? amax : kQuantEps);
    int sum = 0;
    const int64_t Kv = qvec ? K8 : 0;  // 8 values per thread: one 16-byte load, one 8-byte store
    for (int64_t k = threadIdx.x * 8; k < Kv; k += kThreads * 8) {
        uint4 v = *reinterpret_cast<const uint4 *>(xr + k);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int8_t lo = quant_one(__uint_as_float(w[i] << 16), sc);
            const int8_t hi = quant_one(__uint_as_float(w[i] & 0xffff0000u), sc);
            sum += lo + hi;
            packed[i >> 1] |= ((uint32_t)(uint8_t)lo | ((uint32_t)(uint8_t)hi << 8)) << (16 * (i & 1));
        }
        *reinterpret_cast<uint2 *>(qr + k) = make_uint2(packed[0], packed[1]);
    }
    for (int64_t k = Kv + threadIdx.x; k < K; k += kThreads) {
        const int8_t qi = quant_one(bf16_bits_to_float(xr[k]), sc);
        qr[k] = qi;
        sum += qi;
    }
    if (zero_pad)
        for (int64_t k = K + threadIdx.x; k < ldq; k += kThreads) qr[k] = 0;
    sum = block_reduce(sum, [](int a, int b) { return a + b; }, iscratch);
    if (threadIdx.x == 0) {
        s[m] = sc;
        if (rowsum != nullptr) rowsum[m] = sum;
    }
}

}  // namespace bitnet
