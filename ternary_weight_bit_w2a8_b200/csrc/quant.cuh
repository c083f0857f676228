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

// clamp(rne(x * sc), -128, 127), NaN to 0, in full-rate fp32 arithmetic
// (conversion instructions run at a fraction of that rate).  With sc =
// 127 / max|x| the product lies in [-127, 127] up to one rounding, so no
// clamp is needed: adding 1.5 * 2^23 rounds it to the nearest integer, ties
// to even (the float spacing there is 1 and 1.5 * 2^23 is even), and leaves
// that integer in the low mantissa bits.  Returns the word whose low byte
// is the code (the bits of 1.5 * 2^23 for NaN, low byte 0); quant_val gives
// the signed value.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

__device__ __forceinline__ uint32_t quant_bits(float x, float sc) {
    const float v = __fmul_rn(x, sc);
    const uint32_t b = __float_as_uint(__fadd_rn(v, kRoundMagic));
    return v == v ? b : kRoundMagicBits;
}

__device__ __forceinline__ int quant_val(uint32_t bits) { return (int)(bits - kRoundMagicBits); }

__device__ __forceinline__ int8_t quant_one(float x, float sc) { return (int8_t)quant_val(quant_bits(x, sc)); }

// Low bytes of four words in one word, a in byte 0.
__device__ __forceinline__ uint32_t pack4_b0(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    uint32_t ab, cd, r;
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(ab) : "r"(a), "r"(b));
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(cd) : "r"(c), "r"(d));
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(ab), "r"(cd));
    return r;
}

// |x| maximum over the 8 bf16 values of a 16-byte word.
__device__ __forceinline__ float amax8(const uint4 &v, float m) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xffff0000u)));
    }
    return m;
}

// The 8 codes of a 16-byte word of bf16 values (low byte = lowest k), and,
// when SUM, their sum added to `sum`.
template <bool SUM = true>
__device__ __forceinline__ uint2 quant8(const uint4 &v, float sc, int &sum) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        c[2 * i] = quant_bits(__uint_as_float(w[i] << 16), sc);
        c[2 * i + 1] = quant_bits(__uint_as_float(w[i] & 0xffff0000u), sc);
    }
    if (SUM) {
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += quant_val(c[i]);
    }
    return make_uint2(pack4_b0(c[0], c[1], c[2], c[3]), pack4_b0(c[4], c[5], c[6], c[7]));
}

// A team of WPT warps quantises one token row at a time (a CTA of up to
// kThreads threads holds blockDim.x / (32 * WPT) teams; rows are dealt to teams
// grid-stride).  The row is read from HBM once: each thread keeps up to
// kQuantHeld 16-byte words in registers between the absmax pass and the
// quantise pass (rows longer than kQuantHeld * 8 * 32 * WPT values re-read
// the rest, from L1/L2).  Reductions are warp shuffles plus, for WPT > 1, one
// named barrier per team.  q rows have stride ldq (>= K); with zero_pad set,
// K <= k < ldq is written as 0.  rowsum may be null.
constexpr int kQuantHeld = 12;

template <int WPT>
__device__ __forceinline__ float team_max(float v, float *red, int team, int wt) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (WPT > 1) {
        if ((threadIdx.x & 31) == 0) red[team * WPT + wt] = v;
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(WPT * 32) : "memory");
        v = red[team * WPT];
#pragma unroll
        for (int i = 1; i < WPT; ++i) v = fmaxf(v, red[team * WPT + i]);
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(WPT * 32) : "memory");
    }
    return v;
}

template <int WPT>
__device__ __forceinline__ int team_sum(int v, int *red, int team, int wt) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (WPT > 1) {
        if ((threadIdx.x & 31) == 0) red[team * WPT + wt] = v;
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(WPT * 32) : "memory");
        int r = 0;
#pragma unroll
        for (int i = 0; i < WPT; ++i) r += red[team * WPT + i];
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(WPT * 32) : "memory");
        v = r;
    }
    return v;
}

// One token row quantised by a team of WPT warps (team-local thread t of
// 32 * WPT; `team` picks the named barrier and the reduction slots).  Writes
// q (and the zero padding up to ldq), returns the scale; `sum` receives the
// row's code sum when want_sum is set.
template <int WPT>
__device__ __forceinline__ float quant_row(const uint16_t *__restrict__ xr, int64_t K, int8_t *__restrict__ qr,
                                           int64_t ldq, bool zero_pad, bool want_sum, int &sum, float *fred,
                                           int *ired, int team, int t) {
    constexpr int kTeam = 32 * WPT;
    const int wt = t >> 5;
    const bool vec = (reinterpret_cast<uintptr_t>(xr) & 15) == 0;
    const bool qvec = (reinterpret_cast<uintptr_t>(qr) & 7) == 0;
    const int64_t nw = vec ? K / 8 : 0;  // whole 16-byte words of the row

    // every load of the row is issued before the first is used: one memory
    // round trip for the held words (and one per further batch), not one per word
    uint4 held[kQuantHeld];
#pragma unroll
    for (int i = 0; i < kQuantHeld; ++i) {
        const int64_t c = t + (int64_t)i * kTeam;
        held[i] = c < nw ? *reinterpret_cast<const uint4 *>(xr + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kQuantHeld; ++i) amax = amax8(held[i], amax);
    for (int64_t c0 = t + (int64_t)kQuantHeld * kTeam; c0 < nw; c0 += (int64_t)4 * kTeam) {
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t c = c0 + (int64_t)i * kTeam;
            v[i] = c < nw ? *reinterpret_cast<const uint4 *>(xr + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = amax8(v[i], amax);
    }
    for (int64_t k = nw * 8 + t; k < K; k += kTeam) amax = fmaxf(amax, fabsf(bf16_bits_to_float(xr[k])));
    amax = team_max<WPT>(amax, fred, team, wt);
    const float sc = __fdiv_rn(127.0f, amax > kQuantEps ? amax : kQuantEps);

    sum = 0;
    auto put8 = [&](int64_t c, const uint2 &v) {
        if (qvec) {
            *reinterpret_cast<uint2 *>(qr + 8 * c) = v;
        } else {
#pragma unroll
            for (int b = 0; b < 8; ++b) qr[8 * c + b] = (int8_t)(((b < 4 ? v.x : v.y) >> (8 * (b & 3))) & 0xff);
        }
    };
#pragma unroll
    for (int i = 0; i < kQuantHeld; ++i) {
        const int64_t c = t + (int64_t)i * kTeam;
        if (c < nw) put8(c, want_sum ? quant8<true>(held[i], sc, sum) : quant8<false>(held[i], sc, sum));
    }
    for (int64_t c0 = t + (int64_t)kQuantHeld * kTeam; c0 < nw; c0 += (int64_t)4 * kTeam) {
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t c = c0 + (int64_t)i * kTeam;
            v[i] = c < nw ? *reinterpret_cast<const uint4 *>(xr + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t c = c0 + (int64_t)i * kTeam;
            if (c < nw) put8(c, want_sum ? quant8<true>(v[i], sc, sum) : quant8<false>(v[i], sc, sum));
        }
    }
    for (int64_t k = nw * 8 + t; k < K; k += kTeam) {
        const int8_t qi = quant_one(bf16_bits_to_float(xr[k]), sc);
        qr[k] = qi;
        sum += qi;
    }
    if (zero_pad)
        for (int64_t k = K + t; k < ldq; k += kTeam) qr[k] = 0;
    if (want_sum) sum = team_sum<WPT>(sum, ired, team, wt);
    return sc;
}

template <int WPT>
__global__ void __launch_bounds__(kThreads) quant_act_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                             int8_t *__restrict__ q, int64_t ldq, bool zero_pad,
                                                             float *__restrict__ s, int32_t *__restrict__ rowsum) {
    constexpr int kTeam = 32 * WPT;
    const int teams = blockDim.x / kTeam;  // blockDim.x: a multiple of kTeam, at most kThreads
    __shared__ float fred[kThreads / 32];
    __shared__ int ired[kThreads / 32];
    // a dependent kernel may start its own independent work (weight loads)
    // now; it waits for this grid to complete before it reads q or s
    pdl_launch_dependents();
    pdl_wait();
    const int team = threadIdx.x / kTeam, t = threadIdx.x % kTeam;
    for (int64_t m = (int64_t)blockIdx.x * teams + team; m < M; m += (int64_t)gridDim.x * teams) {
        int sum = 0;
        const float sc = quant_row<WPT>(x + m * K, K, q + m * ldq, ldq, zero_pad, rowsum != nullptr, sum, fred, ired,
                                        team, t);
        if (t == 0) {
            s[m] = sc;
            if (rowsum != nullptr) rowsum[m] = sum;
        }
    }
}

}  // namespace bitnet
