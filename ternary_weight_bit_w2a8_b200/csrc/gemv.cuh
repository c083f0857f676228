// gemv.cuh -- the decode GEMV: y[m, n] = sum_k q[m, k] * W_t[n, k] for a few
// tokens m, streaming the packed 2-bit weights once from HBM.
//
// The pages' GEMV (page "如何编译 BitNet W2A8 CUDA 内核并用 test.py 运行 GEMV 加速
// 测试？", section "编译 W2A8 CUDA 内核" and the README optimisations it lists: a
// 16x32 block reorder, 16 interleaved 2-bit values per 32-bit word, dp4a dot
// products; one template instance per hard-coded (N, K), M == 1 only) is an
// Ampere design.  This kernel keeps the 16-values-per-word / dp4a idea and
// otherwise is its own: any N and K, a plain row-major layout, bulk L2
// prefetch ahead of 128-bit loads, activations in shared memory.
//
// Work decomposition
//   - A chunk is 64 consecutive k = 16 packed bytes = four 32-bit words; word i
//     covers k = 16i .. 16i+15 and, for j = 0..3, its byte fields j hold
//     k = 16i+4j .. 16i+4j+3 (layout v1).
//   - The activations of one K-slice live in shared memory as 16-byte pieces in
//     the order [piece i of a chunk][chunk u], so lanes reading consecutive
//     chunks hit consecutive bank groups.
//   - A warp is split into 32/G groups of G lanes; a warp task is RT = (32/G)*R
//     consecutive rows, each group owning R of them; lane l of a group takes
//     chunks l, l+G, l+2G, ... of the slice, the same set for every row, so the
//     activations' sum over a lane's chunks is computed once.
//   - Weights: each warp asks the L2 for the rows of its tasks a few tasks
//     ahead with one bulk prefetch (no registers held), then reads them with
//     16-byte loads in batches of U chunks x R rows, all in flight at once.
//   - Decode without shifts: (word & (3 << 2j) per byte) is the code scaled by
//     4^j; dp4a(unsigned code bytes, signed activations) accumulates each j in
//     its own register, combined by exact arithmetic shifts.  Codes are w + 1,
//     so the slice's activation sum is subtracted at the end.
//   - The G partial sums of a row are combined with warp shuffles.
//   - Split-K (gridDim.y > 1) writes int32 partials; a second kernel adds them
//     in slice order and applies the epilogue.
//   - Programmatic dependent launch: weights never depend on an earlier kernel,
//     so their prefetch and the first batch of loads are issued before
//     griddepcontrol.wait; activations are read, and outputs written, after it.
//     (An earlier kernel on the stream that lets dependents launch early must
//     therefore not write the packed weights; this library's kernels never do.)
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace bitnet {

struct GemvArgs {
    const int8_t *q;      // int8 activations [M, K], row stride ldq (mode 0)
    const uint16_t *x;    // bf16 activations [M, K] (mode 1: quantised in the prologue)
    int64_t ldq;
    const uint8_t *W;     // packed layout v1
    int64_t row_bytes;    // K_pad / 4
    int64_t N;
    int64_t K;
    int nch_total;        // K_pad / 64
    int cps;              // chunks per K-slice
    int M;
    int prefetch_tasks;   // how many tasks ahead a warp prefetches
    int32_t *y_i32;       // [M, N] int32 result (single slice, int output)
    uint16_t *y_bf16;     // [M, N] bf16 result (single slice, BitLinear output)
    int32_t *partial;     // [S, M, N] int32 partials (split-K)
    const float *s_act;   // [M] activation scales (BitLinear, mode 0)
    float *s_out;         // [M] activation scales written in mode 1 (may be null)
    const float *gamma;   // weight scale (BitLinear)
};

__device__ __forceinline__ void mac_word(int (&acc)[4], uint32_t w, const uint4 &x) {
    acc[0] = dp4a_us(w & 0x03030303u, x.x, acc[0]);
    acc[1] = dp4a_us(w & 0x0C0C0C0Cu, x.y, acc[1]);
    acc[2] = dp4a_us(w & 0x30303030u, x.z, acc[2]);
    acc[3] = dp4a_us(w & 0xC0C0C0C0u, x.w, acc[3]);
}

__device__ __forceinline__ int byte_sum(const uint4 &v, int c) {
    c = dp4a_us(0x01010101u, v.x, c);
    c = dp4a_us(0x01010101u, v.y, c);
    c = dp4a_us(0x01010101u, v.z, c);
    return dp4a_us(0x01010101u, v.w, c);
}

// Stages the int8 activations of chunks [c0, c0 + nch) of token row `qrow`
// into qs (zero beyond K).
__device__ __forceinline__ void stage_q_int8(uint4 *qs, const int8_t *qrow, int64_t K, int c0, int nch) {
    for (int p = threadIdx.x; p < 4 * nch; p += blockDim.x) {
        const int64_t k0 = (int64_t)c0 * 64 + (int64_t)p * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (k0 + 16 <= K && ((reinterpret_cast<uintptr_t>(qrow + k0) & 15) == 0)) {
            v = *reinterpret_cast<const uint4 *>(qrow + k0);
        } else if (k0 < K) {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            for (int t = 0; t < 16 && k0 + t < K; ++t) w[t >> 2] |= (uint32_t)(uint8_t)qrow[k0 + t] << (8 * (t & 3));
            v = make_uint4(w[0], w[1], w[2], w[3]);
        }
        qs[(p & 3) * nch + (p >> 2)] = v;
    }
}

// Fused per-token quantisation (same arithmetic as quant_act_kernel<>): absmax
// over the whole row, then the slice's codes into qs.  Returns the scale.
// Thread t owns the 16-value pieces t, t + blockDim, ...; up to kHeld of them
// stay in registers between the absmax pass and the quantise pass.
__device__ __forceinline__ void quant16(const uint4 &lo, const uint4 &hi, float sc, uint4 &out) {
    int unused = 0;
    const uint2 a = quant8<false>(lo, sc, unused), b = quant8<false>(hi, sc, unused);
    out = make_uint4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float amax16(const uint4 &lo, const uint4 &hi, float m) {
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xffff0000u)));
    }
    return m;
}

// 16 bf16 values of piece p of a row (zeros beyond K), as two 16-byte words.
__device__ __forceinline__ void load_x16(const uint16_t *xrow, int64_t K, int64_t p, bool vec, uint4 &lo, uint4 &hi) {
    const int64_t k0 = p * 16;
    if (vec && k0 + 16 <= K) {
        lo = *reinterpret_cast<const uint4 *>(xrow + k0);
        hi = *reinterpret_cast<const uint4 *>(xrow + k0 + 8);
    } else {
        uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        for (int t = 0; t < 16 && k0 + t < K; ++t) w[t >> 1] |= (uint32_t)xrow[k0 + t] << (16 * (t & 1));
        lo = make_uint4(w[0], w[1], w[2], w[3]);
        hi = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

__device__ __forceinline__ float stage_q_bf16(uint4 *qs, float *red, const uint16_t *xrow, int64_t K, int c0,
                                              int nch) {
    constexpr int kHeld = 4;
    const bool vec = ((reinterpret_cast<uintptr_t>(xrow) & 15) == 0);
    const int64_t npieces = ceil_div(K, 16);
    uint4 held[kHeld][2];
    float amax = 0.0f;
#pragma unroll
    for (int h = 0; h < kHeld; ++h) {
        const int64_t p = threadIdx.x + (int64_t)h * blockDim.x;
        if (p < npieces) {
            load_x16(xrow, K, p, vec, held[h][0], held[h][1]);
            amax = amax16(held[h][0], held[h][1], amax);
        }
    }
    for (int64_t p = threadIdx.x + (int64_t)kHeld * blockDim.x; p < npieces; p += blockDim.x) {
        uint4 lo, hi;
        load_x16(xrow, K, p, vec, lo, hi);
        amax = amax16(lo, hi, amax);
    }
    amax = block_reduce(amax, [](float u, float v) { return fmaxf(u, v); }, red);
    const float sc = __fdiv_rn(127.0f, amax > kQuantEps ? amax : kQuantEps);
    // pieces of this slice: global piece index 4*c0 + pl, pl < 4*nch
    const int64_t pbeg = (int64_t)c0 * 4, pend = pbeg + 4 * nch;
#pragma unroll
    for (int h = 0; h < kHeld; ++h) {
        const int64_t p = threadIdx.x + (int64_t)h * blockDim.x;
        if (p >= pbeg && p < pend) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (p < npieces) quant16(held[h][0], held[h][1], sc, v);
            const int pl = (int)(p - pbeg);
            qs[(pl & 3) * nch + (pl >> 2)] = v;
        }
    }
    // pieces of the slice not held in registers (beyond kHeld per thread)
    {
        int64_t first = threadIdx.x + (int64_t)kHeld * blockDim.x;
        if (first < pbeg) first += ceil_div(pbeg - first, (int64_t)blockDim.x) * blockDim.x;
        for (int64_t p = first; p < pend; p += blockDim.x) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (p < npieces) {
                uint4 lo, hi;
                load_x16(xrow, K, p, vec, lo, hi);
                quant16(lo, hi, sc, v);
            }
            const int pl = (int)(p - pbeg);
            qs[(pl & 3) * nch + (pl >> 2)] = v;
        }
    }
    return sc;
}

template <int G>
__device__ __forceinline__ int group_sum(int v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Loads batch `i0` (chunks l + G*(i0 + j), j < U) of R rows into registers;
// chunks past the lane's count are not loaded.
template <int G, int R, int U>
__device__ __forceinline__ void load_batch(uint4 (&wb)[U][R], const uint8_t *const (&p)[R], int i0, int iters) {
#pragma unroll
    for (int j = 0; j < U; ++j) {
        if (i0 + j < iters) {
#pragma unroll
            for (int r = 0; r < R; ++r) wb[j][r] = ldg_stream_v4(p[r] + (int64_t)(i0 + j) * G * 16);
        }
    }
}

template <int G, int R, int U, int XMODE>
__global__ void __launch_bounds__(kThreads, (R * U > 4 ? 2 : 3)) gemv_w2a8_kernel(const GemvArgs a) {
    static_assert(G == 8 || G == 16 || G == 32, "lanes per row");
    static_assert(R >= 1 && R <= G, "rows per lane group");
    extern __shared__ uint4 qs[];
    __shared__ float red[32];
    constexpr int kWarps = kThreads / 32;
    constexpr int RT = (32 / G) * R;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / G, l = lane % G;
    const int m = blockIdx.z;
    const int c0 = blockIdx.y * a.cps;
    const int nch = min(a.nch_total - c0, a.cps);
    const int64_t N = a.N, row_bytes = a.row_bytes;
    const int64_t n_tasks = ceil_div(N, RT);
    const int64_t tw = (int64_t)gridDim.x * kWarps;
    const int64_t t0 = (int64_t)blockIdx.x * kWarps + warp;
    const uint8_t *wbase = a.W + (int64_t)c0 * 16;
    const bool full_rows = (nch == a.nch_total);  // a task's rows form one contiguous block
    // this lane's chunks: l + G*i for i < iters
    const int nfull = nch / G;
    const int iters = nfull + (l < nch - nfull * G ? 1 : 0);

    auto prefetch_task = [&](int64_t t) {
        if (t >= n_tasks) return;
        const int64_t r0 = t * RT;
        const int64_t rows = N - r0 < RT ? N - r0 : RT;
        if (full_rows) {
            if (lane == 0) prefetch_l2_bulk(wbase + r0 * row_bytes, (uint32_t)(rows * row_bytes));
        } else if (lane < rows) {
            prefetch_l2_bulk(wbase + (r0 + lane) * row_bytes, (uint32_t)(nch * 16));
        }
    };
    auto row_ptrs = [&](int64_t t, const uint8_t *(&p)[R]) {
        const int64_t nb = t * RT + grp * R;
#pragma unroll
        for (int r = 0; r < R; ++r) p[r] = wbase + (nb + r < N ? nb + r : N - 1) * row_bytes + l * 16;
    };

    // Weights do not depend on the previous kernel: start streaming them
    // (L2 prefetch of the first tasks, first batch into registers) before
    // waiting for it.
    uint4 wb[U][R];
    const uint8_t *p[R];
    for (int d = 0; d <= a.prefetch_tasks; ++d) prefetch_task(t0 + d * tw);
    if (t0 < n_tasks) {
        row_ptrs(t0, p);
        load_batch<G, R, U>(wb, p, 0, iters);
    }
    pdl_launch_dependents();
    pdl_wait();  // activations may come from the previous kernel on the stream

    float sc = 0.0f;
    if (XMODE == 0) {
        stage_q_int8(qs, a.q + (int64_t)m * a.ldq, a.K, c0, nch);
    } else {
        sc = stage_q_bf16(qs, red, a.x + (int64_t)m * a.K, a.K, c0, nch);
        if (a.s_out != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) a.s_out[m] = sc;
    }
    __syncthreads();

    int qsum = 0;
    for (int i = 0; i < iters; ++i) {
        const int u = l + G * i;
        qsum = byte_sum(qs[u], qsum);
        qsum = byte_sum(qs[nch + u], qsum);
        qsum = byte_sum(qs[2 * nch + u], qsum);
        qsum = byte_sum(qs[3 * nch + u], qsum);
    }
    qsum = group_sum<G>(qsum);

    float f = 0.0f;  // BitLinear rescale factor gamma / s_m
    if (a.y_bf16 != nullptr && a.partial == nullptr) f = __fdiv_rn(*a.gamma, XMODE == 0 ? a.s_act[m] : sc);

    for (int64_t t = t0; t < n_tasks; t += tw) {
        prefetch_task(t + (a.prefetch_tasks + 1) * tw);
        if (t != t0) row_ptrs(t, p);
        int acc[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0;
        for (int i0 = 0; i0 < iters; i0 += U) {
            if (t != t0 || i0 != 0) load_batch<G, R, U>(wb, p, i0, iters);
#pragma unroll
            for (int j = 0; j < U; ++j) {
                if (i0 + j < iters) {
                    const int u = l + G * (i0 + j);
                    const uint4 x0 = qs[u], x1 = qs[nch + u], x2 = qs[2 * nch + u], x3 = qs[3 * nch + u];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        mac_word(acc[r], wb[j][r].x, x0);
                        mac_word(acc[r], wb[j][r].y, x1);
                        mac_word(acc[r], wb[j][r].z, x2);
                        mac_word(acc[r], wb[j][r].w, x3);
                    }
                }
            }
        }

        const int64_t nb = t * RT + grp * R;
        int tot[R];
#pragma unroll
        for (int r = 0; r < R; ++r)
            tot[r] = group_sum<G>(acc[r][0] + (acc[r][1] >> 2) + (acc[r][2] >> 4) + (acc[r][3] >> 6));
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t n = nb + r;
            if (l == r && n < N) {
                const int v = tot[r] - qsum;
                const int64_t o = (int64_t)m * N + n;
                if (a.partial != nullptr)
                    a.partial[(int64_t)blockIdx.y * a.M * N + o] = v;
                else if (a.y_bf16 != nullptr)
                    a.y_bf16[o] = float_to_bf16_bits_rn(__fmul_rn((float)v, f));
                else
                    a.y_i32[o] = v;
            }
        }
    }
}

// Split-K reduction: y[m, n] = sum over slices, in slice order, then the
// epilogue.  In mode 1 the activation scales come from s_out.
__global__ void __launch_bounds__(kThreads) gemv_splitk_reduce_kernel(const GemvArgs a, int S) {
    pdl_wait();
    const int64_t MN = (int64_t)a.M * a.N;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t o = (int64_t)blockIdx.x * kThreads + threadIdx.x; o < MN; o += stride) {
        int acc = 0;
        for (int s = 0; s < S; ++s) acc += a.partial[(int64_t)s * MN + o];
        const int m = (int)(o / a.N);
        if (a.y_bf16 != nullptr) {
            const float f = __fdiv_rn(*a.gamma, a.s_act != nullptr ? a.s_act[m] : a.s_out[m]);
            a.y_bf16[o] = float_to_bf16_bits_rn(__fmul_rn((float)acc, f));
        } else {
            a.y_i32[o] = acc;
        }
    }
}

}  // namespace bitnet
