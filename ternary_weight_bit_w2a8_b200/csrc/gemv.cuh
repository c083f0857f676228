// gemv.cuh -- the decode GEMV: y[m, n] = sum_k q[m, k] * W_t[n, k] for a few
// tokens m, streaming the packed 2-bit weights once from HBM.
//
// The pages' GEMV (page "如何编译 BitNet W2A8 CUDA 内核并用 test.py 运行 GEMV 加速
// 测试？", section "编译 W2A8 CUDA 内核" and the README optimisations it lists: a
// 16x32 block reorder, 16 interleaved 2-bit values per 32-bit word, dp4a dot
// products; one template instance per hard-coded (N, K), M == 1 only) is an
// Ampere design.  This kernel keeps the 16-values-per-word / dp4a idea and
// otherwise is its own: any N and K, 128-bit streaming loads of a plain
// row-major layout, activations in shared memory, no reorder pass.
//
// Work decomposition
//   - Activations of one K-slice live in shared memory, stored as 16-byte
//     pieces in the order [piece i of a chunk][chunk u], so that lanes reading
//     consecutive chunks hit consecutive 16-byte bank groups.
//   - A chunk is 64 consecutive k = 16 packed bytes = four 32-bit words; word i
//     covers k = 16i .. 16i+15 and, for j = 0..3, its byte fields j hold
//     k = 16i+4j .. 16i+4j+3.
//   - A warp is split into 32/G groups of G lanes; each group owns R rows at a
//     time, its lanes take the slice's chunks round-robin.  Each lane keeps
//     UN*R 16-byte loads in flight.
//   - Decode without shifts: (word & (3 << 2j) per byte) is the code scaled by
//     4^j; dp4a(unsigned code bytes, signed activations) accumulates each j in
//     its own register, and the four are combined with exact arithmetic
//     shifts at the end.  Codes are w + 1, so the sum over the slice is
//     corrected by subtracting sum_k q (the slice's activation sum).
//   - The G partial sums of a row are combined with warp shuffles.
//   - Split-K (gridDim.y > 1) writes int32 partials; a second kernel adds them
//     in slice order and applies the epilogue.
#pragma once

#include "common.cuh"

namespace bitnet {

struct GemvArgs {
    const int8_t *q;      // activations [M, K], row stride ldq
    int64_t ldq;
    const uint8_t *W;     // packed layout v1
    int64_t row_bytes;    // K_pad / 4
    int64_t N;
    int64_t K;
    int nch_total;        // K_pad / 64
    int cps;              // chunks per K-slice
    int M;
    int32_t *y_i32;       // [M, N] int32 result (single slice, int output)
    uint16_t *y_bf16;     // [M, N] bf16 result (single slice, BitLinear output)
    int32_t *partial;     // [S, M, N] int32 partials (split-K)
    const float *s_act;   // [M] activation scales (BitLinear)
    const float *gamma;   // weight scale (BitLinear)
};

// Epilogue of one output element.
__device__ __forceinline__ void gemv_store(const GemvArgs &a, int m, int64_t n, int acc) {
    const int64_t o = (int64_t)m * a.N + n;
    if (a.partial != nullptr) {
        a.partial[(int64_t)blockIdx.y * a.M * a.N + o] = acc;
    } else if (a.y_bf16 != nullptr) {
        const float f = __fdiv_rn(*a.gamma, a.s_act[m]);
        a.y_bf16[o] = float_to_bf16_bits_rn(__fmul_rn((float)acc, f));
    } else {
        a.y_i32[o] = acc;
    }
}

__device__ __forceinline__ void mac_word(int (&acc)[4], uint32_t w, const uint4 &x) {
    acc[0] = dp4a_us(w & 0x03030303u, x.x, acc[0]);
    acc[1] = dp4a_us(w & 0x0C0C0C0Cu, x.y, acc[1]);
    acc[2] = dp4a_us(w & 0x30303030u, x.z, acc[2]);
    acc[3] = dp4a_us(w & 0xC0C0C0C0u, x.w, acc[3]);
}

template <int G, int R, int UN>
__global__ void __launch_bounds__(kThreads) gemv_w2a8_kernel(const GemvArgs a) {
    static_assert(G == 8 || G == 16 || G == 32, "lanes per row");
    static_assert(R >= 1 && R <= G, "rows per lane group");
    extern __shared__ uint4 qs[];
    __shared__ int red[32];

    const int m = blockIdx.z;
    const int c0 = blockIdx.y * a.cps;
    const int nch = min(a.nch_total - c0, a.cps);

    // ---- stage this slice's activations: piece p = 4u + i -> qs[i * nch + u]
    const int8_t *qrow = a.q + (int64_t)m * a.ldq;
    int qsum = 0;
    for (int p = threadIdx.x; p < 4 * nch; p += kThreads) {
        const int64_t k0 = (int64_t)c0 * 64 + (int64_t)p * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (k0 + 16 <= a.K && ((reinterpret_cast<uintptr_t>(qrow + k0) & 15) == 0)) {
            v = *reinterpret_cast<const uint4 *>(qrow + k0);
        } else if (k0 < a.K) {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            for (int t = 0; t < 16 && k0 + t < a.K; ++t)
                w[t >> 2] |= (uint32_t)(uint8_t)qrow[k0 + t] << (8 * (t & 3));
            v = make_uint4(w[0], w[1], w[2], w[3]);
        }
        qs[(p & 3) * nch + (p >> 2)] = v;
        qsum = dp4a_us(0x01010101u, v.x, qsum);
        qsum = dp4a_us(0x01010101u, v.y, qsum);
        qsum = dp4a_us(0x01010101u, v.z, qsum);
        qsum = dp4a_us(0x01010101u, v.w, qsum);
    }
    qsum = block_reduce(qsum, [](int x, int y) { return x + y; }, red);  // also a barrier for qs

    // ---- stream rows
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / G, l = lane % G;
    constexpr int RT = (32 / G) * R;
    const int64_t n_tasks = ceil_div(a.N, RT);
    const int64_t tw = (int64_t)gridDim.x * (kThreads / 32);
    const uint8_t *wbase = a.W + (int64_t)c0 * 16;

    for (int64_t t = (int64_t)blockIdx.x * (kThreads / 32) + warp; t < n_tasks; t += tw) {
        const int64_t nb = t * RT + grp * R;
        const uint8_t *wrow[R];
        bool valid[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            valid[r] = nb + r < a.N;
            wrow[r] = wbase + (valid[r] ? nb + r : 0) * a.row_bytes;
        }
        int acc[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0;

        for (int u = l; u < nch; u += G * UN) {
            uint4 wv[UN][R];
#pragma unroll
            for (int s = 0; s < UN; ++s) {
                const int uu = u + s * G;
#pragma unroll
                for (int r = 0; r < R; ++r)
                    wv[s][r] = (uu < nch && valid[r]) ? ldg_stream_v4(wrow[r] + (int64_t)uu * 16)
                                                      : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int s = 0; s < UN; ++s) {
                const int uu = u + s * G;
                if (uu < nch) {
                    const uint4 x0 = qs[uu], x1 = qs[nch + uu], x2 = qs[2 * nch + uu], x3 = qs[3 * nch + uu];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        mac_word(acc[r], wv[s][r].x, x0);
                        mac_word(acc[r], wv[s][r].y, x1);
                        mac_word(acc[r], wv[s][r].z, x2);
                        mac_word(acc[r], wv[s][r].w, x3);
                    }
                }
            }
        }

        int tot[R];
#pragma unroll
        for (int r = 0; r < R; ++r)
            tot[r] = acc[r][0] + (acc[r][1] >> 2) + (acc[r][2] >> 4) + (acc[r][3] >> 6);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1)
#pragma unroll
            for (int r = 0; r < R; ++r) tot[r] += __shfl_xor_sync(0xffffffffu, tot[r], o);
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (l == r && valid[r]) gemv_store(a, m, nb + r, tot[r] - qsum);
    }
}

// Split-K reduction: y[m, n] = sum over slices, in slice order, then the epilogue.
__global__ void __launch_bounds__(kThreads) gemv_splitk_reduce_kernel(const GemvArgs a, int S) {
    const int64_t MN = (int64_t)a.M * a.N;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t o = (int64_t)blockIdx.x * kThreads + threadIdx.x; o < MN; o += stride) {
        int acc = 0;
        for (int s = 0; s < S; ++s) acc += a.partial[(int64_t)s * MN + o];
        const int m = (int)(o / a.N);
        if (a.y_bf16 != nullptr) {
            const float f = __fdiv_rn(*a.gamma, a.s_act[m]);
            a.y_bf16[o] = float_to_bf16_bits_rn(__fmul_rn((float)acc, f));
        } else {
            a.y_i32[o] = acc;
        }
    }
}

}  // namespace bitnet
