// gemm_tc.cuh -- the M > 1 W2A8 contraction on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, accumulators in tensor memory).
//
//   acc[m, n] = sum_k q[m, k] * c[n, k],   c = w + 1 in {0, 1, 2}
//   y[m, n]   = acc[m, n] - sum_k q[m, k]                             (exact)
//
// The pages have no M > 1 kernel: their GEMV handles M == 1 only (page "如何编
// 译 BitNet W2A8 CUDA 内核并用 test.py 运行 GEMV 加速测试？", section 限制与注意
// 事项).  Design:
//   - CTA tile: 128 tokens (UMMA M) x BN weight rows (UMMA N) x 128 k per stage.
//   - Warp 0, one lane: TMA producer.  Per stage it loads the activation tile
//     (int8 [128 x 128 bytes], 128-byte swizzle: the canonical K-major operand
//     layout) into a ring of SAB stages and the packed weight tile (layout v1,
//     [BN rows x 32 bytes], 32-byte swizzle) into a ring of SP stages.
//   - Warps 2..5: decoders.  Each 32-bit packed word (16 consecutive k of one
//     row) becomes 16 code bytes ((word >> 2j) & 0x03030303, j = 0..3), stored
//     as the row's 16-byte chunk in the same swizzled K-major layout; then a
//     proxy fence and an mbarrier arrival hand the tile to the tensor core.
//   - Warp 1: allocates tensor memory and, from one lane, issues per stage four
//     K = 32 MMAs of 128 x BN (int8 activations x codes 0..2 -> s32) plus four
//     128 x 16 MMAs against a constant tile of ones, which leave sum_k q[m, k]
//     in 16 extra accumulator columns: the correction for the +1 code offset
//     comes out of the tensor core, with no extra pass over q.
//     tcgen05.commit on a per-stage mbarrier releases the stage.
//   - After the last stage, warps 2..5 read the accumulators (tcgen05.ld, one
//     row per thread), subtract the row sum and either keep int32 or scale by
//     gamma / s_m to bf16, stage 32-row boxes in the freed operand ring with
//     the 128-byte swizzle and write them with TMA stores (full lines); direct
//     stores are the fallback when the output rows are not 16-byte strided.
//   - Split-K (gridDim.z > 1, for problems with fewer tiles than SMs): each
//     split covers a range of k stages, subtracts its own share of the row
//     sums, and adds its int32 results into a zeroed output with TMA
//     reduce-add stores (integer adds: exact and order-free).
//   - Every mbarrier wait is bounded in time; a role that gives up records
//     BITNET_ERR_DEVICE_TIMEOUT and raises a shared abort flag that stops the
//     others; all roles then drain what they issued (bounded) and tensor
//     memory is freed before the CTA exits.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemv_tma.cuh"

namespace bitnet {

constexpr int kTcBM = 128;              // tokens per tile (UMMA M)
constexpr int kTcBK = 128;              // k per stage (bytes of an activation row)
constexpr int kTcThreads = 192;         // 6 warps
constexpr int kTcAStageBytes = kTcBM * kTcBK;  // 16 KB
constexpr int kTcOnesRows = 16;

struct GemmTcArgs {
    int64_t M, N, K;
    int nk;                 // k stages: K_pad / 128
    int tma_store;          // 1: outputs leave through TMA stores of swizzled boxes (y rows 16-byte strided)
    int sps;                // k stages per split (split-K over gridDim.z)
    int reduce;             // 1: add int32 results into the (zeroed) output instead of storing them
    int32_t *y_i32;         // [M, N] int32 result
    uint16_t *y_bf16;       // [M, N] bf16 result (BitLinear)
    const float *s_act;     // [M] activation scales (BitLinear)
    const float *gamma;     // weight scale (BitLinear)
};

// Shared-memory plan: SAB stages of (activation tile, decoded code tile), SP
// stages of packed tiles (consumed by the decoders as soon as they land).
template <int BN, int SAB, int SP>
struct TcSmem {
    static constexpr int kBStage = BN * kTcBK;      // decoded codes
    static constexpr int kPStage = BN * 32;         // packed bytes
    static constexpr int kA = 0;
    static constexpr int kB = kA + SAB * kTcAStageBytes;
    static constexpr int kP = kB + SAB * kBStage;
    static constexpr int kOnes = kP + SP * kPStage;   // 1024-aligned: all the above are multiples of 1 KB
    static constexpr int kBars = kOnes + kTcOnesRows * kTcBK;
    static constexpr int kBarCount = 3 * SAB + 2 * SP + 2;  // a_full, dec_full, mma_done, p_full, p_empty, accum, drain
    static constexpr int kMisc = kBars + kBarCount * 8;      // tmem base (4 B) + abort flag (4 B)
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kTmemCols = (BN + kTcOnesRows) <= 128 ? 128 : ((BN + kTcOnesRows) <= 256 ? 256 : 512);
};

__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
    // start address >> 4 (bits 0-13), leading byte offset 16 B (ignored for
    // swizzled K-major), stride byte offset 1024 B between 8-row groups,
    // descriptor version 1 (bits 46-47), 128-byte swizzle (layout type 2)
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kind::i8 instruction descriptor: s32 accumulate, A and B signed 8-bit (the
// codes 0, 1, 2 are the same bytes as unsigned), both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcBM >> 4) << 24);
}

__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Bounded wait that also gives up when another role has raised the abort flag.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            record_device_error(BITNET_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    tma_load_box(dst, map, x, y, bar);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, const void *src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
                 "r"(y), "r"(smem_u32(src))
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until at most n committed bulk stores still read shared memory.
template <int n>
__device__ __forceinline__ void tma_store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}

__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Element-wise add of a shared-memory box into global memory (exact for s32).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap *map, int x, int y, const void *src) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

template <int BN, bool BF16_OUT, int SAB, int SP>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_w2a8_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap pmap,
                        const __grid_constant__ CUtensorMap ymap, const GemmTcArgs a) {
    using L = TcSmem<BN, SAB, SP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBars);
    uint64_t *a_full = bars;
    uint64_t *dec_full = bars + SAB;
    uint64_t *mma_done = bars + 2 * SAB;
    uint64_t *p_full = bars + 3 * SAB;
    uint64_t *p_empty = p_full + SP;
    uint64_t *accum_full = p_empty + SP;
    uint64_t *drain = accum_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * BN, m0 = (int64_t)blockIdx.y * kTcBM;
    const int kbase = blockIdx.z * a.sps;  // this split's first k stage
    const int nk = min(a.sps, a.nk - kbase);

    // ---- set-up: barriers, the ones tile, tensor memory
    if (threadIdx.x == 0) {
        for (int s = 0; s < SAB; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&dec_full[s], 4);   // one arrival per decoder warp
            mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < SP; ++s) {
            mbar_init(&p_full[s], 1);
            mbar_init(&p_empty[s], 4);    // one arrival per decoder warp
        }
        mbar_init(accum_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
    }
    for (int i = threadIdx.x; i < kTcOnesRows * kTcBK / 16; i += kTcThreads)
        reinterpret_cast<uint4 *>(sm + L::kOnes)[i] = make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // ones tile -> tensor core
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(L::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // weights never depend on an earlier kernel; activations may
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            pdl_wait();
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % SAB, ps = kb % SP;
                if (kb >= SAB && !tc_wait(&mma_done[s], (uint32_t)((kb / SAB) - 1) & 1u, abort_flag)) break;
                if (kb >= SP && !tc_wait(&p_empty[ps], (uint32_t)((kb / SP) - 1) & 1u, abort_flag)) break;
                mbar_arrive_expect_tx(&a_full[s], kTcAStageBytes);
                tma_load_2d(sm + L::kA + s * kTcAStageBytes, &amap, (kbase + kb) * kTcBK, (int)m0, &a_full[s]);
                mbar_arrive_expect_tx(&p_full[ps], L::kPStage);
                tma_load_2d(sm + L::kP + ps * L::kPStage, &pmap, (kbase + kb) * 32, (int)n0, &p_full[ps]);
                issued = kb + 1;
            }
            // make sure no copy is still landing in shared memory when the CTA leaves
            for (int kb = issued - SAB < 0 ? 0 : issued - SAB; kb < issued; ++kb)
                mbar_wait_bounded(&a_full[kb % SAB], (uint32_t)(kb / SAB) & 1u);
            for (int kb = issued - SP < 0 ? 0 : issued - SP; kb < issued; ++kb)
                mbar_wait_bounded(&p_full[kb % SP], (uint32_t)(kb / SP) & 1u);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_i8(BN);
            const uint32_t idesc1 = umma_idesc_i8(kTcOnesRows);
            const uint32_t ones = smem_u32(sm + L::kOnes);
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % SAB;
                if (!tc_wait(&dec_full[s], (uint32_t)(kb / SAB) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t as = smem_u32(sm + L::kA + s * kTcAStageBytes);
                const uint32_t bs = smem_u32(sm + L::kB + s * L::kBStage);
#pragma unroll
                for (int kk = 0; kk < kTcBK / 32; ++kk) {
                    const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                    const uint64_t ad = umma_desc_sw128(as + kk * 32);
                    umma_i8(tmem, ad, umma_desc_sw128(bs + kk * 32), idesc, acc);
                    umma_i8(tmem + BN, ad, umma_desc_sw128(ones + kk * 32), idesc1, acc);
                }
                umma_commit(&mma_done[s]);
            }
            if (ok) {
                umma_commit(accum_full);
            } else {
                // drain the MMAs already issued before tensor memory is released
                umma_commit(drain);
                mbar_wait_bounded(drain, 0);
            }
        }
    } else {
        // ---------------------------------------------------------------- decoders, then epilogue
        const int t = threadIdx.x - 64;  // 0..127
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % SAB, pst = kb % SP;
            // the packed tile has landed; the activation tile of this stage has too,
            // which also means the MMAs that last read this stage's code tile are done
            if (!tc_wait(&p_full[pst], (uint32_t)(kb / SP) & 1u, abort_flag) ||
                !tc_wait(&a_full[s], (uint32_t)(kb / SAB) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            const uint8_t *ps = sm + L::kP + pst * L::kPStage;
            uint8_t *bs = sm + L::kB + s * L::kBStage;
#pragma unroll
            for (int n = t; n < BN; n += 128) {
                // the packed tile arrives with the 32-byte swizzle: 16-byte half h of
                // row n sits at n * 32 + ((h ^ ((n >> 2) & 1)) * 16)
                const int sw = (n >> 2) & 1;
                const uint4 p0 = *reinterpret_cast<const uint4 *>(ps + n * 32 + (sw << 4));
                const uint4 p1 = *reinterpret_cast<const uint4 *>(ps + n * 32 + ((sw ^ 1) << 4));
                const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                uint8_t *row = bs + n * kTcBK;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 c = make_uint4(w[i] & 0x03030303u, (w[i] >> 2) & 0x03030303u,
                                               (w[i] >> 4) & 0x03030303u, (w[i] >> 6) & 0x03030303u);
                    *reinterpret_cast<uint4 *>(row + ((i ^ (n & 7)) << 4)) = c;
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // codes -> tensor core
            __syncwarp();
            if (lane == 0) {
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&p_empty[pst])) : "memory");
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&dec_full[s])) : "memory");
            }
        }
        // epilogue: thread t owns accumulator row (warp % 4) * 32 + lane
        if (ok && tc_wait(accum_full, 0, abort_flag)) {
            tc_fence_after();
            const int quarter = warp & 3;
            const int row = quarter * 32 + lane;
            const int64_t m = m0 + row;
            const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16);
            uint32_t v[16];
            tmem_ld16(tbase + BN, v);
            const int rowsum = (int)v[0];
            float f = 0.0f;
            if (BF16_OUT && m < a.M) f = __fdiv_rn(*a.gamma, a.s_act[m]);
            pdl_wait();  // the outputs may still be read by the previous kernel
            if (a.tma_store) {
                // Stage 32-row boxes (128 bytes per row: 32 int32 or 64 bf16 values)
                // in the freed activation ring with the 128-byte swizzle (thread =
                // row, conflict-free), two buffers per warp, and store each box
                // with one TMA store; the TMA unit clips rows >= M and columns >= N.
                constexpr int kCols = BF16_OUT ? 64 : 32;
                uint8_t *wbuf = sm + L::kA + quarter * 2 * 4096;
#pragma unroll 1
                for (int c = 0, it = 0; c < BN; c += kCols, ++it) {
                    uint8_t *buf = wbuf + (it & 1) * 4096;
                    if (it >= 2) {
                        if (lane == 0) tma_store_wait_read<1>();
                        __syncwarp();
                    }
                    uint32_t packed_row[32];
                    if (BF16_OUT) {
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            tmem_ld16(tbase + c + 16 * h, v);
#pragma unroll
                            for (int i = 0; i < 16; i += 2) {
                                const uint32_t lo = float_to_bf16_bits_rn(__fmul_rn((float)((int)v[i] - rowsum), f));
                                const uint32_t hi = float_to_bf16_bits_rn(__fmul_rn((float)((int)v[i + 1] - rowsum), f));
                                packed_row[8 * h + i / 2] = lo | (hi << 16);
                            }
                        }
                    } else {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            tmem_ld16(tbase + c + 16 * h, v);
#pragma unroll
                            for (int i = 0; i < 16; ++i) packed_row[16 * h + i] = (uint32_t)((int)v[i] - rowsum);
                        }
                    }
                    uint8_t *rowp = buf + lane * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4 *>(rowp + ((j ^ (lane & 7)) << 4)) =
                            make_uint4(packed_row[4 * j], packed_row[4 * j + 1], packed_row[4 * j + 2],
                                       packed_row[4 * j + 3]);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        if (a.reduce)
                            tma_reduce_add_2d(&ymap, (int)(n0 + c), (int)(m0 + quarter * 32), buf);
                        else
                            tma_store_2d(&ymap, (int)(n0 + c), (int)(m0 + quarter * 32), buf);
                    }
                }
                if (lane == 0) tma_store_wait_all();
                __syncwarp();
            } else {
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    tmem_ld16(tbase + c, v);
                    if (m < a.M) {
                        const int64_t nb = n0 + c;
                        if (BF16_OUT) {
                            uint16_t *dst = a.y_bf16 + m * a.N + nb;
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                if (nb + i < a.N)
                                    dst[i] = float_to_bf16_bits_rn(__fmul_rn((float)((int)v[i] - rowsum), f));
                        } else {
                            int32_t *dst = a.y_i32 + m * a.N + nb;
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                if (nb + i < a.N) {
                                    if (a.reduce)
                                        atomicAdd(dst + i, (int)v[i] - rowsum);
                                    else
                                        dst[i] = (int)v[i] - rowsum;
                                }
                            }
                        }
                    }
                }
            }
        }
    }

    // ---- teardown: every tensor-memory access is complete before the free
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::kTmemCols)
                     : "memory");
    }
}

}  // namespace bitnet
