// gemm_tc.cuh -- the M > 1 W2A8 contraction on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, accumulators in tensor memory).
//
//   y[m, n] = sum_k q[m, k] * w[n, k],   w = c - 1 in {-1, 0, 1}     (exact, int32)
//
// The pages have no M > 1 kernel: their GEMV handles M == 1 only (page "如何编
// 译 BitNet W2A8 CUDA 内核并用 test.py 运行 GEMV 加速测试？", section 限制与注意
// 事项).  Design: the ternary weights are the MMA's A operand and live in
// tensor memory, so decoded weights never pass through shared memory; the
// kernel is persistent, one CTA per SM looping over work units.
//   - Work unit: 128 weight rows (UMMA M) x BT tokens (UMMA N) x one K-split;
//     units are dealt round-robin to the CTAs, weight-row tiles fastest.  A
//     unit is done in stages of 256 k (8 MMAs per hand-over between decoders
//     and tensor core: on B200 the hand-overs, not the MMAs, bounded the stage
//     rate at 128 k per stage); its accumulator D[n, m] takes 128 TMEM
//     lanes x BT columns, and two accumulators alternate so that one unit's
//     epilogue overlaps the next unit's main loop.
//   - Warp 0, one lane: TMA producer of two rings that run on across units,
//     each with full / empty mbarriers: activation tiles (two int8 boxes of
//     [BT tokens x 128 bytes], 128-byte swizzle: the canonical K-major B
//     operand; SA stages) and packed weight tiles (layout v1, [128 rows x 64
//     bytes], 64-byte swizzle; SP stages).  The first packed tiles are requested before
//     griddepcontrol.wait (weights never depend on an earlier kernel).
//   - Warps 2..9: decoders, two groups of four that take alternate stages (a
//     group's tensor-memory store latency hides behind the other group's
//     work).  A thread owns one weight row (its warp's TMEM lane quarter).
//     Per stage the row's 16 packed words (256 k) become 64 words of
//     signed codes: (word >> 2j) & 0x03030303 gives the codes c of 4
//     consecutive k, and ((c + 0x7F7F7F7F) ^ 0x80808080) is c - 1 in every
//     byte with no carry between bytes.  Two tcgen05.st write the 64 words
//     into a code stage of tensor memory (SC stages of 64 columns).
//   - Warp 1: allocates tensor memory and, from one lane, issues per stage
//     eight K = 32 MMAs (A = codes in tensor memory, B = activations in shared
//     memory, s8 x s8 -> s32) into the unit's accumulator; tcgen05.commit on
//     per-stage mbarriers releases the activation and code stages, and on a
//     per-accumulator mbarrier hands a finished unit to the epilogue.
//   - Warps 10..13: epilogue.  They read an accumulator (tcgen05.ld: one weight
//     row per thread, 16 tokens per load), keep int32 or scale by gamma / s_m
//     to bf16, stage 32-token x 32-row boxes in shared memory for TMA stores
//     (direct stores when the output rows are not 16-byte strided) and release
//     the accumulator.
//   - Split-K (for problems with fewer tiles than SMs): each split covers a
//     range of k stages and adds its int32 partial sums into a zeroed output
//     with TMA reduce-add stores (integer adds: exact and order-free).
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

constexpr int kTcRows = 128;            // weight rows per tile (UMMA M)
constexpr int kTcBK = 128;              // k per activation box (bytes of a 128-byte swizzled row)
constexpr int kTcDecGroups = 2;        // decoder groups of 4 warps, taking alternate stages
constexpr int kTcEpiWarp = 2 + 4 * kTcDecGroups;   // first epilogue warp
constexpr int kTcThreads = 32 * (kTcEpiWarp + 4);  // producer, MMA, decoders, 4 epilogue warps
constexpr int kTcBox = 32;              // output box: 32 tokens x 32 weight rows
constexpr int kTcEpiBufs = 2;          // 4 KB output staging buffers per epilogue warp

struct GemmTcArgs {
    int64_t M, N, K;
    int nk;                 // k stages: K_pad / 128
    int tiles_n, tiles_m;   // weight-row tiles (128 rows) and token tiles (BT tokens)
    int splits;             // K-splits; work units = tiles_n * tiles_m * splits
    int tma_store;          // 1: outputs leave through TMA stores of boxes (y rows 16-byte strided)
    int sps;                // k stages per split (split-K over gridDim.z)
    int reduce;             // 1: add int32 results into the (zeroed) output instead of storing them
    int32_t *y_i32;         // [M, N] int32 result
    uint16_t *y_bf16;       // [M, N] bf16 result (BitLinear)
    const float *s_act;     // [M] activation scales (BitLinear)
    const float *gamma;     // weight scale (BitLinear)
    // BitLinear with the quantisation inside this launch (x != null): bf16
    // activations x [M, K] are quantised by the epilogue warps of every CTA into
    // qout (rows of ldq bytes, zero-padded: the tensor the activation map
    // reads) and s_act; the CTAs then meet at grid barrier `bar_slot` before
    // the first activation load
    const uint16_t *x;
    int8_t *qout;
    int64_t ldq;
    int bar_slot;
};

// Grid barriers for launches whose CTAs must all finish a phase before any
// goes on (every CTA of such a launch is resident: one per SM at most).  A
// barrier is one word in device memory owned by this library (zero at load):
// each CTA adds 1, CTA 0 adds 2^31 - (G - 1), so the top bit flips exactly
// when all G have arrived and the low bits return to where they were: the
// word is ready for its next use with no reset, replayed CUDA graphs
// included.  Calls take slots in turn, so launches that overlap on the GPU
// (consecutive calls under programmatic launch) use different words.
constexpr int kGridBarSlots = 1024;
__device__ unsigned int g_grid_bar[kGridBarSlots];

__device__ __forceinline__ unsigned int ld_acquire_u32g(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Arrival of this CTA (one thread; its CTA's writes made visible before);
// returns the word as it was before, for grid_bar_wait.
__device__ __forceinline__ unsigned int grid_bar_arrive(int slot) {
    __threadfence();
    const unsigned int inc = blockIdx.x == 0 ? 0x80000000u - (gridDim.x - 1) : 1u;
    return atomicAdd(&g_grid_bar[slot], inc);
}

// Bounded wait for the flip; false after the limit or when another role
// raised the abort flag.
__device__ __forceinline__ bool grid_bar_wait(int slot, unsigned int old, volatile int *abort_flag) {
    if ((ld_acquire_u32g(&g_grid_bar[slot]) ^ old) & 0x80000000u) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        __nanosleep(32);
        if ((ld_acquire_u32g(&g_grid_bar[slot]) ^ old) & 0x80000000u) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            record_device_error(BITNET_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// Shared-memory plan: SA activation stages, SP packed stages, the epilogue's
// output boxes (4 warps x kTcEpiBufs x 4 KB), mbarriers, the tensor-memory base and the
// abort flag.  Tensor memory: NACC accumulators of BT columns (two let a
// unit's epilogue overlap the next unit's main loop; one leaves room for more
// code stages), then SC code stages of SK / 4 columns.
template <int BT, int SA, int SC, int SP, int SK, int NACC = 2>
struct TcSmem {
    static_assert(SK == 256 || SK == 512, "k per stage");
    static constexpr int kABoxes = SK / kTcBK;                   // activation boxes per stage
    static constexpr int kPRow = SK / 4;                         // packed bytes of a weight row per stage
    static constexpr int kPChunks = kPRow / 16;                  // its 16-byte chunks (4 or 8)
    static constexpr int kPStage = kTcRows * kPRow;              // packed bytes per stage
    static constexpr int kAHalf = BT * kTcBK;                    // one activation box
    static constexpr int kAStage = kABoxes * kAHalf;
    static constexpr int kA = 0;
    static constexpr int kP = kA + SA * kAStage;                 // 1024-aligned (multiples of 1 KB)
    static constexpr int kE = kP + SP * kPStage;
    static constexpr int kBars = kE + 4 * kTcEpiBufs * 4096;
    // a_full, a_empty, p_full, p_empty, c_full, c_empty, accum_full x 2, accum_empty x 2, drain
    static constexpr int kBarCount = 2 * SA + 2 * SP + 2 * SC + 5;
    static constexpr int kMisc = kBars + kBarCount * 8;
    static constexpr int kBytes = kMisc + 16;
    static_assert(NACC == 1 || NACC == 2, "accumulators");
    static constexpr int kCodeCol = NACC * BT;                   // first code-stage column
    static constexpr int kCodeCols = SK / 4;                     // 32-bit columns of one code stage
    static constexpr int kTmemNeed = NACC * BT + kCodeCols * SC;
    static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
    static_assert(kTmemNeed <= 512, "tensor memory");
    static_assert(kAHalf % 1024 == 0, "128-byte swizzled boxes are 1024-byte aligned");
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

// kind::i8 instruction descriptor: s32 accumulate, A and B signed 8-bit, both
// K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);
}

// D (tensor memory) (+)= A (tensor memory) x B (shared memory descriptor).
__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
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

// Writes 32 consecutive 32-bit columns of this thread's tensor-memory lane
// (tcgen05.wait::st, below, waits until such writes are done).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Work unit u -> (split, token tile, weight-row tile), weight-row tiles fastest.
struct TcUnit {
    int z, mt, nt;
};
__device__ __forceinline__ TcUnit tc_unit(const GemmTcArgs &a, int u) {
    TcUnit t;
    t.nt = u % a.tiles_n;
    const int r = u / a.tiles_n;
    t.mt = r % a.tiles_m;
    t.z = r / a.tiles_m;
    return t;
}

template <int BT, bool BF16_OUT, int SA, int SC, int SP, int SK, int NACC = 2>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_w2a8_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap pmap,
                        const __grid_constant__ CUtensorMap ymap, const GemmTcArgs a) {
    using L = TcSmem<BT, SA, SC, SP, SK, NACC>;
    static_assert(BT % 16 == 0 && BT <= 256, "token tile");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBars);
    uint64_t *a_full = bars;
    uint64_t *a_empty = a_full + SA;
    uint64_t *p_full = a_empty + SA;
    uint64_t *p_empty = p_full + SP;
    uint64_t *c_full = p_empty + SP;
    uint64_t *c_empty = c_full + SC;
    uint64_t *accum_full = c_empty + SC;   // [2]
    uint64_t *accum_empty = accum_full + 2; // [2]
    uint64_t *drain = accum_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int units = a.tiles_n * a.tiles_m * a.splits;
    auto unit_stages = [&](const TcUnit &t) { return min(a.sps, a.nk - t.z * a.sps); };

    // ---- set-up: descriptors, barriers, tensor memory
    if (threadIdx.x == 0) {
        prefetch_tensormap(&pmap);
        prefetch_tensormap(&amap);
        if (a.tma_store) prefetch_tensormap(&ymap);
        for (int s = 0; s < SA; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);    // tcgen05.commit
        }
        for (int s = 0; s < SP; ++s) {
            mbar_init(&p_full[s], 1);
            mbar_init(&p_empty[s], 4);    // one arrival per decoder warp
        }
        for (int s = 0; s < SC; ++s) {
            mbar_init(&c_full[s], 4);     // one arrival per decoder warp
            mbar_init(&c_empty[s], 1);    // tcgen05.commit
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(&accum_full[d], 1);   // tcgen05.commit
            mbar_init(&accum_empty[d], 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
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

    pdl_launch_dependents();

    if (a.x != nullptr && warp >= kTcEpiWarp) {
        // quantisation phase (the four epilogue warps, idle until the first
        // accumulator is done: one token row per warp at a time, rows dealt
        // over all CTAs) while the decoders turn the first packed stages into
        // codes.  x may come from the previous kernel and q / s may still be
        // read by it: wait for it first.
        pdl_wait();
        constexpr int kQWarps = 4;
        int rows = 0;
        for (int64_t m = (int64_t)blockIdx.x * kQWarps + (warp - kTcEpiWarp); m < a.M;
             m += (int64_t)gridDim.x * kQWarps) {
            int sum = 0;
            const float sc = quant_row<1>(a.x + m * a.K, a.K, a.qout + m * a.ldq, a.ldq, true, false, sum, nullptr,
                                          nullptr, 0, lane);
            if (lane == 0) const_cast<float *>(a.s_act)[m] = sc;
            ++rows;
        }
        (void)rows;
        // every lane's rows visible at gpu scope (and to the async proxy), then
        // meet the producer, which arrives at the grid barrier for the CTA
        __threadfence();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        asm volatile("bar.sync 1, %0;" ::"n"(5 * 32) : "memory");
    }

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        // cursors (unit, stage) of the next activation and packed loads; ia /
        // ip count the loads issued over all of this CTA's units (lane 0 only)
        int ua = blockIdx.x, ka = 0, up = blockIdx.x, kp = 0, ia = 0, ip = 0;
        TcUnit ta = tc_unit(a, ua), tp = ta;
        auto issue_p = [&]() {
            mbar_arrive_expect_tx(&p_full[ip % SP], L::kPStage);
            tma_load_2d(sm + L::kP + (ip % SP) * L::kPStage, &pmap, (tp.z * a.sps + kp) * L::kPRow, tp.nt * kTcRows,
                        &p_full[ip % SP]);
            ++ip;
            if (++kp == unit_stages(tp)) {
                kp = 0;
                up += gridDim.x;
                if (up < units) tp = tc_unit(a, up);
            }
        };
        // weights never depend on an earlier kernel; activations may
        if (lane == 0)
            while (up < units && ip < SP) issue_p();
        // quantisation inside this launch: this CTA's quantisation warps are
        // done, then every CTA's (grid barrier), so every row of q, written
        // through the generic proxy, is in place before the first TMA read
        bool q_ready = true;
        if (a.x != nullptr) {
            __syncwarp();
            asm volatile("bar.sync 1, %0;" ::"n"(5 * 32) : "memory");  // with the four quantising warps
            if (lane == 0) {
                const unsigned int old = grid_bar_arrive(a.bar_slot);
                q_ready = grid_bar_wait(a.bar_slot, old, abort_flag);
                asm volatile("fence.proxy.async.global;" ::: "memory");
            }
        }
        if (lane == 0) {
            pdl_wait();
            if (!q_ready) ua = up = units;  // aborted: issue nothing more
            // poll both rings without blocking on either (a blocking wait on one
            // would hold back the other); the idle time is bounded like every wait
            uint64_t idle_since = 0;
            while (ua < units || up < units) {
                bool issued = false;
                if (ua < units && (ia < SA || mbar_test_wait(&a_empty[ia % SA], (uint32_t)((ia / SA) - 1) & 1u))) {
                    mbar_arrive_expect_tx(&a_full[ia % SA], L::kAStage);
                    const int kx = (ta.z * a.sps + ka) * SK;
                    uint8_t *ad = sm + L::kA + (ia % SA) * L::kAStage;
#pragma unroll
                    for (int h = 0; h < L::kABoxes; ++h)
                        tma_load_2d(ad + h * L::kAHalf, &amap, kx + h * kTcBK, ta.mt * BT, &a_full[ia % SA]);
                    ++ia;
                    if (++ka == unit_stages(ta)) {
                        ka = 0;
                        ua += gridDim.x;
                        if (ua < units) ta = tc_unit(a, ua);
                    }
                    issued = true;
                }
                if (up < units && mbar_test_wait(&p_empty[ip % SP], (uint32_t)((ip / SP) - 1) & 1u)) {
                    issue_p();
                    issued = true;
                }
                if (issued) {
                    idle_since = 0;
                    continue;
                }
                if (*abort_flag) break;
                const uint64_t now = global_timer_ns();
                if (idle_since == 0) {
                    idle_since = now;
                } else if (now - idle_since > kWaitLimitNs) {
                    record_device_error(BITNET_ERR_DEVICE_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                __nanosleep(20);
            }
            // make sure no copy is still landing in shared memory when the CTA leaves
            for (int i = ia - SA < 0 ? 0 : ia - SA; i < ia; ++i)
                mbar_wait_bounded(&a_full[i % SA], (uint32_t)(i / SA) & 1u);
            for (int i = ip - SP < 0 ? 0 : ip - SP; i < ip; ++i)
                mbar_wait_bounded(&p_full[i % SP], (uint32_t)(i / SP) & 1u);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_i8(BT);
            bool ok = true;
            int g = 0;  // stages consumed over all units
            int li = 0;
            for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++li) {
                const int d = li % NACC;
                // the epilogue has drained this accumulator's previous unit
                if (li >= NACC && !tc_wait(&accum_empty[d], (uint32_t)((li / NACC) - 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dt = tmem + (uint32_t)(d * BT);
                const int ns = unit_stages(tc_unit(a, u));
                for (int kb = 0; kb < ns; ++kb, ++g) {
                    const int sa = g % SA, sc = g % SC;
                    if (!tc_wait(&a_full[sa], (uint32_t)(g / SA) & 1u, abort_flag) ||
                        !tc_wait(&c_full[sc], (uint32_t)(g / SC) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t bs = smem_u32(sm + L::kA + sa * L::kAStage);
                    const uint32_t ac = tmem + (uint32_t)(L::kCodeCol + L::kCodeCols * sc);
#pragma unroll
                    for (int kk = 0; kk < SK / 32; ++kk)
                        umma_i8_ts(dt, ac + 8 * kk,
                                   umma_desc_sw128(bs + (kk >> 2) * L::kAHalf + (kk & 3) * 32), idesc,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&a_empty[sa]);
                    umma_commit(&c_empty[sc]);
                }
                if (ok) umma_commit(&accum_full[d]);
            }
            if (!ok) {
                // drain the MMAs already issued before tensor memory is released
                umma_commit(drain);
                mbar_wait_bounded(drain, 0);
            }
        }
    } else if (warp < kTcEpiWarp) {
        // ---------------------------------------------------------------- decoders
        const int quarter = warp & 3;            // tensor-memory lanes 32 * quarter ...
        const int group = (warp - 2) >> 2;       // stages g with g % kTcDecGroups == group
        const int row = quarter * 32 + lane;     // this thread's weight row in a tile
        const uint32_t tq = tmem + ((uint32_t)(quarter * 32) << 16);
        // packed rows arrive swizzled: 16-byte chunk c of row r at
        // r * kPRow + ((c ^ ((r >> (3 - log2 kPChunks)) & (kPChunks - 1))) * 16)
        // (the 64-byte swizzle for 4 chunks, the 128-byte one for 8)
        const int sw = (row >> (L::kPChunks == 8 ? 0 : 1)) & (L::kPChunks - 1);
        int g = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
            const int ns = unit_stages(tc_unit(a, u));
            for (int kb = 0; kb < ns; ++kb, ++g) {
                if (g % kTcDecGroups != group) continue;
                const int s = g % SC, ps = g % SP;
                // the packed tile has landed and the MMAs that last read this code stage are done
                if (!tc_wait(&p_full[ps], (uint32_t)(g / SP) & 1u, abort_flag) ||
                    (g >= SC && !tc_wait(&c_empty[s], (uint32_t)((g / SC) - 1) & 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t *pr = sm + L::kP + ps * L::kPStage + row * L::kPRow;
                uint32_t w[4 * L::kPChunks];
#pragma unroll
                for (int ch = 0; ch < L::kPChunks; ++ch) {
                    const uint4 p = *reinterpret_cast<const uint4 *>(pr + ((ch ^ sw) << 4));
                    w[4 * ch] = p.x;
                    w[4 * ch + 1] = p.y;
                    w[4 * ch + 2] = p.z;
                    w[4 * ch + 3] = p.w;
                }
                __syncwarp();  // every lane has its packed row in registers
                if (lane == 0)
                    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&p_empty[ps])) : "memory");
                const uint32_t cs = tq + (uint32_t)(L::kCodeCol + L::kCodeCols * s);
                // 16 packed words (256 k) -> 64 code words -> 64 columns at a time
#pragma unroll
                for (int gq = 0; gq < L::kPChunks / 4; ++gq) {
                    uint32_t c[64];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            c[4 * i + j] = (((w[16 * gq + i] >> (2 * j)) & 0x03030303u) + 0x7F7F7F7Fu) ^ 0x80808080u;
                    }
                    tmem_st32(cs + 64 * gq, c);
                    tmem_st32(cs + 64 * gq + 32, c + 32);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&c_full[s])) : "memory");
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t tq = tmem + ((uint32_t)(quarter * 32) << 16);
        uint8_t *wbuf = sm + L::kE + quarter * kTcEpiBufs * 4096;
        constexpr int kTok = BT < kTcBox ? BT : kTcBox;
        bool waited_pdl = false;
        int nbox = 0;  // boxes this warp has stored (its staging buffers take turns)
        int li = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++li) {
            const int d = li % NACC;
            if (!tc_wait(&accum_full[d], (uint32_t)(li / NACC) & 1u, abort_flag)) break;
            tc_fence_after();
            if (!waited_pdl) {
                pdl_wait();  // the outputs may still be read by the previous kernel
                // scales written in this launch by other CTAs: complete (the
                // MMAs waited for the grid barrier) and acquired here before use
                if (a.x != nullptr) (void)ld_acquire_u32g(&g_grid_bar[a.bar_slot]);
                waited_pdl = true;
            }
            const TcUnit t = tc_unit(a, u);
            const int64_t n0 = (int64_t)t.nt * kTcRows, m0 = (int64_t)t.mt * BT;
            const int64_t n = n0 + row;
            const uint32_t dt = tq + (uint32_t)(d * BT);
            // BitLinear factors gamma / s_m of the unit's tokens: a table per
            // epilogue warp in the upper half of its first staging buffer (bf16
            // boxes fill only the lower 2 KB), read back four at a time
            float *fac = reinterpret_cast<float *>(wbuf + 2048);
            if (BF16_OUT) {
                for (int c = lane; c < BT; c += 32) {
                    const int64_t m = m0 + c;
                    fac[c] = m < a.M ? __fdiv_rn(*a.gamma, a.s_act[m]) : 0.0f;
                }
                __syncwarp();
            }
            uint32_t v[16];
            if (a.tma_store) {
                // boxes of (up to) 32 tokens x 32 weight rows, row-major by token as y is
#pragma unroll 1
                for (int c0 = 0; c0 < BT; c0 += kTok, ++nbox) {
                    uint8_t *buf = wbuf + (nbox % kTcEpiBufs) * 4096;
                    if (nbox >= kTcEpiBufs) {
                        if (lane == 0) tma_store_wait_read<kTcEpiBufs - 1>();
                        __syncwarp();
                    }
#pragma unroll
                    for (int h = 0; h < kTok / 16; ++h) {
                        tmem_ld16(dt + (uint32_t)(c0 + 16 * h), v);
                        float f[16];
                        if (BF16_OUT) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float4 f4 = reinterpret_cast<const float4 *>(fac + c0 + 16 * h)[i];
                                f[4 * i] = f4.x, f[4 * i + 1] = f4.y, f[4 * i + 2] = f4.z, f[4 * i + 3] = f4.w;
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int tk = 16 * h + i;
                            if (BF16_OUT)
                                reinterpret_cast<uint16_t *>(buf)[tk * 32 + lane] =
                                    float_to_bf16_bits_rn(__fmul_rn((float)(int)v[i], f[i]));
                            else
                                reinterpret_cast<uint32_t *>(buf)[tk * 32 + lane] = v[i];
                        }
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        if (a.reduce)
                            tma_reduce_add_2d(&ymap, (int)(n0 + quarter * 32), (int)(m0 + c0), buf);
                        else
                            tma_store_2d(&ymap, (int)(n0 + quarter * 32), (int)(m0 + c0), buf);
                    }
                }
            } else {
#pragma unroll 1
                for (int c0 = 0; c0 < BT; c0 += 16) {
                    tmem_ld16(dt + (uint32_t)c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float f = BF16_OUT ? fac[c0 + i] : 0.0f;
                        const int64_t m = m0 + c0 + i;
                        if (n < a.N && m < a.M) {
                            if (BF16_OUT)
                                a.y_bf16[m * a.N + n] = float_to_bf16_bits_rn(__fmul_rn((float)(int)v[i], f));
                            else if (a.reduce)
                                atomicAdd(a.y_i32 + m * a.N + n, (int)v[i]);
                            else
                                a.y_i32[m * a.N + n] = (int)v[i];
                        }
                    }
                }
            }
            // every accumulator load of this unit is complete: release the accumulator
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&accum_empty[d])) : "memory");
        }
        if (lane == 0) tma_store_wait_all();
        __syncwarp();
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
