// gemv_tma.cuh -- the decode GEMV (one to sixteen tokens): packed weights
// stream through shared memory by TMA.
//
// Same contraction and decode as gemv.cuh (layout v1 words, codes scaled by
// 4^j, activation-sum correction); what differs is how the weights reach the
// lanes:
//   - The packed matrix is a 2-D byte tensor [N rows, K_pad/4 bytes].  A TMA
//     box is ROWS rows x 128 bytes (512 k): 32 rows (4 KB) or 16 rows (2 KB),
//     written to shared memory with the 128-byte swizzle (16-byte unit u of
//     box row r at r*128 + ((u ^ (r & 7)) * 16)), so that the reads below are
//     free of bank conflicts.  16-row blocks give shapes of fewer than 148
//     32-row blocks one block for every SM.
//   - Work items are (row block, 128-byte K-slice) pairs.  CTA b owns row
//     blocks b, b + gridDim.x, ...; its items, in (row block, slice) order, are
//     split into equal contiguous ranges, one per warp, which keeps every warp
//     busy for any K and makes a warp leave a row block at most a few times.
//   - Each warp has a private ring of NS boxes and one mbarrier per stage; its
//     lane 0 issues the TMA for the item NS ahead as soon as the warp has read
//     a stage, so up to NS boxes per warp are in flight without holding
//     registers.
//   - Activations live in shared memory as one linear array per token, staged
//     with all of a thread's loads in flight at once.
//   - The product: for one token, each lane takes one row (or half of one)
//     and dots its 16-byte chunks against the activations (all lanes read the
//     same 16 bytes: a broadcast) with dp4a; for 2..16 tokens (and, as a
//     tuned option, for one), the warp runs m16n8k32 integer MMAs over the box
//     (see gemv_tma_kernel), so that every weight box is read from HBM once
//     and the instruction count per box hardly grows with the tokens.
//   - A warp adds its per-row partial sums into a per-row-block int32
//     accumulator in shared memory (atomics: exact and order-free) whenever its
//     item sequence leaves a row block; the warp whose contribution completes
//     the block's item count writes the results.
//   - Every mbarrier wait is bounded in time.  A warp that gives up records
//     BITNET_ERR_DEVICE_TIMEOUT, waits (bounded) for its own boxes in flight and
//     stops; that row block's outputs are then left unwritten.
//   - Programmatic dependent launch as in gemv.cuh: the first boxes of every
//     warp are requested before griddepcontrol.wait.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int kTmaRows = 32;                                // rows per box at one lane per row
constexpr int kTmaSliceBytes = 128;                         // packed bytes per row per box
constexpr int kTmaSliceK = kTmaSliceBytes * 4;              // k values per box
constexpr uint64_t kWaitLimitNs = 1000000000ull;            // 1 s per wait

struct GemvTmaArgs {
    const int8_t *q;      // int8 activations [M, K] (mode 0)
    const uint16_t *x;    // bf16 activations [M, K] (mode 1)
    int M;                // tokens of this launch (<= the kernel's MT)
    int64_t N, K;
    int slices;           // K-slices of 128 packed bytes per row
    int64_t blk_begin;    // first row block of this launch
    int64_t nblocks;      // row blocks of this launch
    int max_blocks_cta;   // accumulator slots per CTA
    int ns;               // ring depth per warp: boxes in flight
    int32_t *y_i32;       // [M, N] int32 result
    uint16_t *y_bf16;     // [M, N] bf16 result (BitLinear)
    const float *gamma;   // weight scale (BitLinear)
    const float *s_act;   // mode 0 with bf16 output: per-token activation scales [M]
    int test_stall;       // test hook: warp 0 never requests its first box, so its first wait times out
    int evict_first;      // 1: weight boxes are read with the L2 evict-first policy
};

// Dynamic shared memory of a launch: ring of warps x stages boxes of `rows`
// rows, linear activations, per-row-block accumulators and counters, slice
// sums, mbarriers.
__host__ __device__ inline int64_t gemv_tma_token_stride(int slices, int tokens) {
    return (int64_t)slices * kTmaSliceK + (tokens > 1 ? 64 : 0);
}

__host__ __device__ inline size_t gemv_tma_smem_bytes(int warps, int stages, int slices, int max_blocks_cta,
                                                      int tokens = 1, int rows = kTmaRows) {
    return 1024 /* alignment slack */ + (size_t)warps * stages * rows * kTmaSliceBytes +
           (size_t)tokens * gemv_tma_token_stride(slices, tokens) + (size_t)max_blocks_cta * tokens * rows * 4 +
           (size_t)max_blocks_cta * 4 + 8 + (size_t)warps * stages * 8 + (size_t)tokens * slices * 4 +
           (size_t)slices * 8 /* slice barriers (one token, int8) */;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of the same (try_wait may suspend the thread for a while
// before it answers that the phase is not complete).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for the phase of the given parity to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// L2 policy for data read once per call (the packed weights): its lines are
// the first to go, so that what the next calls reuse stays in L2 (kernel
// code, activations, outputs, tensor maps).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_box_hint(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar,
                                                  uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
        "%3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_box(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------------ staging

// Adds up the 16-byte piece p of this lane into its K-slice's activation sum:
// a warp stages 32 consecutive pieces (p = 32 w' + lane), exactly one slice of
// 512 k, so one warp reduction gives the slice's sum.
__device__ __forceinline__ void slice_sum(int *qslice, int64_t p, const uint4 &v) {
    const int t = group_sum<32>(byte_sum(v, 0));
    if ((threadIdx.x & 31) == 0) qslice[p >> 5] = t;
}

// Pieces of 16 k a thread keeps in registers while staging: their loads are
// issued together, one memory round trip for all of them (a thread takes
// pieces threadIdx.x + i * blockDim.x, so a CTA of 512 threads stages 2048
// pieces, four 32 K-long rows or one of 32 K, per round trip).
constexpr int kStageHeld = 4;

// Cursor over a thread's pieces of the flat (token, piece) order, ppt pieces
// per token, stepping by blockDim.x without a division per step.
template <int MT>
struct PieceCursor {
    int t, pp, qb, rb, ppt;
    __device__ __forceinline__ explicit PieceCursor(int ppt_) : ppt(ppt_) {
        if (MT == 1) {
            t = 0, pp = threadIdx.x, qb = 0, rb = blockDim.x;
        } else {
            t = threadIdx.x / ppt, pp = threadIdx.x - t * ppt;
            qb = blockDim.x / ppt, rb = blockDim.x - qb * ppt;
        }
    }
    __device__ __forceinline__ bool valid() const { return MT == 1 ? pp < ppt : t < MT; }
    __device__ __forceinline__ void next() {
        pp += rb;
        if (MT > 1) {
            t += qb;
            if (pp >= ppt) pp -= ppt, ++t;
        }
    }
};

// Staging of int8 activations for MT token slots: qlin[t * ldx + k] = q[t * K
// + k] for t < M and k < K, 0 elsewhere up to kq (a multiple of 512), with
// the sum of every 512-k slice of token t in qslice[t * slices + j].  Piece p
// (16 k) of the flat (token, piece) order is staged by thread p mod blockDim.x;
// a warp takes 32 consecutive pieces, one slice of one token, so one warp
// reduction gives the slice's sum.  With slice_bar (one token), the warp then
// arrives on slice_bar[j] for each slice j it staged, so that a consumer waits
// for that slice alone rather than for the whole CTA.
template <int MT>
__device__ __forceinline__ void stage_tokens_int8(int8_t *qlin, int64_t ldx, int *qslice, int slices, const int8_t *q,
                                                  int M, int64_t K, int64_t kq, uint64_t *slice_bar = nullptr) {
    // sixteen tokens hold twice the pieces per round trip (16 tokens of 2560 k:
    // one round trip instead of two; measured on B200, 12 and 16 tokens 0.1 -
    // 0.25 us faster, while 8 tokens of 2560 k ran 0.23 us slower so)
    constexpr int kHeld = MT >= 16 ? 2 * kStageHeld : kStageHeld;
    PieceCursor<MT> cur((int)(kq / 16));  // ppt and blockDim.x are multiples of 32
    while (cur.valid()) {
        uint4 v[kHeld];
        int ts[kHeld], ps[kHeld];
#pragma unroll
        for (int i = 0; i < kHeld; ++i) {
            ts[i] = cur.valid() ? cur.t : MT, ps[i] = cur.pp;
            v[i] = make_uint4(0u, 0u, 0u, 0u);
            const int64_t k0 = (int64_t)ps[i] * 16;
            if (ts[i] < M && k0 < K) {
                const int8_t *qrow = q + (int64_t)ts[i] * K;
                if ((reinterpret_cast<uintptr_t>(qrow) & 15) == 0 && k0 + 16 <= K) {
                    v[i] = *reinterpret_cast<const uint4 *>(qrow + k0);
                } else {
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
                    for (int b = 0; b < 16 && k0 + b < K; ++b) w[b >> 2] |= (uint32_t)(uint8_t)qrow[k0 + b] << (8 * (b & 3));
                    v[i] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            cur.next();
        }
#pragma unroll
        for (int i = 0; i < kHeld; ++i) {
            if (ts[i] < MT) {  // warp-uniform
                *reinterpret_cast<uint4 *>(qlin + ts[i] * ldx + (int64_t)ps[i] * 16) = v[i];
                slice_sum(qslice + ts[i] * slices, ps[i], v[i]);
                if (slice_bar != nullptr) {
                    __syncwarp();  // every lane's piece and the sum are written
                    if ((threadIdx.x & 31) == 0)
                        asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(
                                         smem_u32(&slice_bar[ps[i] >> 5]))
                                     : "memory");
                }
            }
        }
    }
}

// Staging with fused per-token quantisation of bf16 activations (the same
// arithmetic as quant_act_kernel<>): every token's absmax over one pass that
// keeps the first kStageHeld pieces per thread in registers (loads issued
// together), one block reduction for all tokens, then the codes, with slice
// sums as above.  Pieces beyond those held are read again.  Returns the
// scales in sc; token slots t >= M are staged as zeros.  `red` holds MT x 32
// floats; NW is the CTA's warp count (the per-warp maxima are read back with
// all loads in flight at once).
template <int MT, int NW>
__device__ __forceinline__ void stage_tokens_bf16(int8_t *qlin, int64_t ldx, int *qslice, int slices, float *red,
                                                  const uint16_t *x, int M, int64_t K, int64_t kq, float (&sc)[MT]) {
    const int ppt = (int)(kq / 16);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    auto load = [&](int t, int pp, uint4 &lo, uint4 &hi) {
        lo = hi = make_uint4(0u, 0u, 0u, 0u);
        if (t < M) {
            const uint16_t *xr = x + (int64_t)t * K;
            load_x16(xr, K, pp, (reinterpret_cast<uintptr_t>(xr) & 15) == 0, lo, hi);
        }
    };
    float am[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) am[t] = 0.0f;
    auto amax_into = [&](int t, const uint4 &lo, const uint4 &hi) {
#pragma unroll
        for (int u = 0; u < MT; ++u)
            if (u == t) am[u] = amax16(lo, hi, am[u]);
    };
    PieceCursor<MT> cur(ppt);
    uint4 held[kStageHeld][2];
    int ts[kStageHeld], ps[kStageHeld];
#pragma unroll
    for (int i = 0; i < kStageHeld; ++i) {
        ts[i] = cur.valid() ? cur.t : MT, ps[i] = cur.pp;
        load(ts[i], ps[i], held[i][0], held[i][1]);
        cur.next();
    }
#pragma unroll
    for (int i = 0; i < kStageHeld; ++i) amax_into(ts[i], held[i][0], held[i][1]);
    PieceCursor<MT> rest = cur;
    for (; cur.valid(); cur.next()) {
        uint4 lo, hi;
        load(cur.t, cur.pp, lo, hi);
        amax_into(cur.t, lo, hi);
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        float v = am[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[t * 32 + warp] = v;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < NW; ++w) v = fmaxf(v, red[t * 32 + w]);
        sc[t] = t < M ? __fdiv_rn(127.0f, v > kQuantEps ? v : kQuantEps) : 0.0f;
    }
    auto put = [&](int t, int pp, const uint4 &lo, const uint4 &hi) {  // t < MT: warp-uniform
        float s = sc[0];
#pragma unroll
        for (int u = 1; u < MT; ++u)
            if (u == t) s = sc[u];
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (t < M) quant16(lo, hi, s, v);
        *reinterpret_cast<uint4 *>(qlin + t * ldx + (int64_t)pp * 16) = v;
        slice_sum(qslice + t * slices, pp, v);
    };
#pragma unroll
    for (int i = 0; i < kStageHeld; ++i)
        if (ts[i] < MT) put(ts[i], ps[i], held[i][0], held[i][1]);
    for (; rest.valid(); rest.next()) {
        uint4 lo, hi;
        load(rest.t, rest.pp, lo, hi);
        put(rest.t, rest.pp, lo, hi);
    }
}

// ------------------------------------------------------------------ kernel

// One m16n8k32 integer MMA on the warp's tensor-core path: A unsigned bytes
// (scaled 2-bit codes), B signed int8 activations, exact int32 accumulation.
// Fragments (PTX ISA, mma.m16n8k32 with 8-bit operands; g = lane / 4, t =
// lane % 4): a0 = A[g][4t..4t+3], a1 = A[g+8][4t..], a2 = A[g][16+4t..], a3 =
// A[g+8][16+4t..]; b0 = B[4t..4t+3][g], b1 = B[16+4t..][g]; d0,d1 = D[g][2t,
// 2t+1], d2,d3 = D[g+8][2t, 2t+1].
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Resident CTAs the register budget leaves room for: two for the dp4a
// variants of up to two tokens and for the 8-warp ones of up to four, so that
// the next launch's CTA can start beside this one's on an SM (and request its
// weights) while this launch finishes there; one for the MMA variants, whose
// accumulators take 32 registers per 8 tokens.
template <int W, int MT, int MMA>
constexpr int gemv_tma_min_blocks() { return MMA ? 1 : ((MT <= 2 || (W <= 8 && MT <= 4)) ? 2 : 1); }

// MMA = 0: every lane dots its row's 16-byte chunks against the activations
// with dp4a (one token).  MMA = 1: the warp multiplies the box with m16n8k32
// integer MMAs, 16 rows x 8 tokens x 32 k at a time, for 1 to 16 tokens:
//   - A is one code plane of the packed words: (word & (3 << 2j)) holds the
//     codes of k = 16 w + 4 j + b (byte b) times 4^j, as unsigned bytes; the
//     four planes accumulate apart and are scaled back (exact shifts) at the
//     flush, as in the dp4a path.
//   - The MMA's k index is any order both operands agree on: lane (g, t) of a
//     128-k chunk c takes word t of the chunk's first 16-byte unit (a0, a1) and
//     word t of its second unit (a2, a3), for rows g and g + 8; its B
//     registers are then the activation bytes 128 c + 16 t + 4 j .. + 3 and
//     that + 64, i.e. one 16-byte load gives b0 (or b1) for all four planes.
//   - Token rows sit ldx = kq + 64 bytes apart, so that the eight tokens' loads
//     of a quarter warp fall in distinct banks; the box rows' loads are
//     conflict-free under the 128-byte swizzle (distinct units per row).
// SF = 1 (one token, int8, dp4a): per-slice staging barriers (see below).
template <int XMODE, int W, int MT, int ROWS, int MMA, int SF = 0>
__global__ void __launch_bounds__(W * 32, gemv_tma_min_blocks<W, MT, MMA>())
    gemv_tma_kernel(const __grid_constant__ CUtensorMap wmap, const GemvTmaArgs a) {
    static_assert(MT == 1 || MT == 2 || MT == 4 || MT == 8 || MT == 16, "tokens per launch");
    static_assert(SF == 0 || (XMODE == 0 && MT == 1 && MMA == 0), "per-slice barriers: one int8 token, dp4a");
    static_assert(MMA || MT == 1, "several tokens take the MMA path");
    static_assert(ROWS == 32 || ROWS == 16, "rows per box");
    constexpr int kLPR = kTmaRows / ROWS;               // lanes per row (output stores; dp4a MAC)
    constexpr int kCPL = 8 / kLPR;                      // 16-byte chunks per lane per box (dp4a)
    constexpr int kBoxBytes = ROWS * kTmaSliceBytes;
    constexpr int kRG = ROWS / 16;                      // 16-row MMA groups per box
    constexpr int kNT = (MT + 7) / 8;                   // 8-token MMA tiles

    extern __shared__ uint8_t smem_raw[];
    __shared__ float red[(XMODE == 1 ? MT : 1) * 32];
    __shared__ float fsh[MT];  // BitLinear rescale factors gamma / s_t
    // the descriptor fetch is the first long latency of the launch: start it now
    if (threadIdx.x == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
    const int ns = a.ns, slices = a.slices;
    // row blocks cid, cid + ncl, ...; index arithmetic in 32 bits: the
    // divisions on the way to the first weight request stay short
    const int cid = blockIdx.x, ncl = gridDim.x;
    const int64_t kq = (int64_t)slices * kTmaSliceK;
    const int64_t ldx = gemv_tma_token_stride(slices, MT);

    // 1024-byte alignment of the ring (the 128-byte swizzle repeats every 8
    // rows of 128 bytes), computed on the shared-window address so that every
    // pointer below stays a shared-memory pointer
    uint8_t *ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    int8_t *qlin = reinterpret_cast<int8_t *>(ring + W * ns * kBoxBytes);      // [MT][ldx]
    int *accs = reinterpret_cast<int *>(qlin + MT * ldx);                      // [slot][MT][ROWS]
    int *done = accs + a.max_blocks_cta * MT * ROWS;                           // [slot] items done
    int *qslice = done + a.max_blocks_cta;                                     // [MT][slices]
    uint64_t *bars =
        reinterpret_cast<uint64_t *>(qslice + MT * slices + ((a.max_blocks_cta + MT * slices) & 1));
    // one token of int8 activations, launches with many items per CTA: every
    // 512-k slice is staged by one warp, which arrives on that slice's
    // barrier, so a warp starts on its items as soon as their slices are in
    // (no block-wide barrier after the staging; the barriers' set-up costs a
    // block barrier before the launch-chain wait, which short calls feel)
    constexpr bool kSliceFlags = SF == 1;
    uint64_t *slbar = bars + W * ns;  // [slices]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int brow = lane / kLPR, part = lane % kLPR;  // this lane's box row and chunk half
    const int mg = lane >> 2, mt4 = lane & 3;          // MMA fragment coordinates (g, t)
    // this CTA's items, in (row block, slice) order
    const int nblk = (int)a.nblocks;
    const int nb_cta = nblk > cid ? (nblk - cid + ncl - 1) / ncl : 0;
    const int items = nb_cta * slices;
    const int nslots = nb_cta;
    // this warp's items: a contiguous range of the CTA's items
    const int ipw = (items + W - 1) / W;
    const int it_begin = min(items, warp * ipw);
    const int n_items = min(items, it_begin + ipw) - it_begin;
    uint64_t *mybar = bars + warp * ns;
    uint8_t *myring = ring + warp * ns * kBoxBytes;

    // cursor over the warp's items: (slot, slice); row block = cid + slot * ncl
    int islot = it_begin / slices, ij = it_begin - islot * slices;
    const int cslot0 = islot, cj0 = ij;  // the consumer starts where the producer does
    const uint64_t wpolicy = l2_evict_first_policy();
    auto issue_next = [&](int s) {
        const int64_t row0 = (a.blk_begin + cid + (int64_t)islot * ncl) * ROWS;
        mbar_arrive_expect_tx(&mybar[s], kBoxBytes);
        if (a.evict_first)
            tma_load_box_hint(myring + s * kBoxBytes, &wmap, ij * kTmaSliceBytes, (int)row0, &mybar[s], wpolicy);
        else
            tma_load_box(myring + s * kBoxBytes, &wmap, ij * kTmaSliceBytes, (int)row0, &mybar[s]);
        if (++ij == slices) {
            ij = 0;
            ++islot;
        }
    };
    // weights do not depend on the previous kernel: request them before waiting
    // for it.  A warp's ring and barriers are its own, so lane 0 sets them up
    // and issues without waiting for the rest of the CTA.
    if (lane == 0) {
        for (int s = 0; s < ns; ++s) mbar_init(&mybar[s], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < ns && s < n_items; ++s) {
            if (s == 0 && warp == 0 && a.test_stall) {  // skip the request: nothing completes this stage
                if (++ij == slices) {
                    ij = 0;
                    ++islot;
                }
                continue;
            }
            issue_next(s);
        }
    }
    if (kSliceFlags && threadIdx.x == 1) {
        for (int j = 0; j < slices; ++j) mbar_init(&slbar[j], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = threadIdx.x; i < nslots * MT * ROWS; i += blockDim.x) accs[i] = 0;
    for (int i = threadIdx.x; i < nslots; i += blockDim.x) done[i] = 0;
    if (kSliceFlags) __syncthreads();  // slice barriers and accumulators ready, before the wait
    pdl_launch_dependents();
    pdl_wait();

    {
        float sc[MT];
        if (XMODE == 0) {
            stage_tokens_int8<MT>(qlin, ldx, qslice, slices, a.q, a.M, a.K, kq, kSliceFlags ? slbar : nullptr);
        } else {
            stage_tokens_bf16<MT, W>(qlin, ldx, qslice, slices, red, a.x, a.M, a.K, kq, sc);
        }
        if (!kSliceFlags && threadIdx.x == 0) {
#pragma unroll
            for (int t = 0; t < MT; ++t)
                fsh[t] = (t < a.M && a.y_bf16 != nullptr) ? __fdiv_rn(*a.gamma, XMODE == 1 ? sc[t] : a.s_act[t]) : 0.0f;
        }
    }
    if (!kSliceFlags) __syncthreads();

    // dp4a accumulators: one row (or half of one), per code plane
    int acc[4] = {0, 0, 0, 0}, corr = 0;
    // MMA accumulators: [token tile][row group][code plane] fragments, and the
    // activation-sum correction of this lane's two tokens per tile
    int macc[MMA ? kNT : 1][MMA ? kRG : 1][4][4];
    int mcorr[MMA ? kNT : 1][2];
    auto zero_acc = [&]() {
        acc[0] = acc[1] = acc[2] = acc[3] = corr = 0;
        if (MMA) {
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) {
                mcorr[nt][0] = mcorr[nt][1] = 0;
#pragma unroll
                for (int rg = 0; rg < kRG; ++rg)
#pragma unroll
                    for (int j = 0; j < 4; ++j) macc[nt][rg][j][0] = macc[nt][rg][j][1] = macc[nt][rg][j][2] = macc[nt][rg][j][3] = 0;
            }
        }
    };
    zero_acc();
    int ncontrib = 0;
    // folds this warp's partial sums of slot `sl` into shared memory (the
    // activation-sum correction is taken once per row and token); the warp
    // completing the slot's items writes its results
    auto flush = [&](int sl) {
        if (MMA) {
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = nt * 8 + 2 * mt4 + e;
                    if (tok < MT) {
#pragma unroll
                        for (int rg = 0; rg < kRG; ++rg)
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const int (&m)[4][4] = macc[nt][rg];
                                const int v = m[0][2 * h + e] + (m[1][2 * h + e] >> 2) + (m[2][2 * h + e] >> 4) +
                                              (m[3][2 * h + e] >> 6) - mcorr[nt][e];
                                atomicAdd(&accs[(sl * MT + tok) * ROWS + rg * 16 + h * 8 + mg], v);
                            }
                    }
                }
        } else {
            const int v = acc[0] + (acc[1] >> 2) + (acc[2] >> 4) + (acc[3] >> 6) - (part == 0 ? corr : 0);
            atomicAdd(&accs[sl * ROWS + brow], v);
        }
        __threadfence_block();
        __syncwarp();
        int fin = 0;
        if (lane == 0) fin = (atomicAdd(&done[sl], ncontrib) + ncontrib == slices);
        fin = __shfl_sync(0xffffffffu, fin, 0);
        if (fin) {
            __threadfence_block();
            const int64_t n = (a.blk_begin + cid + (int64_t)sl * ncl) * ROWS + brow;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                const int tot = atomicAdd(&accs[(sl * MT + t) * ROWS + brow], 0);
                if (part == 0 && t < a.M && n < a.N) {
                    if (a.y_bf16 != nullptr)
                        a.y_bf16[(int64_t)t * a.N + n] = float_to_bf16_bits_rn(
                            __fmul_rn((float)tot, kSliceFlags ? __fdiv_rn(*a.gamma, a.s_act[0]) : fsh[t]));
                    else
                        a.y_i32[(int64_t)t * a.N + n] = tot;
                }
            }
        }
        zero_acc();
        ncontrib = 0;
    };

    // consume cursor
    int cslot = cslot0, cj = cj0;
    int s = 0;
    uint32_t phase = 0;
    for (int n = 0; n < n_items; ++n) {
        if (kSliceFlags && !mbar_wait_bounded(&slbar[cj], 0u)) {
            if (lane == 0) record_device_error(BITNET_ERR_DEVICE_TIMEOUT);
            // wait (bounded) for this warp's boxes in flight, then stop
            for (int d = 0; d < ns && n + d < n_items; ++d)
                mbar_wait_bounded(&mybar[(n + d) % ns], (uint32_t)((n + d) / ns) & 1u);
            break;
        }
        if (!mbar_wait_bounded(&mybar[s], phase)) {
            if (lane == 0) record_device_error(BITNET_ERR_DEVICE_TIMEOUT);
            // wait (bounded) for this warp's other boxes still in flight, then stop
            for (int d = 1; d < ns && n + d < n_items; ++d)
                mbar_wait_bounded(&mybar[(n + d) % ns], (uint32_t)((n + d) / ns) & 1u);
            break;
        }
        if (MMA) {
            const uint8_t *box = myring + s * kBoxBytes + mg * kTmaSliceBytes + 4 * mt4;
            const int8_t *xs = qlin + cj * kTmaSliceK + 16 * mt4;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 128-k chunks of the slice
                uint32_t bl[kNT][4], bh[kNT][4];
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt) {
                    uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
                    const int tok = nt * 8 + mg;
                    if (tok < MT) {
                        const int8_t *xp = xs + tok * ldx + 128 * c;
                        v0 = *reinterpret_cast<const uint4 *>(xp);
                        v1 = *reinterpret_cast<const uint4 *>(xp + 64);
                    }
                    bl[nt][0] = v0.x, bl[nt][1] = v0.y, bl[nt][2] = v0.z, bl[nt][3] = v0.w;
                    bh[nt][0] = v1.x, bh[nt][1] = v1.y, bh[nt][2] = v1.z, bh[nt][3] = v1.w;
                }
                // rows mg and mg + 8 of each group share (row & 7) = mg
                const int u0 = ((2 * c) ^ mg) << 4, u1 = ((2 * c + 1) ^ mg) << 4;
#pragma unroll
                for (int rg = 0; rg < kRG; ++rg) {
                    const uint8_t *r0 = box + rg * 16 * kTmaSliceBytes, *r1 = r0 + 8 * kTmaSliceBytes;
                    const uint32_t w00 = *reinterpret_cast<const uint32_t *>(r0 + u0);
                    const uint32_t w01 = *reinterpret_cast<const uint32_t *>(r0 + u1);
                    const uint32_t w10 = *reinterpret_cast<const uint32_t *>(r1 + u0);
                    const uint32_t w11 = *reinterpret_cast<const uint32_t *>(r1 + u1);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t mk = 0x03030303u << (2 * j);
#pragma unroll
                        for (int nt = 0; nt < kNT; ++nt)
                            mma_u8s8(macc[nt][rg][j], w00 & mk, w10 & mk, w01 & mk, w11 & mk, bl[nt][j], bh[nt][j]);
                    }
                }
            }
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = nt * 8 + 2 * mt4 + e;
                    if (tok < MT) mcorr[nt][e] += qslice[tok * slices + cj];
                }
        } else {
            const uint8_t *row = myring + s * kBoxBytes + brow * kTmaSliceBytes;
            const int8_t *qk = qlin + cj * kTmaSliceK;
#pragma unroll
            for (int cc = 0; cc < kCPL; ++cc) {
                const int c = part * kCPL + cc;
                const uint4 w = *reinterpret_cast<const uint4 *>(row + ((c ^ (brow & 7)) << 4));
                const uint4 *qp = reinterpret_cast<const uint4 *>(qk + c * 64);
                const uint4 x0 = qp[0], x1 = qp[1], x2 = qp[2], x3 = qp[3];
                mac_word(acc, w.x, x0);
                mac_word(acc, w.y, x1);
                mac_word(acc, w.z, x2);
                mac_word(acc, w.w, x3);
            }
            corr += qslice[cj];
        }
        ++ncontrib;
        __syncwarp();
        if (lane == 0 && n + ns < n_items) issue_next(s);
        if (++s == ns) {
            s = 0;
            phase ^= 1u;
        }
        if (++cj == slices || n + 1 == n_items) {
            flush(cslot);
            cj = 0;
            ++cslot;
        }
    }
}

}  // namespace bitnet
