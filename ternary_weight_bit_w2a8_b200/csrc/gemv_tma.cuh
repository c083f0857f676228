// gemv_tma.cuh -- the decode GEMV (one to eight tokens): packed weights stream
// through shared memory by TMA, one row per lane.
//
// Same contraction and decode as gemv.cuh (layout v1 words, shift-free dp4a
// on codes scaled by 4^j, activation-sum correction); what differs is how the
// weights reach the lanes:
//   - The packed matrix is a 2-D byte tensor [N rows, K_pad/4 bytes].  A TMA
//     box is ROWS rows x 128 bytes (512 k): 32 rows (4 KB, one lane per row)
//     or 16 rows (2 KB, two lanes per row, each taking half of the row's 8
//     chunks), written to shared memory with the 128-byte swizzle, so a lane
//     reading 16-byte chunk c of box row r (address r*128 + ((c ^ (r & 7)) *
//     16)) is free of bank conflicts.  16-row blocks give shapes of fewer than
//     148 32-row blocks one block for every SM.
//   - Work items are (32-row block, 128-byte K-slice) pairs.  CTA b owns row
//     blocks b, b + gridDim.x, ...; its items, in (row block, slice) order, are
//     split into equal contiguous ranges, one per warp, which keeps every warp
//     busy for any K and makes a warp leave a row block at most a few times.
//   - Each warp has a private ring of NS boxes and one mbarrier per stage; its
//     lane 0 issues the TMA for the item NS ahead as soon as the warp has read
//     a stage, so up to NS boxes per warp are in flight without holding
//     registers.
//   - Activations live in shared memory as one linear array per token; all
//     lanes read the same 16 bytes at a time (a broadcast).  With several
//     tokens (MT = 2, 4, 8) every weight box is still read from HBM once: the
//     four code masks of each word are computed once and reused per token.
//   - A warp adds its per-row partial sums into a per-row-block int32
//     accumulator in shared memory (atomics: exact and order-free) whenever its
//     item sequence leaves a row block; the warp whose contribution completes
//     the block's item count writes the 32 results.
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
};

// Dynamic shared memory of a launch: ring of warps x stages boxes of `rows`
// rows, linear activations, per-row-block accumulators and counters, slice
// sums, mbarriers.
__host__ __device__ inline size_t gemv_tma_smem_bytes(int warps, int stages, int slices, int max_blocks_cta,
                                                      int tokens = 1, int rows = kTmaRows) {
    return 1024 /* alignment slack */ + (size_t)warps * stages * rows * kTmaSliceBytes +
           (size_t)tokens * slices * kTmaSliceK + (size_t)max_blocks_cta * tokens * rows * 4 +
           (size_t)max_blocks_cta * 4 + 8 + (size_t)warps * stages * 8 + (size_t)tokens * slices * 4;
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

// Linear staging of int8 activations: qlin[k] = q[k] for k < K, 0 up to kq
// (kq a multiple of 512), with the sum of every 512-k slice in qslice.
__device__ __forceinline__ void stage_qlin_int8(int8_t *qlin, int *qslice, const int8_t *qrow, int64_t K,
                                                int64_t kq) {
    const bool vec = ((reinterpret_cast<uintptr_t>(qrow) & 15) == 0);
    for (int64_t p = threadIdx.x; p < kq / 16; p += blockDim.x) {
        const int64_t k0 = p * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (vec && k0 + 16 <= K) {
            v = *reinterpret_cast<const uint4 *>(qrow + k0);
        } else if (k0 < K) {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            for (int t = 0; t < 16 && k0 + t < K; ++t) w[t >> 2] |= (uint32_t)(uint8_t)qrow[k0 + t] << (8 * (t & 3));
            v = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *reinterpret_cast<uint4 *>(qlin + k0) = v;
        slice_sum(qslice, p, v);
    }
}

// Linear staging with fused per-token quantisation of bf16 activations (same
// arithmetic as quant_act_kernel<>), slice sums as above.  Returns the scale.
__device__ __forceinline__ float stage_qlin_bf16(int8_t *qlin, int *qslice, float *red, const uint16_t *xrow,
                                                 int64_t K, int64_t kq) {
    const bool vec = ((reinterpret_cast<uintptr_t>(xrow) & 15) == 0);
    const int64_t npieces = ceil_div(K, 16);
    float amax = 0.0f;
    for (int64_t p = threadIdx.x; p < npieces; p += blockDim.x) {
        uint4 lo, hi;
        load_x16(xrow, K, p, vec, lo, hi);
        amax = amax16(lo, hi, amax);
    }
    amax = block_reduce(amax, [](float u, float v) { return fmaxf(u, v); }, red);
    const float sc = __fdiv_rn(127.0f, amax > kQuantEps ? amax : kQuantEps);
    for (int64_t p = threadIdx.x; p < kq / 16; p += blockDim.x) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (p < npieces) {
            uint4 lo, hi;
            load_x16(xrow, K, p, vec, lo, hi);
            quant16(lo, hi, sc, v);
        }
        *reinterpret_cast<uint4 *>(qlin + p * 16) = v;
        slice_sum(qslice, p, v);
    }
    return sc;
}

// Linear staging with fused quantisation of MT tokens at once (same
// arithmetic as quant_act_kernel<>): one pass over every token's row for the
// absmax values, one block reduction for all of them, then every token is
// quantised, with slice sums as above.  Token slots t >= M are staged as
// zeros.  `red` holds MT x 32 floats.
template <int MT>
__device__ __forceinline__ void stage_qlin_bf16_tokens(int8_t *qlin, int *qslice, int slices, float *red,
                                                       const uint16_t *x, int M, int64_t K, int64_t kq,
                                                       float (&sc)[MT]) {
    const int64_t npieces = ceil_div(K, 16);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    float am[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) am[t] = 0.0f;
    for (int64_t p = threadIdx.x; p < npieces; p += blockDim.x) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            if (t < M) {
                const uint16_t *xr = x + (int64_t)t * K;
                uint4 lo, hi;
                load_x16(xr, K, p, (reinterpret_cast<uintptr_t>(xr) & 15) == 0, lo, hi);
                am[t] = amax16(lo, hi, am[t]);
            }
        }
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
        for (int w = 0; w < nwarps; ++w) v = fmaxf(v, red[t * 32 + w]);
        sc[t] = t < M ? __fdiv_rn(127.0f, v > kQuantEps ? v : kQuantEps) : 0.0f;
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        const uint16_t *xr = x + (int64_t)t * K;
        const bool vec = (reinterpret_cast<uintptr_t>(xr) & 15) == 0;
        for (int64_t p = threadIdx.x; p < kq / 16; p += blockDim.x) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < M && p < npieces) {
                uint4 lo, hi;
                load_x16(xr, K, p, vec, lo, hi);
                quant16(lo, hi, sc[t], v);
            }
            *reinterpret_cast<uint4 *>(qlin + t * kq + p * 16) = v;
            slice_sum(qslice + t * slices, p, v);
        }
    }
}

// ------------------------------------------------------------------ kernel

// Resident CTAs the register budget leaves room for: two for every variant of
// up to two tokens and for the 8-warp ones of up to four, so that the next
// launch's CTA can start beside this one's on an SM (and request its weights)
// while this launch finishes there.
template <int W, int MT>
constexpr int gemv_tma_min_blocks() { return (MT <= 2 || (W <= 8 && MT <= 4)) ? 2 : 1; }

template <int XMODE, int W, int MT, int ROWS>
__global__ void __launch_bounds__(W * 32, gemv_tma_min_blocks<W, MT>())
    gemv_tma_kernel(const __grid_constant__ CUtensorMap wmap, const GemvTmaArgs a) {
    static_assert(MT == 1 || MT == 2 || MT == 4 || MT == 8, "tokens per launch");
    static_assert(ROWS == 32 || ROWS == 16, "rows per box");
    constexpr int kLPR = kTmaRows / ROWS;               // lanes per row
    constexpr int kCPL = 8 / kLPR;                      // 16-byte chunks per lane per box
    constexpr int kBoxBytes = ROWS * kTmaSliceBytes;

    extern __shared__ uint8_t smem_raw[];
    __shared__ float red[(XMODE == 1 ? MT : 1) * 32];
    // the descriptor fetch is the first long latency of the launch: start it now
    if (threadIdx.x == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
    const int ns = a.ns, slices = a.slices;
    const int64_t cid = blockIdx.x, ncl = gridDim.x;  // row blocks cid, cid + ncl, ...
    const int64_t kq = (int64_t)slices * kTmaSliceK;

    // 1024-byte alignment of the ring (the 128-byte swizzle repeats every 8
    // rows of 128 bytes), computed on the shared-window address so that every
    // pointer below stays a shared-memory pointer
    uint8_t *ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    int8_t *qlin = reinterpret_cast<int8_t *>(ring + W * ns * kBoxBytes);      // [MT][kq]
    int *accs = reinterpret_cast<int *>(qlin + MT * kq);                       // [slot][MT][ROWS]
    int *done = accs + a.max_blocks_cta * MT * ROWS;                           // [slot] items done
    int *qslice = done + a.max_blocks_cta;                                     // [MT][slices]
    uint64_t *bars =
        reinterpret_cast<uint64_t *>(qslice + MT * slices + ((a.max_blocks_cta + MT * slices) & 1));

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int brow = lane / kLPR, part = lane % kLPR;  // this lane's box row and chunk half
    // this CTA's items, in (row block, slice) order
    const int64_t nb_cta = a.nblocks > cid ? ceil_div(a.nblocks - cid, ncl) : 0;
    const int64_t items = nb_cta * slices;
    const int nslots = (int)nb_cta;
    // this warp's items: a contiguous range of the CTA's items
    const int64_t ipw = ceil_div(items, W);
    const int64_t it_begin = min(items, warp * ipw);
    const int n_items = (int)(min(items, it_begin + ipw) - it_begin);
    uint64_t *mybar = bars + warp * ns;
    uint8_t *myring = ring + warp * ns * kBoxBytes;

    // cursor over the warp's items: (slot, slice); row block = cid + slot * ncl
    int islot = (int)(it_begin / slices), ij = (int)(it_begin - (int64_t)islot * slices);
    auto issue_next = [&](int s) {
        const int64_t row0 = (a.blk_begin + cid + (int64_t)islot * ncl) * ROWS;
        mbar_arrive_expect_tx(&mybar[s], kBoxBytes);
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
    for (int i = threadIdx.x; i < nslots * MT * ROWS; i += blockDim.x) accs[i] = 0;
    for (int i = threadIdx.x; i < nslots; i += blockDim.x) done[i] = 0;
    pdl_launch_dependents();
    pdl_wait();

    float sc[MT];
    if (XMODE == 1 && MT > 1) stage_qlin_bf16_tokens<MT>(qlin, qslice, slices, red, a.x, a.M, a.K, kq, sc);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        if (XMODE == 1 && MT > 1) break;  // staged above
        sc[t] = 0.0f;
        int8_t *qt = qlin + t * kq;
        int *qst = qslice + t * slices;
        if (t < a.M) {
            if (XMODE == 0)
                stage_qlin_int8(qt, qst, a.q + (int64_t)t * a.K, a.K, kq);
            else
                sc[t] = stage_qlin_bf16(qt, qst, red, a.x + (int64_t)t * a.K, a.K, kq);
        } else {  // unused token slot: zeros, contributes nothing and is not stored
            for (int64_t p = threadIdx.x; p < kq / 16; p += blockDim.x)
                reinterpret_cast<uint4 *>(qt)[p] = make_uint4(0u, 0u, 0u, 0u);
            for (int j = threadIdx.x; j < slices; j += blockDim.x) qst[j] = 0;
        }
    }
    __syncthreads();
    float f[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        f[t] = 0.0f;
        if (t < a.M && a.y_bf16 != nullptr) f[t] = __fdiv_rn(*a.gamma, XMODE == 1 ? sc[t] : a.s_act[t]);
    }

    int acc[MT][4], corr[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = corr[t] = 0;
    int ncontrib = 0;
    // folds this warp's partial sums of slot `sl` into shared memory (the
    // lanes sharing a row each add their half; the activation-sum correction
    // is taken once per row); the warp completing the slot's items writes its
    // results
    auto flush = [&](int sl) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            const int v = acc[t][0] + (acc[t][1] >> 2) + (acc[t][2] >> 4) + (acc[t][3] >> 6) - (part == 0 ? corr[t] : 0);
            atomicAdd(&accs[(sl * MT + t) * ROWS + brow], v);
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
                        a.y_bf16[(int64_t)t * a.N + n] = float_to_bf16_bits_rn(__fmul_rn((float)tot, f[t]));
                    else
                        a.y_i32[(int64_t)t * a.N + n] = tot;
                }
            }
        }
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = corr[t] = 0;
        ncontrib = 0;
    };

    // consume cursor
    int cslot = (int)(it_begin / slices), cj = (int)(it_begin - (int64_t)cslot * slices);
    int s = 0;
    uint32_t phase = 0;
    for (int n = 0; n < n_items; ++n) {
        if (!mbar_wait_bounded(&mybar[s], phase)) {
            if (lane == 0) record_device_error(BITNET_ERR_DEVICE_TIMEOUT);
            // wait (bounded) for this warp's other boxes still in flight, then stop
            for (int d = 1; d < ns && n + d < n_items; ++d)
                mbar_wait_bounded(&mybar[(n + d) % ns], (uint32_t)((n + d) / ns) & 1u);
            break;
        }
        const uint8_t *row = myring + s * kBoxBytes + brow * kTmaSliceBytes;
        const int8_t *qk = qlin + cj * kTmaSliceK;
#pragma unroll
        for (int cc = 0; cc < kCPL; ++cc) {
            const int c = part * kCPL + cc;
            const uint4 w = *reinterpret_cast<const uint4 *>(row + ((c ^ (brow & 7)) << 4));
            if (MT == 1) {
                const uint4 *qp = reinterpret_cast<const uint4 *>(qk + c * 64);
                const uint4 x0 = qp[0], x1 = qp[1], x2 = qp[2], x3 = qp[3];
                mac_word(acc[0], w.x, x0);
                mac_word(acc[0], w.y, x1);
                mac_word(acc[0], w.z, x2);
                mac_word(acc[0], w.w, x3);
            } else {
                // the four scaled code masks of each word, shared by all tokens
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                uint32_t mk[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    mk[i][0] = ww[i] & 0x03030303u;
                    mk[i][1] = ww[i] & 0x0C0C0C0Cu;
                    mk[i][2] = ww[i] & 0x30303030u;
                    mk[i][3] = ww[i] & 0xC0C0C0C0u;
                }
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    const uint4 *qp = reinterpret_cast<const uint4 *>(qk + t * kq + c * 64);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 x = qp[i];
                        acc[t][0] = dp4a_us(mk[i][0], x.x, acc[t][0]);
                        acc[t][1] = dp4a_us(mk[i][1], x.y, acc[t][1]);
                        acc[t][2] = dp4a_us(mk[i][2], x.z, acc[t][2]);
                        acc[t][3] = dp4a_us(mk[i][3], x.w, acc[t][3]);
                    }
                }
            }
        }
        ++ncontrib;
#pragma unroll
        for (int t = 0; t < MT; ++t) corr[t] += qslice[t * slices + cj];
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
