// bitnet_b200.cu -- the C ABI of libbitnet_b200.so (declared in
// include/bitnet_b200.h): argument checks, plan selection and launches.
// All kernels are in the headers included below; this is the library's single
// translation unit, so file-scope device state (the error word) is shared.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemv.cuh"
#include "gemv_tma.cuh"
#include "gemm_tc.cuh"
#include "quant.cuh"
#include "weights.cuh"

namespace bitnet {
namespace {

std::atomic<int64_t> g_launches{0};

constexpr int kMaxDevices = 64;
constexpr int kMaxSliceChunks = 1536;  // activations of one K-slice: 96 KB of shared memory
constexpr int kPlanSlots = 148 * 16;   // warp slots the K-split aims to fill (fixed: it sizes the workspace)
constexpr int kOccCache = 128;

struct OccEntry {
    int idx;
    size_t smem;
    int ctas;
};

struct DeviceInfo {
    bool init = false;
    int status = BITNET_OK;
    int sm_count = 0;
    uint64_t smem_attr_set = 0;  // GEMV instantiations whose shared-memory limit is raised
    size_t tma_max_dyn[400] = {};  // dynamic shared memory opted into by each TMA GEMV variant
    bool tc_attr_set[2 * 10] = {};    // shared-memory opt-in done, per tensor-core GEMM variant
    size_t smem_optin = 0;       // largest dynamic shared memory a CTA may opt into
    int n_occ = 0;
    OccEntry occ[kOccCache];     // resident CTAs per SM by (instantiation, shared memory)
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BITNET_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BITNET_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.init) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BITNET_ERR_CUDA;
        int optin = 0;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return BITNET_ERR_CUDA;
        d.status = (major == 10) ? BITNET_OK : BITNET_ERR_UNSUPPORTED;
        d.sm_count = sms;
        d.smem_optin = (size_t)optin;
        d.init = true;
    }
    *out = &d;
    return d.status;
}

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline int launched(cudaError_t e = cudaSuccess) {
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return BITNET_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return BITNET_OK;
}

inline bool sizes_ok(int64_t M, int64_t N, int64_t K) {
    return M >= 0 && N >= 0 && K >= 0 && K <= BITNET_MAX_K && M <= (1LL << 31) - 1 && N <= (1LL << 40) &&
           M * N <= (1LL << 46);
}

inline int grid_for(int64_t work, int64_t per_cta, int sm_count, int per_sm = 8) {
    int64_t g = ceil_div(work, per_cta);
    int64_t cap = (int64_t)sm_count * per_sm;
    if (g > cap) g = cap;
    return (int)(g < 1 ? 1 : g);
}

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ------------------------------------------------------------------ fill (K == 0)
template <typename T>
__global__ void __launch_bounds__(kThreads) fill_kernel(T *p, int64_t n, T v) {
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kThreads) p[i] = v;
}

// ------------------------------------------------------------------ GEMV plan
// The K-split depends on the shape only (it sizes the workspace); rows per
// lane group and the grid also depend on the device.
struct GemvSplit {
    int S, cps;
    int64_t ws_bytes;
};

// optional override:
// BITNET_GEMV_TUNE="G,R,U,ctas_per_sm,prefetch_tasks,S,tma,ns,fuse,qwpt,rows,cores,mma,l2,sflags"
// (register GEMV: G, R, U, ctas, prefetch, S; TMA GEMV: tma = 0 off or
// 1..5 a variant of kTmaCfg, ctas per SM, ns ring depth, rows per block 16 or
// 32, cores = 1 the co-residency mode (see tma_plan), mma = 1 / 0 the MMA or
// dp4a product for one token, l2 = 0 weights read without the L2
// evict-first policy, sflags = 1 / 0 per-slice staging barriers always /
// never; tensor-core GEMM: R < 0
// variant, S K-splits, fuse = 1 quantises BitLinear activations inside the
// GEMM launch; activation quantisation: qwpt warps per token, 1..8)
struct GemvTune {
    int G = 0, R = 0, U = 0, ctas = 0, prefetch = -1, S = 0, tma = -1, ns = 0, fuse = -1, qwpt = 0, rows = 0,
        cores = -1, mma = -1, l2 = -1, sflags = -1;
};

const GemvTune &gemv_tune() {
    static GemvTune t;
    static std::once_flag once;
    std::call_once(once, [] {
        const char *e = getenv("BITNET_GEMV_TUNE");
        if (e != nullptr)
            sscanf(e, "%d,%d,%d,%d,%d,%d,%d,%d,%d,%d,%d,%d,%d,%d,%d", &t.G, &t.R, &t.U, &t.ctas, &t.prefetch, &t.S,
                   &t.tma, &t.ns, &t.fuse, &t.qwpt, &t.rows, &t.cores, &t.mma, &t.l2, &t.sflags);
    });
    return t;
}

// ------------------------------------------------------------------ activation quantisation
// Teams of 1..8 warps per token: about a thousand warps in flight whatever M
// (one warp per token from 1024 tokens up), so the pass is one wave that reads
// each row from HBM once, and wide enough teams that a thread holds all of
// its words of the row (one load round trip).
int launch_quant(DeviceInfo *dev, const uint16_t *x, int64_t M, int64_t K, int8_t *q, int64_t ldq, bool zero_pad,
                 float *s, int32_t *rowsum, cudaStream_t st) {
    int wpt = M >= 1024 ? 1 : (M >= 512 ? 2 : (M >= 256 ? 4 : 8));
    while (wpt < 8 && ceil_div(K, 8) > (int64_t)kQuantHeld * 32 * wpt) wpt *= 2;
    const int tw = gemv_tune().qwpt;
    if (tw == 1 || tw == 2 || tw == 4 || tw == 8) wpt = tw;
    // teams per CTA: up to kThreads / (32 wpt), fewer when that spreads one
    // wave of tokens over every SM (1024 tokens: 147 CTAs of 7 one-warp teams
    // rather than 128 of 8)
    int64_t teams_per_cta = kThreads / (32 * wpt);
    if (M <= (int64_t)dev->sm_count * teams_per_cta) {
        const int64_t t = ceil_div(M, (int64_t)dev->sm_count);
        if (t >= 1 && t < teams_per_cta) teams_per_cta = t;
    }
    int64_t grid = ceil_div(M, teams_per_cta);
    const int64_t cap = (int64_t)dev->sm_count * (2048 / kThreads);
    if (grid > cap) grid = cap;
    const dim3 g((unsigned)grid), b((unsigned)(teams_per_cta * 32 * wpt));
    cudaError_t e;
    switch (wpt) {
        case 1: e = launch_pdl(quant_act_kernel<1>, g, b, 0, st, x, M, K, q, ldq, zero_pad, s, rowsum); break;
        case 2: e = launch_pdl(quant_act_kernel<2>, g, b, 0, st, x, M, K, q, ldq, zero_pad, s, rowsum); break;
        case 4: e = launch_pdl(quant_act_kernel<4>, g, b, 0, st, x, M, K, q, ldq, zero_pad, s, rowsum); break;
        default: e = launch_pdl(quant_act_kernel<8>, g, b, 0, st, x, M, K, q, ldq, zero_pad, s, rowsum); break;
    }
    return launched(e);
}

inline int lanes_per_row(int nch) { return nch >= 128 ? 32 : (nch >= 48 ? 16 : 8); }

GemvSplit plan_split(int64_t M, int64_t N, int64_t K) {
    GemvSplit p{};
    const int nch = (int)(k_pad(K) / 64);
    const int G = lanes_per_row(nch);
    const int64_t tasks = ceil_div(N, 32 / G) * M;  // warp tasks at one row per lane group
    int S = (int)ceil_div(nch, kMaxSliceChunks);
    // split K only when rows are too few to fill the GPU and every lane still
    // keeps >= 4 chunks per slice (small problems are latency-bound: a second
    // launch would cost more than it saves)
    while (tasks * S < kPlanSlots / 4 && nch / (2 * S) >= 4 * G) S *= 2;
    if (gemv_tune().S > 0) S = gemv_tune().S;
    p.cps = (int)ceil_div(nch, S);
    p.S = (int)ceil_div(nch, p.cps);
    p.ws_bytes = p.S > 1 ? (int64_t)p.S * M * N * 4 + round_up(M * 4, 256) : 0;
    return p;
}

using GemvKernel = void (*)(const GemvArgs);

// (R, U) pairs: rows per lane group x chunks per load batch
constexpr int kRU[6][2] = {{1, 4}, {1, 8}, {2, 2}, {2, 4}, {4, 1}, {4, 2}};

#define BITNET_GEMV_ROW(X, G)                                                                           \
    gemv_w2a8_kernel<G, 1, 4, X>, gemv_w2a8_kernel<G, 1, 8, X>, gemv_w2a8_kernel<G, 2, 2, X>,          \
        gemv_w2a8_kernel<G, 2, 4, X>, gemv_w2a8_kernel<G, 4, 1, X>, gemv_w2a8_kernel<G, 4, 2, X>

GemvKernel gemv_kernel_for(int G, int ru, int xmode, int *index) {
    static const GemvKernel table[36] = {
        BITNET_GEMV_ROW(0, 8), BITNET_GEMV_ROW(0, 16), BITNET_GEMV_ROW(0, 32),
        BITNET_GEMV_ROW(1, 8), BITNET_GEMV_ROW(1, 16), BITNET_GEMV_ROW(1, 32),
    };
    const int gi = G == 8 ? 0 : (G == 16 ? 1 : 2);
    *index = xmode * 18 + gi * 6 + ru;
    return table[*index];
}
#undef BITNET_GEMV_ROW

// Resident CTAs per SM of a GEMV instantiation at a given shared-memory size.
int gemv_ctas_per_sm(DeviceInfo *dev, int idx, GemvKernel kern, size_t smem) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    for (int i = 0; i < dev->n_occ; ++i)
        if (dev->occ[i].idx == idx && dev->occ[i].smem == smem) return dev->occ[i].ctas;
    if (smem > 48 * 1024 && !(dev->smem_attr_set & (1ull << idx))) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSliceChunks * 64) !=
            cudaSuccess)
            return -1;
        dev->smem_attr_set |= 1ull << idx;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, smem) != cudaSuccess) return -1;
    if (dev->n_occ < kOccCache) dev->occ[dev->n_occ++] = {idx, smem, n};
    return n;
}

// ------------------------------------------------------------------ TMA GEMV
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}


// 2-D tensor maps (inner dimension d0 contiguous, rows of `stride` bytes),
// encoded once per distinct argument set and kept in a small cache: a map is
// a pure function of its arguments, so a cached one stays valid for any
// allocation that reuses the address.  Returns false if encoding fails.
struct MapKey {
    const void *ptr;
    uint64_t d0, d1, stride;
    uint32_t b0, b1;
    int dtype, swizzle, promo;
    bool operator==(const MapKey &o) const {
        return ptr == o.ptr && d0 == o.d0 && d1 == o.d1 && stride == o.stride && b0 == o.b0 && b1 == o.b1 &&
               dtype == o.dtype && swizzle == o.swizzle && promo == o.promo;
    }
};
constexpr int kMapCache = 64;
struct MapCache {
    MapKey key[kMapCache];
    CUtensorMap map[kMapCache];
    int n = 0, next = 0;
};
MapCache g_maps[kMaxDevices];
std::mutex g_maps_mu;

bool encode_2d(CUtensorMap *out, CUtensorMapDataType dtype, const void *ptr, uint64_t d0, uint64_t d1,
               uint64_t stride, uint32_t b0, uint32_t b1, CUtensorMapSwizzle swizzle,
               CUtensorMapL2promotion promo) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    const MapKey k{ptr, d0, d1, stride, b0, b1, (int)dtype, (int)swizzle, (int)promo};
    {
        std::lock_guard<std::mutex> lk(g_maps_mu);
        MapCache &c = g_maps[dev];
        for (int i = 0; i < c.n; ++i)
            if (c.key[i] == k) {
                *out = c.map[i];
                return true;
            }
    }
    if (tensor_map_encoder() == nullptr) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)d0, (cuuint64_t)d1};
    const cuuint64_t gstride[1] = {(cuuint64_t)stride};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t es[2] = {1, 1};
    if (tensor_map_encoder()(out, dtype, 2, const_cast<void *>(ptr), gdim, gstride, box, es,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lk(g_maps_mu);
    MapCache &c = g_maps[dev];
    const int slot = c.n < kMapCache ? c.n++ : c.next;
    if (slot == c.next) c.next = (c.next + 1) % kMapCache;
    c.key[slot] = k;
    c.map[slot] = *out;
    return true;
}

// TMA GEMV variants: (warps per CTA, most boxes in flight per warp); the
// ring depth of a launch is the smaller of the latter and what its items need
constexpr int kTmaNumCfg = 5;
constexpr int kTmaCfg[kTmaNumCfg][2] = {{8, 4}, {12, 3}, {16, 2}, {8, 2}, {4, 4}};
using TmaKernel = void (*)(const CUtensorMap, const GemvTmaArgs);

// Tokens per TMA GEMV launch: up to this many tokens read the weights once in
// one GEMV launch (on the MMA path from 2 tokens up); more go to the
// tensor-core GEMM.
constexpr int kGemvMaxTokens = 16;

// BitLinear with up to this many tokens quantises them inside the GEMV's
// prologue (every CTA reads and quantises all of them); more tokens are
// quantised once by quant_act_kernel first.  The tuning field `fuse` moves
// the boundary: 1 quantises every token count inside the launch, 0 every
// count above one in a pass of its own.
constexpr int kFusedQuantMaxTokens = 4;

int fused_quant_max_tokens() {
    const int f = gemv_tune().fuse;
    return f == 1 ? kGemvMaxTokens : (f == 0 ? 1 : kFusedQuantMaxTokens);
}

// Kernel of (mode, warps, tokens per launch, rows per block, MMA): one token
// on 4, 8, 12 or 16 warps with dp4a or the MMA path, several tokens (MT = 2,
// 4, 8, 16) on 8 or 16 warps with the MMA path, for int8 activations (xmode 0)
// or bf16 activations quantised in the kernel (xmode 1); row blocks of 32 or
// 16 rows.  Slot in the shared-memory
// opt-in table, -1 if no such kernel.
constexpr int kTmaNumSlots = 2 * 2 * 2 * 2 * kTmaNumCfg * 5;
static_assert(kTmaNumSlots <= (int)(sizeof(DeviceInfo::tma_max_dyn) / sizeof(size_t)), "opt-in table");

int tma_kernel_slot(int xmode, int cfg, int mt, int rows, int mma, int sf) {
    const int W = kTmaCfg[cfg][0];
    const int mti = mt == 1 ? 0 : (mt == 2 ? 1 : (mt == 4 ? 2 : (mt == 8 ? 3 : (mt == 16 ? 4 : -1))));
    if (mti < 0 || (mt > 1 && (!mma || (W != 8 && W != 16)))) return -1;
    if (sf && (xmode != 0 || mt != 1 || mma)) return -1;
    return ((((sf ? 1 : 0) * 2 + xmode) * 2 + (rows == 16 ? 1 : 0)) * 2 + (mma ? 1 : 0)) * kTmaNumCfg * 5 + cfg * 5 + mti;
}

template <int X, int R, int MM>
TmaKernel tma_kernel_w(int W, int mt) {
    if (mt == 1) {
        switch (W) {
            case 4: return gemv_tma_kernel<X, 4, 1, R, MM>;
            case 8: return gemv_tma_kernel<X, 8, 1, R, MM>;
            case 12: return gemv_tma_kernel<X, 12, 1, R, MM>;
            default: return gemv_tma_kernel<X, 16, 1, R, MM>;
        }
    }
    if constexpr (MM == 1) {
        const bool w16 = W == 16;
        switch (mt) {
            case 2: return w16 ? gemv_tma_kernel<X, 16, 2, R, 1> : gemv_tma_kernel<X, 8, 2, R, 1>;
            case 4: return w16 ? gemv_tma_kernel<X, 16, 4, R, 1> : gemv_tma_kernel<X, 8, 4, R, 1>;
            case 8: return w16 ? gemv_tma_kernel<X, 16, 8, R, 1> : gemv_tma_kernel<X, 8, 8, R, 1>;
            case 16: return w16 ? gemv_tma_kernel<X, 16, 16, R, 1> : gemv_tma_kernel<X, 8, 16, R, 1>;
            default: break;
        }
    }
    return nullptr;
}

template <int X, int R>
TmaKernel tma_kernel_m(int W, int mt, int mma) {
    return mma ? tma_kernel_w<X, R, 1>(W, mt) : tma_kernel_w<X, R, 0>(W, mt);
}

// one int8 token with per-slice staging barriers
template <int R>
TmaKernel tma_kernel_sf(int W) {
    switch (W) {
        case 4: return gemv_tma_kernel<0, 4, 1, R, 0, 1>;
        case 8: return gemv_tma_kernel<0, 8, 1, R, 0, 1>;
        case 12: return gemv_tma_kernel<0, 12, 1, R, 0, 1>;
        default: return gemv_tma_kernel<0, 16, 1, R, 0, 1>;
    }
}

TmaKernel tma_kernel_for(int xmode, int cfg, int mt, int rows, int mma, int sf) {
    if (tma_kernel_slot(xmode, cfg, mt, rows, mma, sf) < 0) return nullptr;
    const int W = kTmaCfg[cfg][0];
    if (sf) return rows == 16 ? tma_kernel_sf<16>(W) : tma_kernel_sf<32>(W);
    if (xmode == 0) return rows == 16 ? tma_kernel_m<0, 16>(W, mt, mma) : tma_kernel_m<0, 32>(W, mt, mma);
    return rows == 16 ? tma_kernel_m<1, 16>(W, mt, mma) : tma_kernel_m<1, 32>(W, mt, mma);
}

// Opts a TMA GEMV variant into the largest dynamic shared memory left beside
// its static shared memory; returns that size (0 on failure).
size_t tma_max_dynamic_smem(DeviceInfo *dev, int xmode, int cfg, int mt, int rows, int mma, int sf) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    const int si = tma_kernel_slot(xmode, cfg, mt, rows, mma, sf);
    if (si < 0) return 0;
    size_t &slot = dev->tma_max_dyn[si];
    if (slot == 0) {
        TmaKernel kern = tma_kernel_for(xmode, cfg, mt, rows, mma, sf);
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.sharedSizeBytes >= dev->smem_optin) return 0;
        const size_t dyn = dev->smem_optin - fa.sharedSizeBytes;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess) return 0;
        slot = dyn;
    }
    return slot;
}

// Plan of the TMA GEMV, from the shape and B200 reference figures only (148
// SMs, 228 KB of shared memory per SM), so that what a shape needs does not
// depend on the device that runs it.
//   - Row blocks of 32 rows (16 for long rows where that evens out the
//     busiest CTA, see below); CTA c takes row blocks c, c + grid, ..., with
//     at most 148 CTAs.
//   - Variant (measured on B200): 16 warps x up to 2 boxes in flight, 12 x 3
//     for rows of >= 32 K-slices; 8 or 16 warps for several tokens (the MMA
//     product, up to 16 tokens).  The ring is no deeper than the warp's items
//     need.
//   - One CTA per SM per launch, for every launch: its shared memory is padded
//     past half an SM.  Programmatic dependent launch could otherwise start
//     the next call's CTAs beside this call's, to request their weights early;
//     that pays for a shape repeated alone when every SM holds one CTA of each
//     launch (4736 x 2560: 2.44 -> 1.99 us per call; with 16-row blocks so
//     that small shapes reach 148 CTAs too, 2560 x 2560: 2.13 -> 2.01 us), but
//     in the benchmark's sequence of eight different shapes the calls then
//     slow each other down (25.4 -> 30.5 us per step).  The tuning field
//     `cores` = 1 selects that mode (16-row blocks where 32-row ones leave SMs
//     idle, shallower rings for short calls so that two CTAs fit an SM).
struct TmaPlan {
    bool use;
    int cfg, slices, max_blocks, grid;
    int ns;            // ring depth per warp
    int mt;            // tokens per launch (1, 2, 4, 8, 16)
    int rows;          // rows per block (32 or 16)
    int mma;           // 1: the MMA product, 0: dp4a (one token only)
    int64_t nblocks;
    size_t smem;
    int64_t ws_bytes;  // always 0: the TMA GEMV needs no workspace
};

TmaPlan tma_plan(int64_t M, int64_t N, int64_t K) {
    constexpr int kRefSMs = 148;
    constexpr size_t kRefSmemOptin = 232448;  // one CTA per SM
    constexpr size_t kRefSmemHalf = 113664;   // two CTAs per SM (1 KB reserved and 1 KB static memory each)
    const GemvTune &tn = gemv_tune();
    TmaPlan p{};
    const int tune = tn.tma;
    if (M < 1 || M > kGemvMaxTokens || tune == 0 || K < kTmaSliceK || N < 1) return p;
    // a lane accumulates one row's whole K: |acc_j| <= 4096 * K_pad stays
    // inside int32 for K_pad <= 2^19 (shared memory caps K lower still)
    if (k_pad(K) > ((int64_t)1 << 19)) return p;
    p.mt = M == 1 ? 1 : (M == 2 ? 2 : (M <= 4 ? 4 : (M <= 8 ? 8 : 16)));
    p.mma = p.mt > 1 ? 1 : (tn.mma == 1 ? 1 : 0);
    const int64_t row_bytes = packed_row_bytes(K);
    // co-residency mode (tuning field `cores` = 1, see above); eight tokens
    // keep 32-row blocks: their 16-warp variant has no registers to spare for
    // the second lane of a row
    const bool cores = tn.cores == 1;
    p.rows = (!cores || ceil_div(N, kTmaRows) >= kRefSMs || p.mt >= 8) ? 32 : 16;
    p.slices = (int)ceil_div(row_bytes, kTmaSliceBytes);
    // long rows (>= 32 slices) with a leftover of 32-row blocks: 16-row blocks
    // where they cut the busiest CTA's rows by a fifth (5120 x 27648: 64 -> 48
    // rows, 11.2 -> 10.7 us on B200; shorter rows measured slower with them)
    if (!cores && p.mt == 1 && p.slices >= 32) {
        const int64_t r32 = ceil_div(ceil_div(N, 32), (int64_t)kRefSMs) * 32;
        const int64_t r16 = ceil_div(ceil_div(N, 16), (int64_t)kRefSMs) * 16;
        if (r16 * 5 <= r32 * 4) p.rows = 16;
    }
    if (tn.rows == 16 || tn.rows == 32) p.rows = tn.rows;
    p.nblocks = ceil_div(N, p.rows);
    if (tune >= 1 && tune <= kTmaNumCfg)
        p.cfg = tune - 1;
    else
        p.cfg = p.slices >= 32 ? 1 : 2;
    if (p.mt > 1 && kTmaCfg[p.cfg][0] != 8 && kTmaCfg[p.cfg][0] != 16) p.cfg = 2;  // several tokens: 8 or 16 warps
    const int W = kTmaCfg[p.cfg][0], NS = kTmaCfg[p.cfg][1];
    // BITNET_GEMV_TUNE's ctas field: CTAs per SM per launch (1 by default)
    const int per_sm = tn.ctas > 0 ? tn.ctas : 1;
    const int64_t gmax = (int64_t)kRefSMs * per_sm;
    p.grid = (int)(p.nblocks < gmax ? p.nblocks : gmax);
    p.max_blocks = (int)ceil_div(p.nblocks, p.grid);
    const int64_t ipw = ceil_div((int64_t)p.max_blocks * p.slices, W);
    p.ns = (int)(ipw < NS ? (ipw < 1 ? 1 : ipw) : NS);
    if (tn.ns > 0) p.ns = tn.ns < NS ? tn.ns : NS;
    auto bytes = [&](int ns) { return gemv_tma_smem_bytes(W, ns, p.slices, p.max_blocks, p.mt, p.rows); };
    if (cores && p.grid >= kRefSMs && ipw <= 4)
        while (p.ns > 1 && bytes(p.ns) > kRefSmemHalf) --p.ns;
    p.smem = bytes(p.ns);
    if (p.smem > kRefSmemOptin - 1024) return TmaPlan{};
    // one CTA per SM: always, or (co-residency mode) when the launch leaves SMs idle
    if ((!cores || p.grid < kRefSMs) && p.smem <= kRefSmemHalf) p.smem = kRefSmemHalf + 4096;
    p.use = true;
    return p;
}

int launch_gemv_tma(DeviceInfo *dev, int xmode, const int8_t *q, const uint16_t *x, const uint8_t *packed, int64_t M,
                    int64_t N, int64_t K, int32_t *y_i32, uint16_t *y_bf16, const float *gamma, const float *s_act,
                    const TmaPlan &tp, cudaStream_t st) {
    // per-slice staging barriers (a variant of its own: one int8 token, dp4a)
    // where CTAs have many items over few slices; measured on B200: 55296 x
    // 5120 (120 items per CTA) 13.1 -> 12.3 us; 20480 x 3200 (35) 5.21 ->
    // 5.13 us alone but the eight-shape sweep 0.15 us slower per step with it;
    // calls of 15 items or fewer per CTA 0.07-0.19 us slower; 5120 x 27648
    // (54 slices) 0.2 us slower
    int sf = (xmode == 0 && tp.mt == 1 && !tp.mma && (int64_t)tp.max_blocks * tp.slices >= 64 && tp.slices <= 32) ? 1 : 0;
    if (xmode == 0 && tp.mt == 1 && !tp.mma && (gemv_tune().sflags == 0 || gemv_tune().sflags == 1))
        sf = gemv_tune().sflags;
    TmaKernel kern = tma_kernel_for(xmode, tp.cfg, tp.mt, tp.rows, tp.mma, sf);
    if (kern == nullptr) return BITNET_ERR_UNSUPPORTED;
    if (tensor_map_encoder() == nullptr ||
        tp.smem > tma_max_dynamic_smem(dev, xmode, tp.cfg, tp.mt, tp.rows, tp.mma, sf))
        return BITNET_ERR_CUDA;
    const int64_t row_bytes = packed_row_bytes(K);
    CUtensorMap map;
    if (!encode_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)row_bytes, (uint64_t)N, (uint64_t)row_bytes,
                   kTmaSliceBytes, (uint32_t)tp.rows, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
        return BITNET_ERR_CUDA;
    // test hook (BITNET_TEST_STALL=1): the first TMA launch of the process
    // makes one wait run out, exercising the device-timeout path
    static std::atomic<int> stall_once{-1};
    if (stall_once.load() == -1) {
        const char *e = getenv("BITNET_TEST_STALL");
        int expect = -1;
        stall_once.compare_exchange_strong(expect, (e != nullptr && e[0] == '1') ? 1 : 0);
    }
    int one = 1;
    const int test_stall = stall_once.compare_exchange_strong(one, 0) ? 1 : 0;
    GemvTmaArgs a{};
    a.q = q;
    a.x = x;
    a.M = (int)M;
    a.N = N;
    a.K = K;
    a.slices = tp.slices;
    a.blk_begin = 0;
    a.nblocks = tp.nblocks;
    a.max_blocks_cta = tp.max_blocks;
    a.ns = tp.ns;
    a.y_i32 = y_i32;
    a.y_bf16 = y_bf16;
    a.gamma = gamma;
    a.s_act = s_act;
    a.test_stall = test_stall;
    a.evict_first = gemv_tune().l2 == 0 ? 0 : 1;  // measured on B200: 25.9 -> 25.6 us per sweep step
    return launched(launch_pdl(kern, dim3(tp.grid), dim3(kTmaCfg[tp.cfg][0] * 32), tp.smem, st, map, a));
}

// xmode 0: int8 activations q (row stride ldq); xmode 1: bf16 activations x,
// quantised per token inside the kernel.
int launch_gemv(DeviceInfo *dev, int xmode, const int8_t *q, const uint16_t *x, int64_t ldq,
                const uint8_t *packed, int64_t M, int64_t N, int64_t K, int32_t *y_i32, uint16_t *y_bf16,
                const float *s_act, const float *gamma, void *ws, cudaStream_t st) {
    {
        const TmaPlan tp = tma_plan(M, N, K);
        if (tp.use && ldq == K)
            return launch_gemv_tma(dev, xmode, q, x, packed, M, N, K, y_i32, y_bf16, gamma, s_act, tp, st);
    }
    const GemvSplit sp = plan_split(M, N, K);
    const GemvTune &tn = gemv_tune();
    int G = lanes_per_row(sp.cps);
    if (tn.G == 8 || tn.G == 16 || tn.G == 32) G = tn.G;
    const size_t smem = (size_t)sp.cps * 64;

    // rows per lane group: the most that still give >= 2 tasks per resident warp
    int idx = 0, ru = 0;
    for (int cand : {5, 3, 0}) {  // (4,2), (2,4), (1,4)
        GemvKernel k = gemv_kernel_for(G, cand, xmode, &idx);
        const int c = gemv_ctas_per_sm(dev, idx, k, smem);
        if (c <= 0) return BITNET_ERR_CUDA;
        const int64_t warps = (int64_t)dev->sm_count * c * (kThreads / 32);
        ru = cand;
        if (ceil_div(N, (32 / G) * kRU[cand][0]) * M * sp.S >= 2 * warps) break;
    }
    if (tn.R > 0 || tn.U > 0) {
        for (int i = 0; i < 6; ++i)
            if (kRU[i][0] == tn.R && kRU[i][1] == tn.U) ru = i;
    }
    const int R = kRU[ru][0];
    GemvKernel kern = gemv_kernel_for(G, ru, xmode, &idx);
    int ctas = gemv_ctas_per_sm(dev, idx, kern, smem);
    if (ctas <= 0) return BITNET_ERR_CUDA;
    if (tn.ctas > 0 && tn.ctas < ctas) ctas = tn.ctas;

    GemvArgs a{};
    a.ldq = ldq;
    a.W = packed;
    a.row_bytes = packed_row_bytes(K);
    a.N = N;
    a.K = K;
    a.nch_total = (int)(k_pad(K) / 64);
    a.cps = sp.cps;
    a.prefetch_tasks = tn.prefetch >= 0 ? tn.prefetch : 1;
    a.gamma = gamma;
    int32_t *partial = sp.S > 1 ? static_cast<int32_t *>(ws) : nullptr;
    float *s_out = (sp.S > 1 && xmode == 1)
                       ? reinterpret_cast<float *>(static_cast<char *>(ws) + (int64_t)sp.S * M * N * 4)
                       : nullptr;

    const int64_t row_tasks = ceil_div(N, (32 / G) * R);
    // tokens go to gridDim.z (at most 65535 per launch)
    for (int64_t m0 = 0; m0 < M; m0 += 65535) {
        const int64_t mc = M - m0 < 65535 ? M - m0 : 65535;
        GemvArgs c = a;
        c.q = q ? q + m0 * ldq : nullptr;
        c.x = x ? x + m0 * K : nullptr;
        c.M = (int)mc;
        c.y_i32 = y_i32 ? y_i32 + m0 * N : nullptr;
        c.y_bf16 = y_bf16 ? y_bf16 + m0 * N : nullptr;
        c.s_act = s_act ? s_act + m0 : nullptr;
        c.partial = partial;
        c.s_out = s_out ? s_out + m0 : nullptr;
        int64_t gx = ceil_div(row_tasks, kThreads / 32);
        const int64_t cap = ceil_div((int64_t)dev->sm_count * ctas, (int64_t)sp.S * mc);
        if (gx > cap) gx = cap;
        if (gx < 1) gx = 1;
        const dim3 grid((unsigned)gx, (unsigned)sp.S, (unsigned)mc);
        int rc = launched(launch_pdl(kern, grid, dim3(kThreads), smem, st, c));
        if (rc != BITNET_OK) return rc;
        if (sp.S > 1) {
            rc = launched(launch_pdl(gemv_splitk_reduce_kernel, dim3(grid_for(mc * N, kThreads * 4, dev->sm_count)),
                                     dim3(kThreads), (size_t)0, st, c, sp.S));
            if (rc != BITNET_OK) return rc;
        }
    }
    return BITNET_OK;
}

// ------------------------------------------------------------------ allocation-free scratch
// Scratch of bitnet_w2a8_gemm_noalloc: one array per device, shared by every
// call; its device address is looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[BITNET_NOALLOC_SCRATCH_BYTES];
void *g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

int noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BITNET_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BITNET_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return BITNET_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return BITNET_OK;
}

// ------------------------------------------------------------------ tcgen05 GEMM (M > 1)
// Token-tile widths (UMMA N) of the persistent tensor-core GEMM.  The first
// kTcNumPlanned are the planner's candidates (widest first); the rest are
// reached through the tuning override only.
constexpr int kTcNumBT = 10;
constexpr int kTcNumPlanned = 5;
constexpr int kTcBTs[kTcNumBT] = {192, 128, 64, 32, 16, 128, 96, 64, 128, 192};
// k per stage of each variant (its packed rows are k / 4 bytes, 64-byte or
// 128-byte swizzled; its code stages k / 4 tensor-memory columns)
constexpr int kTcSKs[kTcNumBT] = {256, 512, 256, 256, 256, 256, 256, 256, 256, 256};
// Time of one stage of each variant with every SM busy, measured on B200 (us):
// the MMA time for the wide tiles, the decoder-to-tensor-core hand-over
// (~0.6 us) for the narrow ones.
constexpr double kTcStageUs[kTcNumBT] = {0.69, 1.12, 0.60, 0.60, 0.60, 0.60, 0.60, 0.60, 0.60, 0.69};
using TcKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const GemmTcArgs);

// Rings (activation, code, packed stages) per variant.  The 192-, 128- and
// 64-token variants take all 512 tensor-memory columns (2 accumulators + code
// stages) and more than half an SM's shared memory, so one CTA per SM; the
// narrower ones take 256 columns.  The next three trade accumulator width for
// code stages (4, 5 and 6 in flight instead of 2); the last two keep a single
// accumulator (no overlap of a unit's epilogue with the next unit) for 6 and
// 5 code stages.
#define BITNET_TC_VARIANTS(OUT)                                                                                      \
    gemm_w2a8_tc_kernel<192, OUT, 3, 2, 4, 256>, gemm_w2a8_tc_kernel<128, OUT, 2, 2, 3, 512>,                      \
        gemm_w2a8_tc_kernel<64, OUT, 6, 4, 6, 256>, gemm_w2a8_tc_kernel<32, OUT, 8, 3, 6, 256>,                    \
        gemm_w2a8_tc_kernel<16, OUT, 8, 3, 6, 256>, gemm_w2a8_tc_kernel<128, OUT, 4, 4, 6, 256>,                   \
        gemm_w2a8_tc_kernel<96, OUT, 5, 5, 6, 256>, gemm_w2a8_tc_kernel<64, OUT, 6, 6, 8, 256>,                    \
        gemm_w2a8_tc_kernel<128, OUT, 4, 6, 6, 256, 1>, gemm_w2a8_tc_kernel<192, OUT, 3, 5, 4, 256, 1>
TcKernel tc_kernel_for(int bt_idx, bool bf16, size_t *smem) {
    static const TcKernel k[2 * kTcNumBT] = {BITNET_TC_VARIANTS(false), BITNET_TC_VARIANTS(true)};
    static const size_t raw[kTcNumBT] = {TcSmem<192, 3, 2, 4, 256>::kBytes, TcSmem<128, 2, 2, 3, 512>::kBytes,
                                         TcSmem<64, 6, 4, 6, 256>::kBytes,  TcSmem<32, 8, 3, 6, 256>::kBytes,
                                         TcSmem<16, 8, 3, 6, 256>::kBytes,  TcSmem<128, 4, 4, 6, 256>::kBytes,
                                         TcSmem<96, 5, 5, 6, 256>::kBytes,  TcSmem<64, 6, 6, 8, 256>::kBytes,
                                         TcSmem<128, 4, 6, 6, 256, 1>::kBytes, TcSmem<192, 3, 5, 4, 256, 1>::kBytes};
    *smem = raw[bt_idx] + 1024;  // + alignment slack
    return k[(bf16 ? kTcNumBT : 0) + bt_idx];
}
#undef BITNET_TC_VARIANTS

// Token-tile width and K-split of the tensor-core GEMM, from a small cost
// model of the persistent kernel on the B200's 148 SMs (so the workspace a
// shape needs is fixed whatever the device): an SM runs its work units one
// after another, each stage taking the variant's measured time (kTcStageUs;
// at 128 k per stage every variant took ~0.4 us, bounded by the hand-over
// between decoders and tensor core, which is why the stages are now 256 or
// 512 k); the pipeline fill and the last epilogue add ~2 us.  A K-split is
// considered only when the tiles do not fill the SMs; it adds a launch
// (~2.5 us) plus the zeroing of the int32 output and one reduce-add pass over
// it per split, each at ~1.4 TB/s (measured: a 2-way split of M = 2048,
// N = 13824 cost more than the whole unsplit GEMM).  Candidates: token tiles
// from the smallest that holds M (at most 192) down to 16, splits 1..16.
struct TcPlan {
    int bt_idx, S, sps;
};

TcPlan tc_plan(int64_t M, int64_t N, int64_t K) {
    constexpr int kRefSMs = 148;
    TcPlan p{};
    const GemvTune &tn = gemv_tune();
    const int64_t nt = ceil_div(N, kTcRows);
    int first = kTcNumPlanned - 1;
    while (first > 0 && kTcBTs[first] < M) --first;  // smallest tile >= M, else the widest
    double best = 1e30;
    for (int i = first; i < kTcNumPlanned; ++i) {
        const int BT = kTcBTs[i];
        const int nk = (int)ceil_div(k_pad(K), kTcSKs[i]);
        const int64_t tiles = nt * ceil_div(M, BT);
        const double stage_us = kTcStageUs[i];
        const double out_us = (double)M * (double)N * 4.0 / 1.4e6;  // one pass over the int32 output
        for (int S = 1; S <= 16 && S <= nk; ++S) {
            if (S > 1 && tiles >= kRefSMs) break;
            const int sps = (int)ceil_div(nk, S);
            if (ceil_div(nk, sps) != S) continue;
            const int64_t rounds = ceil_div(tiles * S, kRefSMs);
            const double t = (double)rounds * sps * stage_us + 2.0 + (S > 1 ? 2.5 + (S + 1) * out_us : 0.0);
            if (t < best * 0.999) {
                best = t;
                p.bt_idx = i;
                p.S = S;
                p.sps = sps;
            }
        }
    }
    // tuning overrides: R = -1..-10 picks the variant, S the split count
    if (tn.R < 0 && -tn.R <= kTcNumBT) p.bt_idx = -tn.R - 1;
    const int nk = (int)ceil_div(k_pad(K), kTcSKs[p.bt_idx]);
    if (tn.S > 0) {
        const int S = tn.S < nk ? tn.S : nk;
        p.sps = (int)ceil_div(nk, S);
        p.S = (int)ceil_div(nk, p.sps);
    } else if (tn.R < 0) {
        p.S = 1;
        p.sps = nk;
    }
    return p;
}

// reduce: add int32 results into y_i32 (which the caller has zeroed).
// BitLinear with the activation quantisation inside the GEMM launch: the bf16
// activations (the quantised rows go where the activation map points).
struct TcFuse {
    const uint16_t *x = nullptr;
};
std::atomic<uint32_t> g_bar_slot{0};

int launch_gemm_tc(DeviceInfo *dev, const int8_t *q, int64_t lda, const uint8_t *packed, int64_t M, int64_t N,
                   int64_t K, int32_t *y_i32, uint16_t *y_bf16, const float *s_act, const float *gamma,
                   const TcPlan &tp, int reduce, cudaStream_t st, const TcFuse &fuse = TcFuse{}) {
    if (tensor_map_encoder() == nullptr) return BITNET_ERR_CUDA;
    const int bi = tp.bt_idx;
    const int BT = kTcBTs[bi];
    const bool bf16 = y_bf16 != nullptr;
    size_t smem = 0;
    TcKernel kern = tc_kernel_for(bi, bf16, &smem);
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        bool &set = dev->tc_attr_set[(bf16 ? kTcNumBT : 0) + bi];
        if (!set) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
                return BITNET_ERR_CUDA;
            set = true;
        }
    }
    CUtensorMap amap, pmap;
    if (!encode_2d(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)M, (uint64_t)lda, kTcBK,
                   (uint32_t)BT, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
        return BITNET_ERR_CUDA;
    {
        const int64_t row_bytes = packed_row_bytes(K);
        if (!encode_2d(&pmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)row_bytes, (uint64_t)N,
                       (uint64_t)row_bytes, (uint32_t)(kTcSKs[bi] / 4), kTcRows,
                       kTcSKs[bi] == 512 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
            return BITNET_ERR_CUDA;
    }
    // outputs: 32-row boxes of 128 bytes per row, stored through TMA when the
    // rows are 16-byte strided and the base 16-byte aligned
    CUtensorMap ymap;
    memset(&ymap, 0, sizeof(ymap));
    const int esize = bf16 ? 2 : 4;
    void *ybase = bf16 ? static_cast<void *>(y_bf16) : static_cast<void *>(y_i32);
    int tma_store = ((N * esize) % 16 == 0) && aligned(ybase, 16);
    // boxes of 32 weight rows (inner) x up to 32 tokens, unswizzled
    if (tma_store && !encode_2d(&ymap, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_INT32, ybase,
                                (uint64_t)N, (uint64_t)M, (uint64_t)(N * esize), kTcBox,
                                (uint32_t)(BT < kTcBox ? BT : kTcBox), CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE))
        tma_store = 0;
    GemmTcArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.nk = (int)ceil_div(k_pad(K), kTcSKs[bi]);
    a.y_i32 = y_i32;
    a.y_bf16 = y_bf16;
    a.s_act = s_act;
    a.gamma = gamma;
    a.tma_store = tma_store;
    a.sps = tp.sps;
    a.reduce = reduce;
    a.tiles_n = (int)ceil_div(N, kTcRows);
    a.tiles_m = (int)ceil_div(M, BT);
    a.splits = tp.S;
    if (fuse.x != nullptr) {  // q and s_act are written by this launch
        a.x = fuse.x;
        a.qout = const_cast<int8_t *>(q);
        a.ldq = lda;
        a.bar_slot = (int)(g_bar_slot.fetch_add(1, std::memory_order_relaxed) % kGridBarSlots);
    }
    // persistent: one CTA per SM (or fewer, when there are fewer work units)
    const int64_t units = (int64_t)a.tiles_n * a.tiles_m * a.splits;
    if (units > (int64_t)1 << 30) return BITNET_ERR_UNSUPPORTED;  // work units are counted in int
    const int grid = (int)(units < dev->sm_count ? units : dev->sm_count);
    return launched(launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st, amap, pmap, ymap, a));
}

// Copies int8 activations [M, K] into rows of K_pad bytes, zero-padded, so the
// tensor map's row stride is a multiple of 16 bytes.
__global__ void __launch_bounds__(kThreads) repack_q_kernel(const int8_t *__restrict__ q, int64_t M, int64_t K,
                                                            int64_t ld, int8_t *__restrict__ out) {
    const int64_t total = M * ld;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total; i += (int64_t)gridDim.x * kThreads) {
        const int64_t m = i / ld, k = i - m * ld;
        out[i] = k < K ? q[m * K + k] : (int8_t)0;
    }
}

// BitLinear epilogue after a K-split: y = bf16_rne(acc * (gamma / s_m)), the
// same fp32 operations as the GEMM's own epilogue.
__global__ void __launch_bounds__(kThreads) rescale_bf16_kernel(const int32_t *__restrict__ acc, int64_t M, int64_t N,
                                                                const float *__restrict__ s, const float *__restrict__ gamma,
                                                                uint16_t *__restrict__ y) {
    pdl_wait();
    const float g = *gamma;
    const int64_t total = M * N;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total; i += (int64_t)gridDim.x * kThreads) {
        const float f = __fdiv_rn(g, s[i / N]);
        y[i] = float_to_bf16_bits_rn(__fmul_rn((float)acc[i], f));
    }
}

// ------------------------------------------------------------------ dispatch
// One plan for every caller of the contraction, so the path taken and the
// scratch it needs always agree.
enum { kPathGemv = 0, kPathTc = 1 };
struct GemmPlan {
    int path;
    bool repack;       // int8 activations copied to K_pad-strided rows first
    int64_t ws_bytes;
    TcPlan tc;
};

GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, bool q_tma_ok, bool bitlinear) {
    GemmPlan p{};
    (void)q_tma_ok;
    if (M <= kGemvMaxTokens) {  // decode and small batches: the TMA GEMV reads the weights once
        const TmaPlan tp = tma_plan(M, N, K);
        if (tp.use) {
            p.path = kPathGemv;
            p.ws_bytes = tp.ws_bytes;
            // BitLinear on more tokens than the fused prologue takes quantises
            // them once into the workspace (before the GEMV's own scratch)
            if (bitlinear && M > fused_quant_max_tokens())
                p.ws_bytes += round_up(M * K, 256) + round_up(M * 4, 256);
            return p;
        }
    }
    if (M >= 2 && K >= kTcBK) {
        p.path = kPathTc;
        p.tc = tc_plan(M, N, K);
        const int64_t qbytes = round_up(M * k_pad(K), 256);
        if (bitlinear) {
            // quantised activations, scales and, for a K-split, int32 sums
            p.ws_bytes = qbytes + round_up(M * 4, 256) + (p.tc.S > 1 ? round_up(M * N * 4, 256) : 0);
        } else {
            p.repack = !q_tma_ok;
            p.ws_bytes = p.repack ? qbytes : 0;
        }
    } else {
        p.path = kPathGemv;
        const TmaPlan tp = tma_plan(M, N, K);
        p.ws_bytes = tp.use ? tp.ws_bytes : plan_split(M, N, K).ws_bytes;
    }
    return p;
}

// The whole int32 contraction for M, N, K >= 1 (validated by the caller).
int run_w2a8_gemm(DeviceInfo *dev, const int8_t *q, const uint8_t *packed, int32_t *y, int64_t M, int64_t N,
                  int64_t K, void *ws, const GemmPlan &p, cudaStream_t st) {
    if (p.path == kPathGemv) return launch_gemv(dev, 0, q, nullptr, K, packed, M, N, K, y, nullptr, nullptr, nullptr, ws, st);
    const int8_t *qa = q;
    int64_t lda = K;
    if (p.repack) {
        int8_t *qp = static_cast<int8_t *>(ws);
        lda = k_pad(K);
        repack_q_kernel<<<grid_for(M * lda, kThreads * 8, dev->sm_count), kThreads, 0, st>>>(q, M, K, lda, qp);
        const int rc = launched();
        if (rc != BITNET_OK) return rc;
        qa = qp;
    }
    if (p.tc.S > 1) {  // K-split: the splits add into a zeroed output
        fill_kernel<int32_t><<<grid_for(M * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(y, M * N, 0);
        const int rc = launched();
        if (rc != BITNET_OK) return rc;
    }
    return launch_gemm_tc(dev, qa, lda, packed, M, N, K, y, nullptr, nullptr, nullptr, p.tc, p.tc.S > 1, st);
}

inline bool q_tma_ok(const int8_t *q, int64_t K) { return (K % 16) == 0 && aligned(q, 16); }

}  // namespace
}  // namespace bitnet

using namespace bitnet;

extern "C" {

BITNET_API const char *bitnet_status_string(int status) {
    switch (status) {
        case BITNET_OK: return "BITNET_OK";
        case BITNET_ERR_INVALID_ARG: return "BITNET_ERR_INVALID_ARG: null pointer or invalid size";
        case BITNET_ERR_ALIGNMENT: return "BITNET_ERR_ALIGNMENT: pointer misses its required alignment";
        case BITNET_ERR_WORKSPACE: return "BITNET_ERR_WORKSPACE: workspace missing or too small";
        case BITNET_ERR_CUDA: return "BITNET_ERR_CUDA: CUDA runtime call or kernel launch failed";
        case BITNET_ERR_DEVICE_TIMEOUT: return "BITNET_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait";
        case BITNET_ERR_UNSUPPORTED: return "BITNET_ERR_UNSUPPORTED: device is not an sm_100 (B200-class) GPU";
        default: return "unknown bitnet status";
    }
}

BITNET_API int bitnet_layout_version(void) { return BITNET_LAYOUT_VERSION; }

BITNET_API int64_t bitnet_packed_bytes(int64_t N, int64_t K) {
    if (!sizes_ok(1, N, K)) return -1;
    return N * packed_row_bytes(K);
}

BITNET_API int64_t bitnet_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (!sizes_ok(M, N, K)) return -1;
    int64_t need = (int64_t)kAbsmeanMaxBlocks * 8;  // bitnet_absmean partials
    if (M > 0 && N > 0 && K > 0) {
        const int64_t g = plan_gemm(M, N, K, false, false).ws_bytes;
        const int64_t b = plan_gemm(M, N, K, false, true).ws_bytes;
        if (g > need) need = g;
        if (b > need) need = b;
    }
    return need;
}

BITNET_API int bitnet_absmean(const uint16_t *W, int64_t N, int64_t K, float *gamma, void *workspace,
                              int64_t workspace_bytes, void *stream) {
    if (gamma == nullptr || !sizes_ok(1, N, K) || (N * K > 0 && W == nullptr)) return BITNET_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(gamma, 4)) return BITNET_ERR_ALIGNMENT;
    const int64_t total = N * K;
    const int nblk = absmean_blocks(total);
    if (workspace == nullptr || workspace_bytes < (int64_t)nblk * 8) return BITNET_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BITNET_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double *partial = static_cast<double *>(workspace);
    absmean_partial_kernel<<<nblk, kThreads, 0, st>>>(W, total, partial);
    if ((rc = launched()) != BITNET_OK) return rc;
    absmean_final_kernel<<<1, kThreads, 0, st>>>(partial, nblk, total, gamma);
    return launched();
}

BITNET_API int bitnet_ternarize(const uint16_t *W, int64_t N, int64_t K, const float *gamma, int8_t *W_t,
                                void *stream) {
    if (!sizes_ok(1, N, K) || gamma == nullptr || (N * K > 0 && (W == nullptr || W_t == nullptr)))
        return BITNET_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(gamma, 4)) return BITNET_ERR_ALIGNMENT;
    if (N * K == 0) return BITNET_OK;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    ternarize_kernel<<<grid_for(N * K, kThreads * 8, dev->sm_count), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        W, N * K, gamma, W_t);
    return launched();
}

BITNET_API int bitnet_pack_weights(const int8_t *W_t, int64_t N, int64_t K, uint8_t *packed, int32_t *invalid_count,
                                   void *stream) {
    if (!sizes_ok(1, N, K) || (N > 0 && packed == nullptr) || (N * K > 0 && W_t == nullptr))
        return BITNET_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(invalid_count, 4)) return BITNET_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (invalid_count != nullptr && cudaMemsetAsync(invalid_count, 0, sizeof(int32_t), st) != cudaSuccess)
        return BITNET_ERR_CUDA;
    const int64_t wpr = packed_row_bytes(K) / 4;
    if (N * wpr == 0) return BITNET_OK;
    pack_v1_kernel<<<grid_for(N * wpr, kThreads, dev->sm_count, 16), kThreads, 0, st>>>(
        W_t, N, K, wpr, reinterpret_cast<uint32_t *>(packed), invalid_count);
    return launched();
}

BITNET_API int bitnet_quant_act(const uint16_t *x, int64_t M, int64_t K, int8_t *q, float *s, int32_t *rowsum,
                                void *stream) {
    if (!sizes_ok(M, 1, K) || (M > 0 && s == nullptr) || (M * K > 0 && (x == nullptr || q == nullptr)))
        return BITNET_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(s, 4) || !aligned(rowsum, 4)) return BITNET_ERR_ALIGNMENT;
    if (M == 0) return BITNET_OK;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    return launch_quant(dev, x, M, K, q, K, false, s, rowsum, static_cast<cudaStream_t>(stream));
}

BITNET_API int bitnet_w2a8_gemm(const int8_t *q, const uint8_t *packed, int32_t *y, int64_t M, int64_t N, int64_t K,
                                void *workspace, int64_t workspace_bytes, void *stream) {
    if (!sizes_ok(M, N, K)) return BITNET_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BITNET_OK;
    if (y == nullptr || (K > 0 && (q == nullptr || packed == nullptr))) return BITNET_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(y, 4)) return BITNET_ERR_ALIGNMENT;
    const GemmPlan p = K > 0 ? plan_gemm(M, N, K, q_tma_ok(q, K), false) : GemmPlan{};
    if (p.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < p.ws_bytes)) return BITNET_ERR_WORKSPACE;
    if (p.ws_bytes > 0 && !aligned(workspace, 256)) return BITNET_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        fill_kernel<int32_t><<<grid_for(M * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(y, M * N, 0);
        return launched();
    }
    return run_w2a8_gemm(dev, q, packed, y, M, N, K, workspace, p, st);
}

BITNET_API int bitnet_bitlinear(const uint16_t *x, const uint8_t *packed, const float *gamma, uint16_t *y, int64_t M,
                                int64_t N, int64_t K, void *workspace, int64_t workspace_bytes, void *stream) {
    if (!sizes_ok(M, N, K)) return BITNET_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BITNET_OK;
    if (y == nullptr || gamma == nullptr || (K > 0 && (x == nullptr || packed == nullptr)))
        return BITNET_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(packed, 16) || !aligned(y, 2) || !aligned(gamma, 4)) return BITNET_ERR_ALIGNMENT;
    const GemmPlan p = K > 0 ? plan_gemm(M, N, K, false, true) : GemmPlan{};
    if (p.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < p.ws_bytes)) return BITNET_ERR_WORKSPACE;
    if (p.ws_bytes > 0 && !aligned(workspace, 256)) return BITNET_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        fill_kernel<uint16_t><<<grid_for(M * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(y, M * N, 0);
        return launched();
    }
    if (p.path == kPathGemv && M > fused_quant_max_tokens() && M <= kGemvMaxTokens && tma_plan(M, N, K).use) {
        // small batch: quantise the tokens once, then one pass over the weights
        int8_t *q = static_cast<int8_t *>(workspace);
        float *s = reinterpret_cast<float *>(static_cast<char *>(workspace) + round_up(M * K, 256));
        void *gws = static_cast<char *>(workspace) + round_up(M * K, 256) + round_up(M * 4, 256);
        if ((rc = launch_quant(dev, x, M, K, q, K, false, s, nullptr, st)) != BITNET_OK) return rc;
        return launch_gemv(dev, 0, q, nullptr, K, packed, M, N, K, nullptr, y, s, gamma, gws, st);
    }
    if (p.path == kPathGemv)  // the tokens are quantised inside the GEMV's prologue: one launch
        return launch_gemv(dev, 1, nullptr, x, K, packed, M, N, K, nullptr, y, nullptr, gamma, workspace, st);
    // quantise into K_pad-strided, zero-padded rows of the workspace, then the
    // tensor-core GEMM with the bf16 epilogue.  The quantisation pass is a
    // launch of its own: measured on B200 it beats quantising inside the GEMM
    // launch (tuning field `fuse` = 1), whose CTAs must all meet at a grid
    // barrier before the first activation load.
    const int64_t ldq = k_pad(K);
    int8_t *q = static_cast<int8_t *>(workspace);
    float *s = reinterpret_cast<float *>(static_cast<char *>(workspace) + round_up(M * ldq, 256));
    TcFuse fuse;
    if (gemv_tune().fuse == 1) {
        fuse.x = x;
    } else if ((rc = launch_quant(dev, x, M, K, q, ldq, true, s, nullptr, st)) != BITNET_OK) {
        return rc;
    }
    if (p.tc.S == 1) return launch_gemm_tc(dev, q, ldq, packed, M, N, K, nullptr, y, s, gamma, p.tc, 0, st, fuse);
    // K-split: int32 sums in the workspace, then the rescale to bf16
    int32_t *acc = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(s) + round_up(M * 4, 256));
    fill_kernel<int32_t><<<grid_for(M * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(acc, M * N, 0);
    if ((rc = launched()) != BITNET_OK) return rc;
    if ((rc = launch_gemm_tc(dev, q, ldq, packed, M, N, K, acc, nullptr, s, nullptr, p.tc, 1, st, fuse)) != BITNET_OK)
        return rc;
    return launched(launch_pdl(rescale_bf16_kernel, dim3(grid_for(M * N, kThreads * 4, dev->sm_count)),
                               dim3(kThreads), (size_t)0, st, (const int32_t *)acc, M, N, (const float *)s, gamma, y));
}

BITNET_API int bitnet_w2a8_gemm_noalloc(const int8_t *q, const uint8_t *packed, int32_t *y, int64_t M, int64_t N,
                                        int64_t K, void *stream) {
    if (!sizes_ok(M, N, K)) return BITNET_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BITNET_OK;
    if (y == nullptr || (K > 0 && (q == nullptr || packed == nullptr))) return BITNET_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(y, 4)) return BITNET_ERR_ALIGNMENT;
    const GemmPlan p = K > 0 ? plan_gemm(M, N, K, q_tma_ok(q, K), false) : GemmPlan{};
    if (p.ws_bytes > (int64_t)BITNET_NOALLOC_SCRATCH_BYTES) return BITNET_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != BITNET_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        fill_kernel<int32_t><<<grid_for(M * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(y, M * N, 0);
        return launched();
    }
    return run_w2a8_gemm(dev, q, packed, y, M, N, K, scratch, p, st);
}

BITNET_API int bitnet_get_device_error(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return BITNET_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
        // a launch that gave up may have left a grid barrier half-counted
        static const unsigned int zeros[kGridBarSlots] = {};
        if (cudaMemcpyToSymbol(g_grid_bar, zeros, sizeof(zeros)) != cudaSuccess) return BITNET_ERR_CUDA;
    }
    return v;
}

BITNET_API int64_t bitnet_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
