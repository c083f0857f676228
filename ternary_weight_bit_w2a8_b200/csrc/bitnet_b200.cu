// bitnet_b200.cu -- the C ABI of libbitnet_b200.so (declared in
// include/bitnet_b200.h): argument checks, plan selection and launches.
// All kernels are in the headers included below; this is the library's single
// translation unit, so file-scope device state (the error word) is shared.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "gemv.cuh"
#include "quant.cuh"
#include "weights.cuh"

namespace bitnet {
namespace {

std::atomic<int64_t> g_launches{0};

constexpr int kMaxDevices = 64;
constexpr int kMaxSliceChunks = 1536;  // activations of one K-slice: 96 KB of shared memory
constexpr int kPlanSlots = 148 * 16;   // warp slots the GEMV plan aims to fill (fixed: plans depend on shape only)

struct DeviceInfo {
    bool init = false;
    int status = BITNET_OK;
    int sm_count = 0;
    unsigned smem_attr_set = 0;  // GEMV instantiations whose shared-memory limit is raised
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
        d.status = (major == 10) ? BITNET_OK : BITNET_ERR_UNSUPPORTED;
        d.sm_count = sms;
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

// ------------------------------------------------------------------ fill (K == 0)
template <typename T>
__global__ void __launch_bounds__(kThreads) fill_kernel(T *p, int64_t n, T v) {
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kThreads) p[i] = v;
}

// ------------------------------------------------------------------ GEMV plan
struct GemvPlan {
    int G, R, UN, S, cps;
    size_t smem;
    int64_t ws_bytes;
};

GemvPlan plan_gemv(int64_t M, int64_t N, int64_t K) {
    GemvPlan p{};
    const int nch = (int)(k_pad(K) / 64);
    p.G = nch >= 128 ? 32 : (nch >= 48 ? 16 : 8);
    const int64_t lanes_rows = 32 / p.G;
    auto tasks = [&](int R) { return ceil_div(N, lanes_rows * R) * M; };
    p.R = tasks(4) >= 2 * kPlanSlots ? 4 : (tasks(2) >= 2 * kPlanSlots ? 2 : 1);
    int S = (int)ceil_div(nch, kMaxSliceChunks);
    // split K only when rows are too few to fill the GPU and every lane still
    // keeps >= 4 chunks per slice (small problems are latency-bound: a second
    // launch would cost more than it saves)
    while (tasks(p.R) * S < kPlanSlots / 4 && nch / (2 * S) >= 4 * p.G) S *= 2;
    p.cps = (int)ceil_div(nch, S);
    p.S = (int)ceil_div(nch, p.cps);
    p.UN = 8 / p.R;
    p.smem = (size_t)p.cps * 64;
    p.ws_bytes = p.S > 1 ? (int64_t)p.S * M * N * 4 : 0;
    return p;
}

using GemvKernel = void (*)(const GemvArgs);

GemvKernel gemv_kernel_for(int G, int R, int *index) {
    static const GemvKernel table[9] = {
        gemv_w2a8_kernel<8, 4, 2>,  gemv_w2a8_kernel<8, 2, 4>,  gemv_w2a8_kernel<8, 1, 8>,
        gemv_w2a8_kernel<16, 4, 2>, gemv_w2a8_kernel<16, 2, 4>, gemv_w2a8_kernel<16, 1, 8>,
        gemv_w2a8_kernel<32, 4, 2>, gemv_w2a8_kernel<32, 2, 4>, gemv_w2a8_kernel<32, 1, 8>,
    };
    const int gi = G == 8 ? 0 : (G == 16 ? 1 : 2);
    const int ri = R == 4 ? 0 : (R == 2 ? 1 : 2);
    *index = gi * 3 + ri;
    return table[*index];
}

int launch_gemv(DeviceInfo *dev, const int8_t *q, int64_t ldq, const uint8_t *packed, int64_t M, int64_t N,
                int64_t K, int32_t *y_i32, uint16_t *y_bf16, const float *s_act, const float *gamma,
                void *ws, cudaStream_t st) {
    const GemvPlan p = plan_gemv(M, N, K);
    GemvArgs a{};
    a.q = q;
    a.ldq = ldq;
    a.W = packed;
    a.row_bytes = packed_row_bytes(K);
    a.N = N;
    a.K = K;
    a.nch_total = (int)(k_pad(K) / 64);
    a.cps = p.cps;
    a.M = (int)M;
    a.y_i32 = y_i32;
    a.y_bf16 = y_bf16;
    a.partial = p.S > 1 ? static_cast<int32_t *>(ws) : nullptr;
    a.s_act = s_act;
    a.gamma = gamma;

    int idx = 0;
    GemvKernel kern = gemv_kernel_for(p.G, p.R, &idx);
    if (p.smem > 48 * 1024) {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        if (!(dev->smem_attr_set & (1u << idx))) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSliceChunks * 64) !=
                cudaSuccess)
                return BITNET_ERR_CUDA;
            dev->smem_attr_set |= 1u << idx;
        }
    }
    const int64_t row_tasks = ceil_div(N, (32 / p.G) * p.R);
    // tokens go to gridDim.z (at most 65535 per launch)
    for (int64_t m0 = 0; m0 < M; m0 += 65535) {
        const int64_t mc = M - m0 < 65535 ? M - m0 : 65535;
        GemvArgs c = a;
        c.q = q + m0 * ldq;
        c.M = (int)mc;
        c.y_i32 = y_i32 ? y_i32 + m0 * N : nullptr;
        c.y_bf16 = y_bf16 ? y_bf16 + m0 * N : nullptr;
        c.s_act = s_act ? s_act + m0 : nullptr;
        int64_t gx = ceil_div(row_tasks, kThreads / 32);
        const int64_t cap = ceil_div((int64_t)dev->sm_count * 4, (int64_t)p.S * mc);
        if (gx > cap) gx = cap;
        if (gx < 1) gx = 1;
        dim3 grid((unsigned)gx, (unsigned)p.S, (unsigned)mc);
        kern<<<grid, kThreads, p.smem, st>>>(c);
        int rc = launched();
        if (rc != BITNET_OK) return rc;
        if (p.S > 1) {
            gemv_splitk_reduce_kernel<<<grid_for(mc * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(c, p.S);
            if ((rc = launched()) != BITNET_OK) return rc;
        }
    }
    return BITNET_OK;
}

int64_t bitlinear_q_bytes(int64_t M, int64_t K) { return round_up(M * K, 256); }

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
        const int64_t g = plan_gemv(M, N, K).ws_bytes;
        int64_t gemm = g;
        int64_t bl = bitlinear_q_bytes(M, K) + round_up(M * 4, 256) + g;
        if (gemm > need) need = gemm;
        if (bl > need) need = bl;
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
    quant_act_kernel<<<(unsigned)M, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(x, K, q, K, false, s, rowsum);
    return launched();
}

BITNET_API int bitnet_w2a8_gemm(const int8_t *q, const uint8_t *packed, int32_t *y, int64_t M, int64_t N, int64_t K,
                                void *workspace, int64_t workspace_bytes, void *stream) {
    if (!sizes_ok(M, N, K)) return BITNET_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BITNET_OK;
    if (y == nullptr || (K > 0 && (q == nullptr || packed == nullptr))) return BITNET_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(y, 4)) return BITNET_ERR_ALIGNMENT;
    const int64_t need = K > 0 ? plan_gemv(M, N, K).ws_bytes : 0;
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return BITNET_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 256)) return BITNET_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        fill_kernel<int32_t><<<grid_for(M * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(y, M * N, 0);
        return launched();
    }
    return launch_gemv(dev, q, K, packed, M, N, K, y, nullptr, nullptr, nullptr, workspace, st);
}

BITNET_API int bitnet_bitlinear(const uint16_t *x, const uint8_t *packed, const float *gamma, uint16_t *y, int64_t M,
                                int64_t N, int64_t K, void *workspace, int64_t workspace_bytes, void *stream) {
    if (!sizes_ok(M, N, K)) return BITNET_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BITNET_OK;
    if (y == nullptr || gamma == nullptr || (K > 0 && (x == nullptr || packed == nullptr)))
        return BITNET_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(packed, 16) || !aligned(y, 2) || !aligned(gamma, 4)) return BITNET_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        int rc = device_info(&dev);
        if (rc != BITNET_OK) return rc;
        fill_kernel<uint16_t><<<grid_for(M * N, kThreads * 4, dev->sm_count), kThreads, 0, st>>>(y, M * N, 0);
        return launched();
    }
    const int64_t qb = bitlinear_q_bytes(M, K), sb = round_up(M * 4, 256);
    const int64_t gw = plan_gemv(M, N, K).ws_bytes;
    if (workspace == nullptr || workspace_bytes < qb + sb + gw) return BITNET_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BITNET_ERR_ALIGNMENT;
    int rc = device_info(&dev);
    if (rc != BITNET_OK) return rc;
    int8_t *q = static_cast<int8_t *>(workspace);
    float *s = reinterpret_cast<float *>(static_cast<char *>(workspace) + qb);
    void *rest = static_cast<char *>(workspace) + qb + sb;
    quant_act_kernel<<<(unsigned)M, kThreads, 0, st>>>(x, K, q, K, false, s, nullptr);
    if ((rc = launched()) != BITNET_OK) return rc;
    return launch_gemv(dev, q, K, packed, M, N, K, nullptr, y, s, gamma, rest, st);
}

BITNET_API int bitnet_get_device_error(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return BITNET_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
    }
    return v;
}

BITNET_API int64_t bitnet_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
