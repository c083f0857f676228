/*
 * bitnet_b200.h -- C ABI of libbitnet_b200.so: the BitNet b1.58 W2A8 BitLinear
 * hot path (ternary weights packed 2 bits each x per-token int8 activations,
 * exact int32 accumulation, bf16 rescale) for NVIDIA B200 (sm_100a).
 *
 * Pages cited (title, address):
 *   [WIN]  "Windows 上跑通 BitNet b1.58：Flash Attention 与 CUDA sm_86 部署实录"
 *          (hmyw.cn/news/146226)
 *   [CPU]  "微软BitNet：1-bit量化大模型CPU部署实践" (m.mzlw.cn/news/189456)
 *   [GEMV] "如何编译 BitNet W2A8 CUDA 内核并用 test.py 运行 GEMV 加速测试？"
 *          (pwwt.cn/news/4591536)
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Pointers named as device pointers must point to memory of the current
 *    CUDA device; the caller owns all memory.  No entry point allocates device
 *    memory; scratch space is the caller-provided `workspace`, sized with
 *    bitnet_workspace_bytes().
 *  - Matrices are row-major with the last index contiguous: weights W[N, K]
 *    (N = output features, K = input features, as a linear layer stores them),
 *    activations x[M, K], outputs y[M, N].  The product is y = x * W^T.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *    is asynchronous on that stream and does no host synchronisation, except
 *    bitnet_get_device_error().
 *  - Return value: BITNET_OK, or an error code.  Argument, alignment and
 *    workspace errors are detected on the host before anything is launched
 *    (nothing is written).  BITNET_ERR_CUDA reports a launch failure.  No
 *    entry point prints, aborts or traps.
 *  - Sizes: 0 <= M, N and 0 <= K <= BITNET_MAX_K.  M == 0 or N == 0 is a no-op;
 *    K == 0 yields an all-zero product.
 */
#ifndef BITNET_B200_H
#define BITNET_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

enum {
    BITNET_OK = 0,
    BITNET_ERR_INVALID_ARG = 1,    /* null pointer, negative or too large size */
    BITNET_ERR_ALIGNMENT = 2,      /* a pointer misses its required alignment */
    BITNET_ERR_WORKSPACE = 3,      /* workspace missing or smaller than required */
    BITNET_ERR_CUDA = 4,           /* a CUDA runtime call or kernel launch failed */
    BITNET_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up a bounded wait (see below) */
    BITNET_ERR_UNSUPPORTED = 6     /* device is not sm_100 class */
};

/* Largest K accepted: keeps every int32 partial sum of the kernels exact. */
#define BITNET_MAX_K 2097152

/* Version of the packed weight layout written by bitnet_pack_weights. */
#define BITNET_LAYOUT_VERSION 1

/* Human-readable name of a status code (static string, never NULL). */
BITNET_API const char *bitnet_status_string(int status);

/* BITNET_LAYOUT_VERSION of this library. */
BITNET_API int bitnet_layout_version(void);

/*
 * Bytes of the packed weight buffer for an N x K ternary matrix, or -1 for
 * invalid sizes.  Packed layout version 1 (2-bit codes per [CPU] §2.1:
 * -1 -> 00, 0 -> 01, +1 -> 10; four values per byte per [CPU] §2.2):
 *   K_pad = 128 * ceil(K / 128); each row n occupies K_pad/4 bytes at offset
 *   n * K_pad/4; value k of the row sits in byte 4*floor(k/16) + (k mod 4) at
 *   bits 2*floor((k mod 16)/4); padding (K <= k < K_pad) holds code 01.
 * So each little-endian 32-bit word covers 16 consecutive k, and
 * (word >> 2j) & 0x03030303 holds the codes of k = 16i+4j .. 16i+4j+3, one per
 * byte, aligned with four consecutive int8 activations.
 * The result is N * K_pad / 4; the buffer is a plain byte array the caller
 * may save and reload as long as bitnet_layout_version() matches.
 */
BITNET_API int64_t bitnet_packed_bytes(int64_t N, int64_t K);

/*
 * Workspace bytes that bitnet_w2a8_gemm / bitnet_bitlinear / bitnet_absmean
 * need for an M x N x K problem (the maximum over the three), or -1 for
 * invalid sizes.  Depends only on (M, N, K).  0 means no workspace is needed.
 */
BITNET_API int64_t bitnet_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * Absmean weight scale ([WIN] §3.1; [CPU] §6.3): gamma = mean over the whole
 * matrix of |W[n,k]|, summed in fp64 and rounded once to fp32 (0 for an empty
 * matrix).  The summation order is fixed for a given (N, K), so the result is
 * deterministic; it may differ from a sequential sum in the last fp32 ulp.
 *   W         device, bf16 bit patterns [N, K], 2-byte aligned
 *   gamma     device, 1 float (output)
 *   workspace device, >= bitnet_workspace_bytes(0, N, K) bytes, 256-byte aligned
 */
BITNET_API int bitnet_absmean(const uint16_t *W, int64_t N, int64_t K, float *gamma,
                              void *workspace, int64_t workspace_bytes, void *stream);

/*
 * Ternarisation with a given scale ([WIN] §3.1; [CPU] §6.3):
 *   W_t[n,k] = clamp(rne(W[n,k] / gamma), -1, 1), fp32 IEEE division, round to
 *   nearest even; gamma <= 0 (or NaN) gives all zeros, a NaN ratio gives 0.
 *   W     device, bf16 bit patterns [N, K]
 *   gamma device, 1 float (e.g. written by bitnet_absmean)
 *   W_t   device, int8 [N, K] (output)
 */
BITNET_API int bitnet_ternarize(const uint16_t *W, int64_t N, int64_t K, const float *gamma,
                                int8_t *W_t, void *stream);

/*
 * Packs ternary weights into layout version 1 (see bitnet_packed_bytes).
 *   W_t           device, int8 [N, K], values in {-1, 0, 1}
 *   packed        device, bitnet_packed_bytes(N, K) bytes, 16-byte aligned (output)
 *   invalid_count device, 1 int32 or NULL: receives the number of W_t values
 *                 outside {-1, 0, 1}; such values are stored as 0 (code 01)
 */
BITNET_API int bitnet_pack_weights(const int8_t *W_t, int64_t N, int64_t K, uint8_t *packed,
                                   int32_t *invalid_count, void *stream);

/*
 * Per-token absmax int8 activation quantisation ([GEMV] opening paragraph:
 * W2A8 = 2-bit weights x 8-bit activations; the formula is this library's
 * reading, the pages give none):
 *   amax_m = max_k |x[m,k]|, s[m] = 127 / max(amax_m, 1e-5)   (fp32)
 *   q[m,k] = clamp(rne(x[m,k] * s[m]), -128, 127)            (fp32 multiply)
 *   rowsum[m] = sum_k q[m,k]
 *   x      device, bf16 bit patterns [M, K], 2-byte aligned
 *   q      device, int8 [M, K] (output)
 *   s      device, float [M] (output)
 *   rowsum device, int32 [M] or NULL (output)
 */
BITNET_API int bitnet_quant_act(const uint16_t *x, int64_t M, int64_t K, int8_t *q, float *s,
                                int32_t *rowsum, void *stream);

/*
 * The W2A8 contraction ([GEMV] sections on test.py: an int32 matrix product of
 * int8 activations with the ternary weights, equal element by element to an
 * integer matmul):
 *   y[m,n] = sum_k q[m,k] * W_t[n,k]    exact in int32.
 * Paths: M <= 16 with K >= 512 runs the TMA-staged GEMV, one pass over the
 * weights for all M tokens; M >= 2 otherwise (K >= 128) runs the persistent
 * tcgen05 tensor-core GEMM; what remains (M == 1 with K < 512, or K < 128)
 * runs the register-streaming GEMV.  All give the same exact result.
 *   q         device, int8 [M, K], any alignment
 *   packed    device, layout version 1, 16-byte aligned
 *   y         device, int32 [M, N], 4-byte aligned (output)
 *   workspace device, >= bitnet_workspace_bytes(M, N, K) bytes, 256-byte aligned
 *             (may be NULL when that size is 0)
 */
BITNET_API int bitnet_w2a8_gemm(const int8_t *q, const uint8_t *packed, int32_t *y, int64_t M,
                                int64_t N, int64_t K, void *workspace, int64_t workspace_bytes,
                                void *stream);

/*
 * Full BitLinear forward ([WIN] §3.1: output = (ternary product) * scale):
 *   q, s = bitnet_quant_act(x);  acc = bitnet_w2a8_gemm(q, packed);
 *   y[m,n] = bf16_rne( (float)acc[m,n] * (gamma / s[m]) )   (fp32 arithmetic)
 *   x         device, bf16 bit patterns [M, K], 2-byte aligned
 *   packed    device, layout version 1, 16-byte aligned
 *   gamma     device, 1 float: the absmean weight scale
 *   y         device, bf16 bit patterns [M, N], 2-byte aligned (output)
 *   workspace device, >= bitnet_workspace_bytes(M, N, K) bytes, 256-byte aligned
 */
BITNET_API int bitnet_bitlinear(const uint16_t *x, const uint8_t *packed, const float *gamma,
                                uint16_t *y, int64_t M, int64_t N, int64_t K, void *workspace,
                                int64_t workspace_bytes, void *stream);

/*
 * Allocation-free variant of bitnet_w2a8_gemm.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory --
 * for instance a host program that only receives device buffers from another
 * framework and has no device allocator of its own, or a service whose device
 * memory is fixed up front -- and so cannot provide the workspace that
 * bitnet_w2a8_gemm may need.  Instead it uses one scratch array of
 * BITNET_NOALLOC_SCRATCH_BYTES compiled into this library as a file-scope
 * __device__ array, which every GPU that loads the library holds until the
 * process exits.
 *   Same arguments, layouts, result and errors as bitnet_w2a8_gemm, without
 *   the workspace.  Returns BITNET_ERR_WORKSPACE (before any device work) when
 *   the problem needs more scratch than BITNET_NOALLOC_SCRATCH_BYTES; many
 *   shapes need none (bitnet_workspace_bytes(M, N, K) <= 8192 means the
 *   contraction itself needs none).
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.
 *   All calls share the one array and it keeps the contents of the last call;
 *   every call writes the scratch it reads, so nothing has to be cleared, but
 *   calls that overlap on the GPU (other streams, other threads) race on it
 *   and must be serialised by the caller.
 *   No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define BITNET_NOALLOC_SCRATCH_BYTES 1048576
BITNET_API int bitnet_w2a8_gemm_noalloc(const int8_t *q, const uint8_t *packed, int32_t *y, int64_t M,
                                        int64_t N, int64_t K, void *stream);

/*
 * Device-side error word.  Kernels whose threads wait on one another bound
 * every wait; a wait that runs out records BITNET_ERR_DEVICE_TIMEOUT in a
 * per-device word (the kernel then stops and leaves its output incomplete).
 * This call synchronises `stream`, returns the recorded status of the current
 * device (BITNET_OK if none) and clears it.
 */
BITNET_API int bitnet_get_device_error(void *stream);

/* Number of kernels this library has launched in this process (all devices). */
BITNET_API int64_t bitnet_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_H */
