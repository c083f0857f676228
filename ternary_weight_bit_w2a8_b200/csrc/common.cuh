// common.cuh -- shared helpers of the sm_100a kernels (device PTX wrappers,
// sizes of the packed layout, the per-device error word).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bitnet_b200.h"

namespace bitnet {

constexpr int kThreads = 256;  // threads per CTA of the streaming kernels

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Packed layout v1: K is padded to a multiple of 128, a row takes K_pad/4 bytes.
__host__ __device__ __forceinline__ int64_t k_pad(int64_t K) { return round_up(K, 128); }
__host__ __device__ __forceinline__ int64_t packed_row_bytes(int64_t K) { return k_pad(K) / 4; }

// Per-device error word: kernels that give up a bounded wait record
// BITNET_ERR_DEVICE_TIMEOUT here (read and cleared by bitnet_get_device_error).
__device__ int g_device_error;

__device__ __forceinline__ void record_device_error(int code) { atomicCAS(&g_device_error, 0, code); }

// 4-way byte dot product: unsigned bytes of a times signed bytes of b, plus c.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// 16-byte streaming load: read-only path, not kept in L1, 256-byte L2 prefetch.
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Asks the L2 to fetch [p, p + bytes) from HBM (16-byte aligned address and
// size); nothing is returned to the thread and no completion is tracked.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before its predecessor on the stream finishes;
// pdl_wait() blocks until that predecessor has completed and its writes are
// visible.  pdl_launch_dependents() lets the successor start early.  Both are
// no-ops for a normal launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
    return __uint_as_float(((uint32_t)h) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits_rn(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&b);
}

// Block-wide reductions over kThreads threads; `scratch` holds >= 32 words.
template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, Op op, T *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();  // scratch may still be read by a previous reduction
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    T r = scratch[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = op(r, scratch[w]);
    return r;
}

}  // namespace bitnet
