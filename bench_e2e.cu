// bench_e2e.cu -- the end-to-end leg of bench.py without Python in the loop.
//
// One step of the M = 1 GEMV sweep through the library's C ABI with host
// buffers: copy the shapes' int8 activations from pinned host memory to the
// device (one copy), call bitnet_w2a8_gemm for every shape, copy the int32
// results back to pinned host memory (one copy), synchronise the stream (the
// host holds every result).  The loop is timed with CUDA events on the
// stream, so the figure holds the copies, the library's host-side work per
// call (argument checks, plan, tensor-map lookup, launch) and the
// synchronisation, but no interpreter.
//
// Built by bench.py into bench_e2e.so (nvcc, static CUDA runtime) and called
// through ctypes; it reaches libbitnet_b200.so through dlopen of the path it
// is given, which returns the copy the process has already loaded.
#include <cuda_runtime.h>
#include <dlfcn.h>
#include <stdint.h>

typedef int (*gemm_fn)(const int8_t *, const uint8_t *, int32_t *, int64_t, int64_t, int64_t, void *, int64_t,
                       void *);

// h_q / d_q: all shapes' activations (q_bytes); d_qs: each shape's view of
// d_q.  packed: copies x n_shapes weight pointers.  d_ys: each shape's output,
// views of d_y (y_bytes), copied to h_y.  Returns the elapsed milliseconds of
// `steps` steps, or a negative value on failure (-1: library or symbol not
// found, -2: a CUDA call failed, -3: the library returned a non-zero status,
// stored in *status).
extern "C" double e2e_sweep_loop(const char *lib_path, int n_shapes, const int64_t *N, const int64_t *K,
                                 const void *h_q, void *d_q, int64_t q_bytes, void *const *d_qs, int copies,
                                 void *const *packed, void *const *d_ys, void *h_y, int64_t y_bytes,
                                 const void *d_y, void *const *ws, const int64_t *ws_bytes, int steps, void *stream,
                                 int *status) {
    void *h = dlopen(lib_path, RTLD_NOW | RTLD_NOLOAD);
    if (h == nullptr) h = dlopen(lib_path, RTLD_NOW);
    if (h == nullptr) return -1.0;
    gemm_fn gemm = reinterpret_cast<gemm_fn>(dlsym(h, "bitnet_w2a8_gemm"));
    if (gemm == nullptr) return -1.0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return -2.0;
    double ms = -2.0;
    *status = 0;
    if (cudaEventRecord(e0, st) != cudaSuccess) goto done;
    for (int s = 0; s < steps; ++s) {
        const int c = s % copies;
        if (cudaMemcpyAsync(d_q, h_q, (size_t)q_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) goto done;
        for (int j = 0; j < n_shapes; ++j) {
            const int rc = gemm(static_cast<const int8_t *>(d_qs[j]),
                                static_cast<const uint8_t *>(packed[(int64_t)c * n_shapes + j]),
                                static_cast<int32_t *>(d_ys[j]), 1, N[j], K[j], ws[j], ws_bytes[j], stream);
            if (rc != 0) {
                *status = rc;
                ms = -3.0;
                goto done;
            }
        }
        if (cudaMemcpyAsync(h_y, d_y, (size_t)y_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) goto done;
        if (cudaStreamSynchronize(st) != cudaSuccess) goto done;
    }
    if (cudaEventRecord(e1, st) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess) goto done;
    {
        float f = 0.0f;
        if (cudaEventElapsedTime(&f, e0, e1) == cudaSuccess) ms = f;
    }
done:
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    return ms;
}
