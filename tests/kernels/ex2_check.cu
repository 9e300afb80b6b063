// Test harness for the FMA-pipe 2^x (ex2_fma2 in ptx.cuh): evaluates it on a host
// array of arguments so a test can compare it with 2^x in double precision. Built by
// the test itself with nvcc; not part of the library.
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace {
__global__ void ex2_fma2_kernel(const float* x, float* y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        attn::ex2_fma2(x[i], x[i + 1], y[i], y[i + 1]);
    } else if (i < n) {
        float dummy;
        attn::ex2_fma2(x[i], 0.f, y[i], dummy);
    }
}
}  // namespace

// y[i] = ex2_fma2(x[i]) for i < n; host pointers; returns a cudaError_t value.
extern "C" int ex2_fma2_eval(const float* x_host, float* y_host, int n) {
    if (n <= 0) return 0;
    float *x = nullptr, *y = nullptr;
    const size_t bytes = sizeof(float) * static_cast<size_t>(n);
    cudaError_t e = cudaMalloc(&x, bytes);
    if (e == cudaSuccess) e = cudaMalloc(&y, bytes);
    if (e == cudaSuccess) e = cudaMemcpy(x, x_host, bytes, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
        const int pairs = (n + 1) / 2;
        ex2_fma2_kernel<<<(pairs + 255) / 256, 256>>>(x, y, n);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpy(y_host, y, bytes, cudaMemcpyDeviceToHost);
    cudaFree(x);
    cudaFree(y);
    return static_cast<int>(e);
}
