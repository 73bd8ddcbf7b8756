// exp2_probe.cu -- test-only library: evaluates the library's device-side 2^x
// routines (the FMA-pipe polynomial exp2_poly2 and the MUFU ex2.approx wrapper)
// on an array, so that a test can compare them with float64 2^x. Built by the
// tests with the library's own nvcc flags; not part of the product.
#include <cstdint>

#include "ptx.cuh"

namespace {

__global__ void exp2_probe_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                  float* __restrict__ y_mufu, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        const float2 p = attn::exp2_poly2(make_float2(x[i], x[i + 1]));
        y_poly[i] = p.x;
        y_poly[i + 1] = p.y;
        y_mufu[i] = attn::ex2_approx(x[i]);
        y_mufu[i + 1] = attn::ex2_approx(x[i + 1]);
    } else if (i < n) {
        y_poly[i] = attn::exp2_poly2(make_float2(x[i], 0.f)).x;
        y_mufu[i] = attn::ex2_approx(x[i]);
    }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int exp2_probe(const float* x, float* y_poly,
                                                                 float* y_mufu, int n,
                                                                 void* stream) {
    if (n <= 0) return 0;
    const int threads = 256;
    const int blocks = (n / 2 + threads) / threads;
    exp2_probe_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_mufu, n);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}
