// selftest.cu -- device self-tests for helpers of the kernels (test support
// library libattn_sink_selftest.so; not part of the product ABI).
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

namespace {
__global__ void exp2_kernel(const float *x, float *fast, float *mufu, float *ref, int n)
{
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 >= n) return;
    const float2 f = attn_sink::fast_exp2x2(make_float2(x[i], x[i + 1]));
    fast[i] = f.x;
    fast[i + 1] = f.y;
    mufu[i] = attn_sink::ex2(x[i]);
    mufu[i + 1] = attn_sink::ex2(x[i + 1]);
    ref[i] = exp2f(x[i]);
    ref[i + 1] = exp2f(x[i + 1]);
}
}  // namespace

// the kernels reference these two functions through kernels.h
namespace attn_sink {
unsigned *device_status_ptr() { return nullptr; }
long long wait_timeout_ns() { return 0; }
}  // namespace attn_sink

extern "C" __attribute__((visibility("default"))) int attn_sink_selftest_exp2(const float *x, float *fast,
                                                                               float *mufu, float *ref, int n,
                                                                               void *stream)
{
    if (n <= 0 || (n & 1)) return -1;
    exp2_kernel<<<(n / 2 + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, fast, mufu, ref, n);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}
