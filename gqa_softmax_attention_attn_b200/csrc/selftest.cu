// selftest.cu -- device self-tests for helpers of the kernels (test support
// library libattn_sink_selftest.so; not part of the product ABI).
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

// the helpers reference these two functions through kernels.h
namespace attn_sink {
unsigned *device_status_ptr() { return nullptr; }
long long wait_timeout_ns() { return 0; }
}  // namespace attn_sink

namespace {

// fast_exp2x2 (FMA pipe), ex2.approx (MUFU) and CUDA's exp2f on the same inputs
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

// One CTA waits (bounded) on an mbarrier that nothing ever arrives on: the
// wait must give up after `timeout_ns`, set the status bit and let the kernel
// return normally.  result[0] = 1 if the wait reported failure, result[1] = the
// abort flag it raised.
__global__ void timeout_kernel(unsigned *status, int *result, long long timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        attn_sink::mbar_init(&bar, 1);
        abort_flag = 0;
        attn_sink::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = attn_sink::mbar_wait(&bar, 0, &abort_flag, status, timeout_ns);
        result[0] = ok ? 0 : 1;
        result[1] = abort_flag;
    }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int attn_sink_selftest_exp2(const float *x, float *fast,
                                                                               float *mufu, float *ref, int n,
                                                                               void *stream)
{
    if (n <= 0 || (n & 1)) return -1;
    exp2_kernel<<<(n / 2 + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, fast, mufu, ref, n);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

extern "C" __attribute__((visibility("default"))) int attn_sink_selftest_timeout(unsigned *status, int *result,
                                                                                  long long timeout_ns, void *stream)
{
    timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, result, timeout_ns);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}
