// selftest.cu -- device self-tests for helpers of the kernels and pipe-rate
// microbenchmarks (test and measurement support library
// libattn_sink_selftest.so; not part of the product ABI).
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

// Throughput of one instruction kind: 8 independent chains per thread, 4
// CTAs of 512 threads resident per SM (<= 32 registers).  which = 0: the
// MUFU ex2.approx the softmax uses; 1: the cvt.rn.bf16x2.f32 that packs P.
constexpr int kRateChains = 8, kRateIters = 256, kRateThreads = 512, kRateCtasPerSm = 4;
template <int WHICH>
__global__ void __launch_bounds__(kRateThreads, kRateCtasPerSm) pipe_rate_kernel(float *sink, long long *cycles)
{
    float x[kRateChains];
#pragma unroll
    for (int c = 0; c < kRateChains; ++c) x[c] = -0.001f * (float)(threadIdx.x + c);
    const long long t0 = clock64();
    for (int i = 0; i < kRateIters; ++i) {
#pragma unroll
        for (int c = 0; c < kRateChains; ++c) {
            if (WHICH == 0) {
                x[c] = attn_sink::ex2(-x[c]);  // stays in (0, 1]
            } else {
                uint32_t d;
                asm volatile("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(x[c]));
                x[c] = __uint_as_float(d & 0x3fff3fffu);  // keep the value finite
            }
        }
    }
    const long long t1 = clock64();
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < kRateChains; ++c) acc += x[c];
    sink[blockIdx.x * blockDim.x + threadIdx.x] = acc;
    if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

}  // namespace

// Measured results per clock per SM of instruction kind `which` (0: ex2.approx
// on MUFU, 1: cvt.rn.bf16x2.f32); synchronous; 0 on success.
extern "C" __attribute__((visibility("default"))) int attn_sink_selftest_pipe_rate(int which, double *per_clk_per_sm)
{
    if ((which != 0 && which != 1) || !per_clk_per_sm) return -1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return -6;
    const int blocks = sms * kRateCtasPerSm;
    float *sink = nullptr;
    long long *cyc = nullptr;
    if (cudaMalloc(&sink, (size_t)blocks * kRateThreads * sizeof(float)) != cudaSuccess) return -6;
    if (cudaMalloc(&cyc, (size_t)blocks * sizeof(long long)) != cudaSuccess) {
        cudaFree(sink);
        return -6;
    }
    int rc = 0;
    for (int rep = 0; rep < 2 && rc == 0; ++rep) {  // the first launch warms up
        if (which == 0)
            pipe_rate_kernel<0><<<blocks, kRateThreads>>>(sink, cyc);
        else
            pipe_rate_kernel<1><<<blocks, kRateThreads>>>(sink, cyc);
        if (cudaDeviceSynchronize() != cudaSuccess) rc = -6;
    }
    if (rc == 0) {
        long long *h = new long long[blocks];
        if (cudaMemcpy(h, cyc, (size_t)blocks * sizeof(long long), cudaMemcpyDeviceToHost) != cudaSuccess) {
            rc = -6;
        } else {
            double mean = 0.0;
            for (int b = 0; b < blocks; ++b) mean += (double)h[b];
            mean /= blocks;
            *per_clk_per_sm = mean > 0 ? (double)kRateCtasPerSm * kRateThreads * kRateChains * kRateIters / mean : 0.0;
        }
        delete[] h;
    }
    cudaFree(sink);
    cudaFree(cyc);
    cudaGetLastError();
    return rc;
}

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
