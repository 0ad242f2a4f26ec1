// ex2_rate.cu -- throughput of the exponential unit (ex2.approx.ftz.f32), for the attention
// kernel's exponential lower bound: exps per launch / (measured ex2 per second).
//
// Each thread runs kChains independent chains x <- 2^-x (a contraction with fixed point near
// 0.64, so the values stay finite), so every exponential waits only on its own chain and enough
// are in flight to keep the unit busy.  The host times a launch with CUDA events on its stream
// and divides blocks * threads * kChains * iters by the time.
#include <cuda_runtime.h>

namespace {

constexpr int kChains = 8;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) ex2_rate_kernel(float *out, int iters)
{
    float x[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c)
        x[c] = 0.25f + 0.001f * static_cast<float>((threadIdx.x + c) & 63);
#pragma unroll 1
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int c = 0; c < kChains; ++c) {
            float y;
            asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-x[c]));
            x[c] = y;
        }
    }
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kChains; ++c)
        s += x[c];
    out[blockIdx.x * kThreads + threadIdx.x] = s;
}

}  // namespace

// Launches `blocks` blocks of 256 threads, each thread computing 8 * iters exponentials, on
// `stream`; `out` (device, blocks * 256 floats) receives one sum per thread.  Returns the CUDA
// error code of the launch (0 on success).
extern "C" int rra_mb_ex2_launch(float *out, int blocks, int iters, void *stream)
{
    if (out == nullptr || blocks <= 0 || iters <= 0)
        return static_cast<int>(cudaErrorInvalidValue);
    ex2_rate_kernel<<<blocks, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(out, iters);
    return static_cast<int>(cudaGetLastError());
}

// Exponentials one launch computes per block and iteration (threads * chains).
extern "C" int rra_mb_ex2_per_block_iter(void) { return kThreads * kChains; }
