// mask.cu -- Threshold-l2 token selection, the step in front of the pack -> attend -> unpack
// pipeline ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers", aissential.tech
// summary, Summary: the DeiT models are pruned with Threshold-l2, EViT and other methods).
//
// One block per image.  Each thread scores whole tokens: the squared l2 norm of the token's
// embedding row, accumulated as fma(x_c, x_c, acc) in double over c = 0..C-1 (16-bit inputs
// widen exactly, so the score is one reproducible number), read as 16-byte vectors.  The
// scores go to shared memory as order-preserving integer keys (0 = not a candidate, 1 = NaN,
// otherwise the bits of the non-negative double plus 2).  A candidate's rank is then the number
// of candidates that beat it (higher key, or equal key and lower index); it is kept when that
// rank is below k_b.  Ranking by counting costs N^2 comparisons per image -- 39 K at N = 197,
// 1 M at N = 1024, spread over 256 threads -- and needs no sort and no synchronisation beyond
// one barrier.
#include <cuda_fp16.h>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int kMaskThreads = 256;

template <bool kBF16>
__device__ __forceinline__ double widen(uint32_t bits16)
{
    if constexpr (kBF16)
        return static_cast<double>(__uint_as_float(bits16 << 16));
    else
        return static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(bits16))));
}

template <bool kBF16>
__global__ void __launch_bounds__(kMaskThreads) l2_mask_kernel(const uint16_t *__restrict__ x, int N, int C,
                                                                const int32_t *__restrict__ k_keep, double thr_sq,
                                                                const uint8_t *prev, uint8_t *mask)
{
    extern __shared__ unsigned long long key[];  // [N]
    pdl_trigger();
    pdl_wait();  // the embeddings and the previous stage's mask may come from the previous kernel
    const int b = blockIdx.x;
    const int64_t row0 = static_cast<int64_t>(b) * N;
    for (int n = threadIdx.x; n < N; n += kMaskThreads) {
        const bool cand = n >= 1 && (prev == nullptr || prev[row0 + n] != 0);
        unsigned long long k = 0;
        if (cand) {
            const uint4 *row = reinterpret_cast<const uint4 *>(x + (row0 + n) * C);
            double acc = 0.0;
            for (int c8 = 0; c8 < C / 8; ++c8) {
                const uint4 w = __ldg(row + c8);
                const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double lo = widen<kBF16>(v[i] & 0xFFFFu), hi = widen<kBF16>(v[i] >> 16);
                    acc = __fma_rn(lo, lo, acc);  // element 2i, then 2i + 1: index order
                    acc = __fma_rn(hi, hi, acc);
                }
            }
            k = acc != acc ? 1ull : static_cast<unsigned long long>(__double_as_longlong(acc)) + 2ull;
        }
        key[n] = k;
    }
    __syncthreads();
    const int kb = k_keep != nullptr ? k_keep[b] : 0;
    for (int n = threadIdx.x; n < N; n += kMaskThreads) {
        const unsigned long long kn = key[n];
        uint8_t keep;
        if (n == 0) {
            keep = 1;  // CLS
        } else if (kn == 0) {
            keep = 0;  // not a candidate
        } else if (k_keep != nullptr) {
            int r = 0;
            for (int m = 1; m < N && r < kb; ++m) {
                const unsigned long long km = key[m];
                r += (km > kn || (km == kn && m < n)) ? 1 : 0;
            }
            keep = r < kb ? 1 : 0;
        } else {
            keep = (kn != 1 && __longlong_as_double(static_cast<long long>(kn - 2)) >= thr_sq) ? 1 : 0;
        }
        mask[row0 + n] = keep;
    }
}

}  // namespace

cudaError_t launch_l2_mask(const void *x, int B, int N, int C, bool bf16, const int32_t *k_keep, double thr_sq,
                           const uint8_t *prev, uint8_t *mask, cudaStream_t stream)
{
    if (B == 0)
        return cudaSuccess;
    const size_t smem = static_cast<size_t>(N) * sizeof(unsigned long long);
    const auto *xs = static_cast<const uint16_t *>(x);
    return bf16 ? launch_pdl(l2_mask_kernel<true>, dim3(B), dim3(kMaskThreads), smem, stream, xs, N, C, k_keep,
                             thr_sq, prev, mask)
                : launch_pdl(l2_mask_kernel<false>, dim3(B), dim3(kMaskThreads), smem, stream, xs, N, C, k_keep,
                             thr_sq, prev, mask);
}

}  // namespace rra
