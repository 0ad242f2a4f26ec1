// mask.cu -- Threshold-l2 token selection, the step in front of the pack -> attend -> unpack
// pipeline ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers", aissential.tech
// summary, Summary: the DeiT models are pruned with Threshold-l2, EViT and other methods).
//
// One block per image.  The image's embeddings pass through shared memory in column chunks
// (16-byte cp.async, coalesced along each token's row, double-buffered), and each thread extends
// the squared-norm chain of its tokens chunk by chunk: acc = fmaf(x_c, x_c, acc) in single
// precision over c = 0..C-1 in index order (16-bit inputs widen exactly and their squares are
// exact, so the score is one reproducible number).  The scores go to shared memory as
// order-preserving integer keys (0 = not a candidate, 1 = NaN, otherwise the bits of the
// non-negative float plus 2).  A candidate's rank
// is the number of candidates that beat it (higher key, or equal key and lower index); it is
// kept when that rank is below k_b.  Ranking by counting costs N^2 comparisons per image -- 39 K
// at N = 197, 1 M at N = 1024, spread over 256 threads -- and needs no sort.
#include <cuda_fp16.h>

#include <atomic>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int kMaskThreads = 256;

template <bool kBF16>
__device__ __forceinline__ float widen(uint32_t bits16)
{
    if constexpr (kBF16)
        return __uint_as_float(bits16 << 16);
    else
        return __half2float(__ushort_as_half(static_cast<unsigned short>(bits16)));
}

// Shared memory: the keys [N] (8 bytes each), then two staging buffers of N token rows, each row
// `w` embedding columns (w * 2 bytes), padded by 16 bytes when w >= 16 so that the 16-byte reads
// of consecutive tokens fall in different banks.
constexpr int kMaxTokPerThread = kMaskMaxN / kMaskThreads;

__host__ __device__ constexpr int staging_stride(int w) { return w * 2 + (w >= 16 ? 16 : 0); }

template <bool kBF16>
__global__ void __launch_bounds__(kMaskThreads) l2_mask_kernel(const uint16_t *__restrict__ x, int N, int C, int w,
                                                                const int32_t *__restrict__ k_keep, double thr_sq,
                                                                const uint8_t *prev, uint8_t *mask)
{
    extern __shared__ __align__(16) uint8_t sm[];
    unsigned long long *key = reinterpret_cast<unsigned long long *>(sm);
    const int stride = staging_stride(w);
    uint8_t *buf0 = sm + ((static_cast<size_t>(N) * 8 + 15) & ~static_cast<size_t>(15));
    uint8_t *buf1 = buf0 + static_cast<size_t>(N) * stride;
    pdl_trigger();
    pdl_wait();  // the embeddings and the previous stage's mask may come from the previous kernel
    const int b = blockIdx.x;
    const int64_t row0 = static_cast<int64_t>(b) * N;
    const int tid = threadIdx.x;

    // the image's embedding columns [c0, c0 + wj) into a staging buffer, 16 bytes per cp.async
    auto stage = [&](int c0, uint8_t *dst) {
        const int wj = min(w, C - c0);
        const int parts = wj / 8;
        const uint32_t d0 = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
        for (int i = tid; i < N * parts; i += kMaskThreads) {
            const int n = i / parts, q = i - n * parts;
            const uint16_t *src = x + (row0 + n) * C + c0 + q * 8;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d0 + n * stride + q * 16), "l"(src)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    // squared norms: each thread continues the fma chain of its tokens chunk by chunk, columns in
    // index order, so the result is the one sequential accumulation the definition names
    float acc[kMaxTokPerThread];
#pragma unroll
    for (int t = 0; t < kMaxTokPerThread; ++t)
        acc[t] = 0.0f;
    const int nchunks = (C + w - 1) / w;
    stage(0, buf0);
    for (int j = 0; j < nchunks; ++j) {
        if (j + 1 < nchunks)
            stage((j + 1) * w, (j & 1) ? buf0 : buf1);
        else
            asm volatile("cp.async.commit_group;" ::: "memory");  // keep the group count uniform
        asm volatile("cp.async.wait_group 1;" ::: "memory");      // this thread's copies of chunk j
        __syncthreads();                                          // everyone's copies of chunk j
        const uint8_t *cur = (j & 1) ? buf1 : buf0;
        const int wj = min(w, C - j * w);
#pragma unroll
        for (int t = 0; t < kMaxTokPerThread; ++t) {
            const int n = tid + t * kMaskThreads;
            if (n < N) {
                const uint4 *row = reinterpret_cast<const uint4 *>(cur + n * stride);
                float a = acc[t];
                for (int q = 0; q < wj / 8; ++q) {
                    const uint4 v4 = row[q];
                    const uint32_t v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float lo = widen<kBF16>(v[i] & 0xFFFFu), hi = widen<kBF16>(v[i] >> 16);
                        a = __fmaf_rn(lo, lo, a);  // element 2i, then 2i + 1: index order
                        a = __fmaf_rn(hi, hi, a);
                    }
                }
                acc[t] = a;
            }
        }
        __syncthreads();  // the buffer is refilled two chunks later
    }
#pragma unroll
    for (int t = 0; t < kMaxTokPerThread; ++t) {
        const int n = tid + t * kMaskThreads;
        if (n < N) {
            const bool cand = n >= 1 && (prev == nullptr || prev[row0 + n] != 0);
            const float a = acc[t];
            key[n] = !cand ? 0ull : (a != a ? 1ull : static_cast<unsigned long long>(__float_as_uint(a)) + 2ull);
        }
    }
    __syncthreads();
    const int kb = k_keep != nullptr ? k_keep[b] : 0;
    for (int n = tid; n < N; n += kMaskThreads) {
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
            keep = (kn != 1 && static_cast<double>(__uint_as_float(static_cast<uint32_t>(kn - 2))) >= thr_sq) ? 1 : 0;
        }
        mask[row0 + n] = keep;
    }
}

// Staging width: the widest of 64, 32, 16 columns whose two buffers fit in 128 KB, else 8 (two
// unpadded 16-byte rows per token: 128 KB at the largest N).
int staging_width(int N)
{
    for (int w = 64; w > 8; w /= 2)
        if (2 * static_cast<int64_t>(N) * staging_stride(w) <= 128 * 1024)
            return w;
    return 8;
}

size_t mask_smem_bytes(int N, int w)
{
    return ((static_cast<size_t>(N) * 8 + 15) & ~static_cast<size_t>(15)) +
           2 * static_cast<size_t>(N) * static_cast<size_t>(staging_stride(w));
}
static_assert(((kMaskMaxN * 8 + 15) & ~15) + 2 * kMaskMaxN * staging_stride(8) <= 227 * 1024,
              "staging buffers exceed shared memory at the largest N");

template <bool kBF16>
cudaError_t set_mask_smem(size_t bytes)
{
    static std::atomic<size_t> done{0};
    if (done.load(std::memory_order_relaxed) >= bytes)
        return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(l2_mask_kernel<kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e == cudaSuccess)
        done.store(bytes, std::memory_order_relaxed);
    return e;
}

}  // namespace

cudaError_t launch_l2_mask(const void *x, int B, int N, int C, bool bf16, const int32_t *k_keep, double thr_sq,
                           const uint8_t *prev, uint8_t *mask, cudaStream_t stream)
{
    if (B == 0)
        return cudaSuccess;
    const int w = staging_width(N);
    const size_t smem = mask_smem_bytes(N, w);
    const cudaError_t e = bf16 ? set_mask_smem<true>(smem) : set_mask_smem<false>(smem);
    if (e != cudaSuccess)
        return e;
    const auto *xs = static_cast<const uint16_t *>(x);
    return bf16 ? launch_pdl(l2_mask_kernel<true>, dim3(B), dim3(kMaskThreads), smem, stream, xs, N, C, w, k_keep,
                             thr_sq, prev, mask)
                : launch_pdl(l2_mask_kernel<false>, dim3(B), dim3(kMaskThreads), smem, stream, xs, N, C, w, k_keep,
                             thr_sq, prev, mask);
}

}  // namespace rra
