// pack_unpack.cu -- the token packer and unpacker around the ragged attention
// ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers": aissential.tech summary,
// Method -- a two-phase packer, index computation then gather; sota2.com card, Abstract -- the
// pack-attend-unpack pipeline back to the padded layout).
//
// Both kernels are HBM-bound row movers.  A block owns up to 256 padded rows of one image
// (grid = splits x images) and derives everything it needs from the keep mask in one pass:
//   * pack: the packed start of its image (nonzero mask bytes of images < b), the rank of its
//     first row inside the image, and the image length, counted together from 16-byte mask
//     chunks and reduced once -- so no second launch and no inter-block wait is needed; this
//     reads B^2 N / 2 mask bytes over the grid, so from 1025 images on a one-block launch writes
//     cu_seqlens first and the gather blocks read their image's start from it;
//   * both: the slot of every kept row of its range (warp ballots + one block prefix).
// Rows then move as 16-byte vectors, one warp per row, every load of a row (all tensors) in
// flight before its stores.
#include <type_traits>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kChunkBatch = 4;  // 16-byte mask chunks in flight per thread

struct SrcPtrs { const uint8_t *p[3]; };
struct DstPtrs { uint8_t *p[3]; };

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Bit k of the result is set iff byte k of the 16-byte chunk is nonzero.
__device__ __forceinline__ uint32_t kept_bits16(uint4 c)
{
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t t = (((w[i] & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w[i]) & 0x80808080u;
        const uint32_t nib = ((t >> 7) & 1u) | ((t >> 14) & 2u) | ((t >> 21) & 4u) | ((t >> 28) & 8u);
        m |= nib << (4 * i);
    }
    return m;
}

// Bits k (0..15) with lo <= s + k < hi.
__device__ __forceinline__ uint32_t range_bits16(int64_t s, int64_t lo, int64_t hi)
{
    const int64_t a = lo - s, b = hi - s;
    const int l = a < 0 ? 0 : (a > 16 ? 16 : static_cast<int>(a));
    const int h = b < 0 ? 0 : (b > 16 ? 16 : static_cast<int>(b));
    return h > l ? (((1u << h) - 1u) & ~((1u << l) - 1u)) : 0u;
}

// Per-thread counts of nonzero mask bytes (byte indices relative to `mask`) in [0, r0),
// [r0, r1) and [r0, r2), r0 <= r1 <= r2, read as 16-byte-aligned chunks.  Bytes outside
// [0, r2) are ignored; an aligned 16-byte chunk never crosses a page, so reading the whole
// chunk around either end of the range cannot fault.
struct Counts { int before, upto, total; };

__device__ __forceinline__ Counts count_ranges(const uint8_t *mask, int64_t r0, int64_t r1, int64_t r2)
{
    const uintptr_t addr = reinterpret_cast<uintptr_t>(mask);
    const int off = static_cast<int>(addr & 15u);
    const uint4 *base = reinterpret_cast<const uint4 *>(addr - off);
    const int64_t nchunks = (off + r2 + 15) >> 4;
    Counts c{0, 0, 0};
    for (int64_t j0 = threadIdx.x; j0 < nchunks; j0 += static_cast<int64_t>(kThreads) * kChunkBatch) {
        uint4 v[kChunkBatch];
#pragma unroll
        for (int u = 0; u < kChunkBatch; ++u) {
            const int64_t j = j0 + static_cast<int64_t>(u) * kThreads;
            v[u] = j < nchunks ? __ldg(base + j) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kChunkBatch; ++u) {
            const int64_t s = (j0 + static_cast<int64_t>(u) * kThreads) * 16 - off;
            const uint32_t m = kept_bits16(v[u]) & range_bits16(s, 0, r2);
            c.before += __popc(m & range_bits16(s, 0, r0));
            c.upto += __popc(m & range_bits16(s, r0, r1));
            c.total += __popc(m & range_bits16(s, r0, r2));
        }
    }
    return c;
}

struct BlockScan {
    int before, upto, total;  // block-wide sums of Counts
    int nk;                   // kept rows in the block's range
};

// One barrier round: reduces the three counts and prefixes the kept flags of rows [n0, n1)
// (one row per thread).  slot_of[i] = slot of row n0+i among the kept rows of the range, or
// -1; n_of_slot[slot] = i.
__device__ __forceinline__ BlockScan block_scan(Counts c, const uint8_t *row, int n0, int n1, int16_t *slot_of,
                                                int16_t *n_of_slot, int (*part)[4])
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = n0 + static_cast<int>(threadIdx.x);
    const bool keep = n < n1 && row[n] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    c.before = __reduce_add_sync(0xffffffffu, c.before);
    c.upto = __reduce_add_sync(0xffffffffu, c.upto);
    c.total = __reduce_add_sync(0xffffffffu, c.total);
    if (lane == 0) {
        part[warp][0] = c.before;
        part[warp][1] = c.upto;
        part[warp][2] = c.total;
        part[warp][3] = __popc(bal);
    }
    __syncthreads();
    BlockScan r{0, 0, 0, 0};
    int warp_base = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        r.before += part[w][0];
        r.upto += part[w][1];
        r.total += part[w][2];
        warp_base += (w < warp) ? part[w][3] : 0;
        r.nk += part[w][3];
    }
    if (n < n1) {
        const int slot = keep ? warp_base + __popc(bal & ((1u << lane) - 1u)) : -1;
        slot_of[threadIdx.x] = static_cast<int16_t>(slot);
        if (keep)
            n_of_slot[slot] = static_cast<int16_t>(threadIdx.x);
    }
    __syncthreads();
    return r;
}

// cu_seqlens of the whole batch from one block of 1024 threads: thread t counts image base + t
// from 16-byte mask chunks, then one block scan per 1024 images.  rra_pack launches it first
// for large batches, so that its gather blocks read their image's start from cu_seqlens instead of
// counting the mask bytes of every earlier image (B^2 N / 2 bytes in all).
constexpr int kScanThreads = 1024;
constexpr int kPackScanMinBatch = 1025;  // batches from this size on take the two-launch form

__global__ void __launch_bounds__(kScanThreads) cu_kernel(const uint8_t *__restrict__ mask, int B, int N,
                                                          int64_t capacity, int32_t *__restrict__ cu, int32_t *err)
{
    __shared__ int warp_tot[kScanThreads / 32];
    pdl_trigger();
    pdl_wait();  // the mask may come from the previous kernel
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(mask);
    const int off = static_cast<int>(addr & 15u);
    const uint4 *base = reinterpret_cast<const uint4 *>(addr - off);
    int64_t carry = 0;
    for (int b0 = 0; b0 < B; b0 += kScanThreads) {
        const int b = b0 + static_cast<int>(threadIdx.x);
        int cnt = 0;
        if (b < B) {
            const int64_t lo = static_cast<int64_t>(b) * N, hi = lo + N;
            for (int64_t j = (off + lo) >> 4; j < (off + hi + 15) >> 4; ++j)
                cnt += __popc(kept_bits16(__ldg(base + j)) & range_bits16(j * 16 - off, lo, hi));
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += t;
        }
        if (lane == 31)
            warp_tot[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < kScanThreads / 32; ++w) {
            before += (w < warp) ? warp_tot[w] : 0;
            total += warp_tot[w];
        }
        if (b < B)
            cu[b + 1] = static_cast<int32_t>(carry + before + incl);
        carry += total;
        __syncthreads();  // warp_tot is rewritten by the next round
    }
    if (threadIdx.x == 0) {
        cu[0] = 0;
        if (carry > capacity)
            raise_error(err, RRA_ERR_CAPACITY);
    }
}

template <int VPL, bool kFromCu>
__global__ void __launch_bounds__(kThreads) pack_kernel(const uint8_t *__restrict__ mask, int N, int rows_per_split,
                                                        int V, int n_tensors, SrcPtrs src, DstPtrs dst,
                                                        int64_t capacity, int32_t *__restrict__ cu, int32_t *err)
{
    __shared__ int part[kWarps][4];
    __shared__ int16_t slot_of[kThreads];
    __shared__ int16_t n_of_slot[kThreads];

    pdl_trigger();
    const int b = blockIdx.y;
    const int n0 = blockIdx.x * rows_per_split;
    if (n0 >= N)
        return;
    const int n1 = min(N, n0 + rows_per_split);
    const int64_t img0 = static_cast<int64_t>(b) * N;
    pdl_wait();  // the mask and the padded tensors may come from the previous kernel

    // Phase 1: image start, rank of row n0 inside the image, image length -- one pass (the image
    // start read from cu_seqlens instead when the previous launch has written it).
    const Counts c = kFromCu ? count_ranges(mask + img0, 0, n0, N) : count_ranges(mask, img0, img0 + n0, img0 + N);
    const BlockScan s = block_scan(c, mask + img0, n0, n1, slot_of, n_of_slot, part);
    const int64_t image_start = kFromCu ? static_cast<int64_t>(cu[b]) : static_cast<int64_t>(s.before);
    if (!kFromCu && blockIdx.x == 0 && threadIdx.x == 0) {
        if (b == 0)
            cu[0] = 0;
        cu[b + 1] = static_cast<int32_t>(image_start + s.total);
        if (image_start + s.total > capacity)
            raise_error(err, RRA_ERR_CAPACITY);
    }

    // Phase 2: one warp per kept row, all tensors' vectors loaded before any store.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t out0 = image_start + s.upto;
    for (int slot = warp; slot < s.nk; slot += kWarps) {
        const int64_t out_row = out0 + slot;
        if (out_row >= capacity)
            break;
        const int64_t in_row = img0 + n0 + n_of_slot[slot];
        uint4 buf[3][VPL];
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            if (t < n_tensors) {
                const uint4 *sp =
                    reinterpret_cast<const uint4 *>(t == 0 ? src.p[0] : (t == 1 ? src.p[1] : src.p[2])) + in_row * V;
#pragma unroll
                for (int k = 0; k < VPL; ++k)
                    if (lane + 32 * k < V)
                        buf[t][k] = ld_stream(sp + lane + 32 * k);
            }
        }
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            if (t < n_tensors) {
                uint4 *dp = reinterpret_cast<uint4 *>(t == 0 ? dst.p[0] : (t == 1 ? dst.p[1] : dst.p[2])) + out_row * V;
#pragma unroll
                for (int k = 0; k < VPL; ++k)
                    if (lane + 32 * k < V)
                        dp[lane + 32 * k] = buf[t][k];
            }
        }
    }
}

template <int VPL>
__global__ void __launch_bounds__(kThreads) unpack_kernel(const uint8_t *__restrict__ packed,
                                                          const int32_t *__restrict__ cu,
                                                          const uint8_t *__restrict__ mask, int N, int rows_per_split,
                                                          int V, int fill_mode, int64_t capacity,
                                                          uint8_t *__restrict__ dst, int32_t *err)
{
    __shared__ int part[kWarps][4];
    __shared__ int16_t slot_of[kThreads];
    __shared__ int16_t n_of_slot[kThreads];

    pdl_trigger();
    const int b = blockIdx.y;
    const int n0 = blockIdx.x * rows_per_split;
    if (n0 >= N)
        return;
    const int n1 = min(N, n0 + rows_per_split);
    const int64_t img0 = static_cast<int64_t>(b) * N;
    pdl_wait();  // cu_seqlens and the packed rows come from the previous kernels
    const int64_t start = cu[b];
    const int64_t end = cu[b + 1];

    const Counts c = count_ranges(mask + img0, 0, n0, N);
    const BlockScan s = block_scan(c, mask + img0, n0, n1, slot_of, n_of_slot, part);
    const bool image_ok = start >= 0 && end >= start;
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        if (!image_ok || s.total != end - start)
            raise_error(err, RRA_ERR_BAD_SEQLENS);
        else if (end > capacity)
            raise_error(err, RRA_ERR_CAPACITY);
    }
    // kept rows read packed rows [start, lim) only; a malformed image reads nothing
    const int64_t lim = image_ok ? min(end, capacity) : start;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = warp; i < n1 - n0; i += kWarps) {
        const int slot = slot_of[i];
        uint4 *dp = reinterpret_cast<uint4 *>(dst) + (img0 + n0 + i) * V;
        if (slot >= 0) {
            const int64_t in_row = start + s.upto + slot;
            if (in_row < start || in_row >= lim)
                continue;
            const uint4 *sp = reinterpret_cast<const uint4 *>(packed) + in_row * V;
            uint4 buf[VPL];
#pragma unroll
            for (int k = 0; k < VPL; ++k)
                if (lane + 32 * k < V)
                    buf[k] = ld_stream(sp + lane + 32 * k);
#pragma unroll
            for (int k = 0; k < VPL; ++k)
                if (lane + 32 * k < V)
                    dp[lane + 32 * k] = buf[k];
        } else if (fill_mode == 0) {
#pragma unroll
            for (int k = 0; k < VPL; ++k)
                if (lane + 32 * k < V)
                    dp[lane + 32 * k] = make_uint4(0, 0, 0, 0);
        }
    }
}

int choose_splits(int B, int N, int num_sms)
{
    const int target_blocks = 4 * num_sms;
    int splits = (target_blocks + B - 1) / (B > 0 ? B : 1);
    const int max_splits = (N + 15) / 16;  // at least 16 padded rows per block
    if (splits > max_splits)
        splits = max_splits;
    const int min_splits = (N + kThreads - 1) / kThreads;  // at most one row per thread
    if (splits < min_splits)
        splits = min_splits;
    return splits < 1 ? 1 : splits;
}

template <typename F>
cudaError_t dispatch_vpl(int V, F &&launch)
{
    switch ((V + 31) / 32) {
    case 1: return launch(std::integral_constant<int, 1>{});
    case 2: return launch(std::integral_constant<int, 2>{});
    case 3: return launch(std::integral_constant<int, 3>{});
    case 4: return launch(std::integral_constant<int, 4>{});
    case 5:
    case 6: return launch(std::integral_constant<int, 6>{});
    case 7:
    case 8: return launch(std::integral_constant<int, 8>{});
    case 9:
    case 10:
    case 11:
    case 12: return launch(std::integral_constant<int, 12>{});
    default: return launch(std::integral_constant<int, 16>{});
    }
}

}  // namespace

cudaError_t launch_pack(const uint8_t *mask, int B, int N, int64_t row_bytes, int n_tensors,
                        const void *const *src, void *const *dst, int64_t capacity, int32_t *cu, int32_t *err,
                        int num_sms, cudaStream_t stream)
{
    SrcPtrs s{};
    DstPtrs d{};
    for (int i = 0; i < n_tensors; ++i) {
        s.p[i] = static_cast<const uint8_t *>(src[i]);
        d.p[i] = static_cast<uint8_t *>(dst[i]);
    }
    if (B == 0)
        return cudaMemsetAsync(cu, 0, sizeof(int32_t), stream);  // cu_seqlens = {0}
    const int splits = choose_splits(B, N, num_sms);
    const int rows = (N + splits - 1) / splits;
    const int V = static_cast<int>(row_bytes / 16);
    const dim3 grid(splits, B);
    if (B >= kPackScanMinBatch) {
        const cudaError_t e = launch_pdl(cu_kernel, dim3(1), dim3(kScanThreads), 0, stream, mask, B, N, capacity, cu, err);
        if (e != cudaSuccess)
            return e;
        return dispatch_vpl(V, [&](auto vpl) {
            return launch_pdl(pack_kernel<decltype(vpl)::value, true>, grid, dim3(kThreads), 0, stream, mask, N, rows,
                              V, n_tensors, s, d, capacity, cu, err);
        });
    }
    return dispatch_vpl(V, [&](auto vpl) {
        return launch_pdl(pack_kernel<decltype(vpl)::value, false>, grid, dim3(kThreads), 0, stream, mask, N, rows, V,
                          n_tensors, s, d, capacity, cu, err);
    });
}

cudaError_t launch_unpack(const void *packed, const int32_t *cu, const uint8_t *mask, int B, int N,
                          int64_t row_bytes, int fill_mode, int64_t capacity, void *dst, int32_t *err, int num_sms,
                          cudaStream_t stream)
{
    if (B == 0)
        return cudaSuccess;
    const int splits = choose_splits(B, N, num_sms);
    const int rows = (N + splits - 1) / splits;
    const int V = static_cast<int>(row_bytes / 16);
    const dim3 grid(splits, B);
    return dispatch_vpl(V, [&](auto vpl) {
        return launch_pdl(unpack_kernel<decltype(vpl)::value>, grid, dim3(kThreads), 0, stream,
                          static_cast<const uint8_t *>(packed), cu, mask, N, rows, V, fill_mode, capacity,
                          static_cast<uint8_t *>(dst), err);
    });
}

}  // namespace rra
