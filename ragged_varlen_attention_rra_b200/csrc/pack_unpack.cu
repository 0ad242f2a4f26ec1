// pack_unpack.cu -- the token packer and unpacker around the ragged attention
// ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers": aissential.tech summary,
// Method -- a two-phase packer, index computation then gather; sota2.com card, Abstract -- the
// pack-attend-unpack pipeline back to the padded layout).
//
// Both kernels are HBM-bound byte movers.  A block owns a range of padded rows of one image
// (grid = splits x images).  It derives everything it needs from the keep mask itself:
//   * the packed start of its image, cu[b] = number of nonzero mask bytes of images < b
//     (pack only; a block-wide count with 16-byte loads, so no second launch and no
//     inter-block wait is needed), and
//   * the rank of each kept row inside the image (warp ballots + a block prefix),
// then moves rows as 16-byte vectors, eight independent loads in flight per thread.
#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 8;  // 16-byte vectors in flight per thread

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

__device__ __forceinline__ int block_sum(int v, int *red)
{
    v = __reduce_add_sync(0xffffffffu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // red[] may still be read by a previous call
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    int total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
        total += red[w];
    return total;
}

// Number of nonzero bytes in p[0, n), computed by the whole block.
__device__ int block_count_nonzero(const uint8_t *p, int64_t n, int *red)
{
    int local = 0;
    if (n > 0) {
        const uintptr_t addr = reinterpret_cast<uintptr_t>(p);
        const int64_t align_gap = static_cast<int64_t>((16u - (addr & 15u)) & 15u);
        const int64_t head = n < align_gap ? n : align_gap;
        if (threadIdx.x < head)
            local += p[threadIdx.x] != 0;
        const uint4 *body = reinterpret_cast<const uint4 *>(p + head);
        const int64_t nvec = (n - head) >> 4;
        for (int64_t i0 = threadIdx.x; i0 < nvec; i0 += static_cast<int64_t>(kThreads) * kBatch) {
            uint4 v[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int64_t i = i0 + static_cast<int64_t>(u) * kThreads;
                v[u] = (i < nvec) ? __ldg(body + i) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                local += nonzero_bytes(v[u].x) + nonzero_bytes(v[u].y) + nonzero_bytes(v[u].z) +
                         nonzero_bytes(v[u].w);
        }
        const int64_t tail0 = head + (nvec << 4);
        if (tail0 + threadIdx.x < n)
            local += p[tail0 + threadIdx.x] != 0;
    }
    return block_sum(local, red);
}

// Scan mask row bytes [n0, n1): for every kept position write its local rank slot into
// `slot_of` (indexed n - n0; -1 when pruned).  Returns the number of kept positions.
__device__ int block_scan_row(const uint8_t *row, int n0, int n1, int16_t *slot_of, int *warp_tot)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int running = 0;
    for (int c0 = n0; c0 < n1; c0 += kThreads) {
        const int n = c0 + threadIdx.x;
        const bool keep = (n < n1) && row[n] != 0;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        __syncthreads();
        if (lane == 0)
            warp_tot[warp] = __popc(bal);
        __syncthreads();
        int before = 0, chunk = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int t = warp_tot[w];
            before += (w < warp) ? t : 0;
            chunk += t;
        }
        if (n < n1)
            slot_of[n - n0] = keep ? static_cast<int16_t>(running + before + __popc(bal & ((1u << lane) - 1u)))
                                   : static_cast<int16_t>(-1);
        running += chunk;
    }
    __syncthreads();
    return running;
}

__global__ void __launch_bounds__(kThreads) pack_kernel(const uint8_t *__restrict__ mask, int B, int N,
                                                        int rows_per_split, int vec_per_row, int n_tensors,
                                                        SrcPtrs src, DstPtrs dst, int64_t capacity,
                                                        int32_t *__restrict__ cu, int32_t *err)
{
    __shared__ int red[kWarps];
    __shared__ int warp_tot[kWarps];
    __shared__ int16_t slot_of[kMaxRowsPerSplit];
    __shared__ int16_t n_of_slot[kMaxRowsPerSplit];

    const int b = blockIdx.y;
    const int n0 = blockIdx.x * rows_per_split;
    if (n0 >= N)
        return;
    const int n1 = min(N, n0 + rows_per_split);
    const uint8_t *row = mask + static_cast<int64_t>(b) * N;

    // Phase 1: where this image starts in the packed layout, and where this split starts in it.
    const int64_t image_start = block_count_nonzero(mask, static_cast<int64_t>(b) * N, red);
    const int rank0 = block_count_nonzero(row, n0, red);
    if (blockIdx.x == 0) {
        const int Lb = block_count_nonzero(row, N, red);
        if (threadIdx.x == 0) {
            if (b == 0)
                cu[0] = 0;
            cu[b + 1] = static_cast<int32_t>(image_start + Lb);
            if (image_start + Lb > capacity)
                raise_error(err, RRA_ERR_CAPACITY);
        }
    }
    const int nk = block_scan_row(row, n0, n1, slot_of, warp_tot);
    for (int i = threadIdx.x; i < n1 - n0; i += kThreads)
        if (slot_of[i] >= 0)
            n_of_slot[slot_of[i]] = static_cast<int16_t>(i);
    __syncthreads();

    // Phase 2: gather, 16-byte vectors; work index = ((slot * n_tensors) + tensor) * V + vec.
    const int64_t out_row0 = image_start + rank0;
    const int V = vec_per_row;
    const int total = nk * n_tensors * V;
    for (int i0 = threadIdx.x; i0 < total; i0 += kThreads * kBatch) {
        uint4 val[kBatch];
        uint4 *dptr[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kThreads;
            dptr[u] = nullptr;
            if (i < total) {
                const int pair = i / V;
                const int vec = i - pair * V;
                const int slot = pair / n_tensors;
                const int t = pair - slot * n_tensors;
                const int64_t out_row = out_row0 + slot;
                if (out_row < capacity) {
                    const int64_t in_row = static_cast<int64_t>(b) * N + n0 + n_of_slot[slot];
                    const uint8_t *sp = t == 0 ? src.p[0] : (t == 1 ? src.p[1] : src.p[2]);
                    uint8_t *dp = t == 0 ? dst.p[0] : (t == 1 ? dst.p[1] : dst.p[2]);
                    val[u] = ld_stream(reinterpret_cast<const uint4 *>(sp) + in_row * V + vec);
                    dptr[u] = reinterpret_cast<uint4 *>(dp) + out_row * V + vec;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (dptr[u] != nullptr)
                *dptr[u] = val[u];
    }
}

__global__ void __launch_bounds__(kThreads) unpack_kernel(const uint8_t *__restrict__ packed,
                                                          const int32_t *__restrict__ cu,
                                                          const uint8_t *__restrict__ mask, int B, int N,
                                                          int rows_per_split, int vec_per_row, int fill_mode,
                                                          int64_t capacity, uint8_t *__restrict__ dst, int32_t *err)
{
    __shared__ int red[kWarps];
    __shared__ int warp_tot[kWarps];
    __shared__ int16_t slot_of[kMaxRowsPerSplit];

    const int b = blockIdx.y;
    const int n0 = blockIdx.x * rows_per_split;
    if (n0 >= N)
        return;
    const int n1 = min(N, n0 + rows_per_split);
    const uint8_t *row = mask + static_cast<int64_t>(b) * N;
    const int64_t start = cu[b];
    const int64_t end = cu[b + 1];

    const int rank0 = block_count_nonzero(row, n0, red);
    const int nk = block_scan_row(row, n0, n1, slot_of, warp_tot);
    const bool image_ok = start >= 0 && end >= start;
    if (threadIdx.x == 0) {
        if (!image_ok || (n1 == N && rank0 + nk != end - start))
            raise_error(err, RRA_ERR_BAD_SEQLENS);
        else if (start + rank0 + nk > capacity)
            raise_error(err, RRA_ERR_CAPACITY);
    }
    // kept rows read packed rows [start, lim) only; a malformed image reads nothing
    const int64_t lim = image_ok ? min(end, capacity) : start;

    const int V = vec_per_row;
    const int total = (n1 - n0) * V;
    for (int i0 = threadIdx.x; i0 < total; i0 += kThreads * kBatch) {
        uint4 val[kBatch];
        uint4 *dptr[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kThreads;
            dptr[u] = nullptr;
            if (i < total) {
                const int r = i / V;
                const int vec = i - r * V;
                const int slot = slot_of[r];
                const int64_t out_row = static_cast<int64_t>(b) * N + n0 + r;
                if (slot >= 0) {
                    const int64_t in_row = start + rank0 + slot;
                    if (in_row >= start && in_row < lim) {
                        val[u] = ld_stream(reinterpret_cast<const uint4 *>(packed) + in_row * V + vec);
                        dptr[u] = reinterpret_cast<uint4 *>(dst) + out_row * V + vec;
                    }
                } else if (fill_mode == 0) {
                    val[u] = make_uint4(0, 0, 0, 0);
                    dptr[u] = reinterpret_cast<uint4 *>(dst) + out_row * V + vec;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (dptr[u] != nullptr)
                *dptr[u] = val[u];
    }
}

int choose_splits(int B, int N, int num_sms)
{
    const int target_blocks = 4 * num_sms;
    int splits = (target_blocks + B - 1) / (B > 0 ? B : 1);
    const int max_splits = (N + 15) / 16;  // at least 16 padded rows per block
    if (splits > max_splits)
        splits = max_splits;
    const int min_splits = (N + kMaxRowsPerSplit - 1) / kMaxRowsPerSplit;
    if (splits < min_splits)
        splits = min_splits;
    return splits < 1 ? 1 : splits;
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
    if (B == 0) {
        // Nothing to gather; cu_seqlens = {0}.
        return cudaMemsetAsync(cu, 0, sizeof(int32_t), stream);
    }
    const int splits = choose_splits(B, N, num_sms);
    const int rows = (N + splits - 1) / splits;
    dim3 grid(splits, B);
    pack_kernel<<<grid, kThreads, 0, stream>>>(mask, B, N, rows, static_cast<int>(row_bytes / 16), n_tensors, s, d,
                                               capacity, cu, err);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const void *packed, const int32_t *cu, const uint8_t *mask, int B, int N,
                          int64_t row_bytes, int fill_mode, int64_t capacity, void *dst, int32_t *err, int num_sms,
                          cudaStream_t stream)
{
    if (B == 0)
        return cudaSuccess;
    const int splits = choose_splits(B, N, num_sms);
    const int rows = (N + splits - 1) / splits;
    dim3 grid(splits, B);
    unpack_kernel<<<grid, kThreads, 0, stream>>>(static_cast<const uint8_t *>(packed), cu, mask, B, N, rows,
                                                 static_cast<int>(row_bytes / 16), fill_mode, capacity,
                                                 static_cast<uint8_t *>(dst), err);
    return cudaGetLastError();
}

}  // namespace rra
