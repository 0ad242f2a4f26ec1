// attend.cu -- bidirectional ragged attention on tcgen05 tensor cores (sm_100a).
//
// What it computes ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// sota2.com card, Abstract: a bidirectional attention kernel over the variable-length
// sequences left after token pruning): for every image b, head h and kept token i,
//     o_i = sum_j softmax_j(scale * q_i . k_j) v_j,   j over all L_b kept tokens of image b.
//
// How (B200-specific design, not the pages' Triton kernel):
//   * one persistent launch; each block walks a list of (image, q-tile, head) work items that
//     it derives from cu_seqlens on the device, so the host never learns T;
//   * Q, K, V tiles [128 tokens x 64] of one head are fetched by TMA straight from the packed
//     [T, H, 64] layout (a 3-D tensor map; the head is a coordinate), 128-byte swizzled;
//   * S = Q K^T and O_chunk = P V run as tcgen05.mma with fp32 accumulators in TMEM; P goes
//     from registers back to TMEM and feeds the PV MMA as its A operand;
//   * thread r of the 128-thread block owns row r of S and O (TMEM lane r), so the softmax
//     row max / row sum are thread-local; keys are processed in chunks of 128 with an online
//     (running max, rescaled sum) merge of O in registers;
//   * for bf16 inputs P is split into a bf16 head and a bf16 remainder (two PV MMAs), which
//     keeps P at ~16 significant bits; fp16 P (11 bits) is used as is;
//   * key rows past the sequence end are masked to probability 0 and the matching V rows are
//     zeroed in shared memory, so whatever bytes lie there (the next image, or uninitialised
//     capacity rows) never reach the output;
//   * every wait on an asynchronous copy or MMA is bounded in time; on expiry the block
//     records RRA_ERR_TIMEOUT, waits for its own outstanding work and leaves.
#include <cuda.h>

#include <mutex>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int BM = 128;                 // query rows per tile (TMEM lanes)
constexpr int BN = 128;                 // keys per chunk
constexpr int kD = 64;                  // head dim
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;           // S chunk, fp32 [128 x 128]; P (head part) reuses its first 64 columns
constexpr uint32_t kColPlo = 128;       // P remainder part (bf16 only), 64 columns
constexpr uint32_t kColO = 192;         // O chunk, fp32 [128 x 64]
constexpr uint32_t kTileBytes = 128 * 128;
constexpr int kSmemFixed = 1024 /*align*/ + 3 * kTileBytes + 64;
constexpr int kSmemFloor = 90 * 1024;   // keeps at most two blocks (2 x 256 TMEM columns) per SM

struct Params {
    const int32_t *cu;
    void *out;
    int B, H;
    int64_t capacity;
    float scale_log2;
    int out_dt;
    int32_t *err;
    uint64_t wait_ns;
};

constexpr uint64_t kDrainNs = 2000000000ull;

__device__ __forceinline__ uint32_t pack_pair(float a, float b, bool bf16, float &ra, float &rb)
{
    if (bf16) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        const float2 f = __bfloat1622float2(h);
        ra = a - f.x;
        rb = b - f.y;
        return *reinterpret_cast<const uint32_t *>(&h);
    } else {
        const __half2 h = __floats2half2_rn(a, b);
        ra = 0.f;
        rb = 0.f;
        return *reinterpret_cast<const uint32_t *>(&h);
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;
    uint8_t *sK = base + kTileBytes;
    uint8_t *sV = base + 2 * kTileBytes;
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(base + 3 * kTileBytes);
    uint64_t *bar_mma = bar_load + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 2);
    int *warp_sums = reinterpret_cast<int *>(bar_load + 4);        // 4 ints
    int32_t *tile_pre = reinterpret_cast<int32_t *>(base + 3 * kTileBytes + 64);  // [B+1]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = p.B, H = p.H;

    if (tid == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }

    // ---- work list: tile_pre[b] = number of 128-row query tiles of images < b.
    if (tid == 0)
        tile_pre[0] = 0;
    int carry = 0;
    for (int c0 = 0; c0 < B; c0 += kThreads) {
        const int b = c0 + tid;
        int tiles = 0;
        if (b < B) {
            const int64_t s0 = p.cu[b], s1 = p.cu[b + 1];
            if (s0 < 0 || s1 < s0 || s1 > p.capacity) {
                if (blockIdx.x == 0)
                    raise_error(p.err, RRA_ERR_BAD_SEQLENS);
            } else {
                tiles = static_cast<int>((s1 - s0 + BM - 1) / BM);
            }
        }
        int incl = tiles;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off)
                incl += t;
        }
        if (lane == 31)
            warp_sums[warp] = incl;
        __syncthreads();
        int before = carry;
        int chunk = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            before += (w < warp) ? warp_sums[w] : 0;
            chunk += warp_sums[w];
        }
        if (b < B)
            tile_pre[b + 1] = before + incl;
        carry += chunk;
        __syncthreads();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t total_items = static_cast<int64_t>(tile_pre[B]) * H;

    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t sQa = smem_addr(sQ), sKa = smem_addr(sK), sVa = smem_addr(sV);
    uint32_t ld_phase = 0, mma_phase = 0;
    bool failed = false;

    for (int64_t item = blockIdx.x; item < total_items && !failed; item += gridDim.x) {
        const int g = static_cast<int>(item / H);
        const int h = static_cast<int>(item - static_cast<int64_t>(g) * H);
        int lo = 0, hi = B;  // tile_pre[lo] <= g < tile_pre[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tile_pre[mid] <= g)
                lo = mid;
            else
                hi = mid;
        }
        const int b = lo;
        const int qt = g - tile_pre[b];
        const int seq0 = p.cu[b];
        const int L = p.cu[b + 1] - seq0;
        const int q0 = qt * BM;
        const int qrows = min(BM, L - q0);
        const int nkc = (L + BN - 1) / BN;
        const bool warp_active = warp * 32 < qrows;

        float m_run = -INFINITY, l_run = 0.f;
        float o[kD];
#pragma unroll
        for (int j = 0; j < kD; ++j)
            o[j] = 0.f;

        for (int kc = 0; kc < nkc; ++kc) {
            const int k0 = kc * BN;
            const int nk = min(BN, L - k0);
            const int nk16 = (nk + 15) & ~15;

            // ---- TMA: (Q on the first chunk) + K + V chunk of this head
            if (tid == 0) {
                mbar_arrive_expect_tx(bar_load, (kc == 0 ? 3u : 2u) * kTileBytes);
                if (kc == 0)
                    tma_load_3d(sQ, &tm_q, bar_load, 0, h, seq0 + q0);
                tma_load_3d(sK, &tm_k, bar_load, 0, h, seq0 + k0);
                tma_load_3d(sV, &tm_v, bar_load, 0, h, seq0 + k0);
            }
            bool ok = mbar_wait_bounded(bar_load, ld_phase, p.wait_ns);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) {
                    raise_error(p.err, RRA_ERR_TIMEOUT);
                    mbar_wait_bounded(bar_load, ld_phase, kDrainNs);
                }
                failed = true;
                break;
            }
            ld_phase ^= 1;

            // ---- zero V rows [nk, nk16): they enter the PV MMA with probability 0
            if (nk < nk16) {
                const int nz = (nk16 - nk) * 8;
                for (int i = tid; i < nz; i += kThreads) {
                    const int r = nk + (i >> 3);
                    *reinterpret_cast<uint4 *>(sV + r * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncthreads();

            // ---- S = Q K^T  (M = 128, N = nk16, K = 64 in four steps of 16)
            if (tid == 0) {
                tc_fence_after();
                const uint32_t idS = idesc_f16(BM, nk16, kBF16 ? 1u : 0u, 0u);
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint64_t ad = smem_desc_sw128(sQa + ks * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(sKa + ks * 32, 16, 1024);
                    mma_ss(tmem + kColS, ad, bd, idS, ks > 0 ? 1u : 0u);
                }
                mma_commit(bar_mma);
            }
            ok = mbar_wait_bounded(bar_mma, mma_phase, p.wait_ns);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) {
                    raise_error(p.err, RRA_ERR_TIMEOUT);
                    mbar_wait_bounded(bar_mma, mma_phase, kDrainNs);
                }
                failed = true;
                break;
            }
            mma_phase ^= 1;
            tc_fence_after();

            // ---- softmax of this chunk: row max, P = exp2(scale*log2e*(s - m)), row sum
            float m_new = m_run, l_add = 0.f;
            if (warp_active) {
                float mx = -INFINITY;
                for (int c = 0; c < nk16; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(lane_base + kColS + c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c + j < nk)
                            mx = fmaxf(mx, __uint_as_float(r[j]));
                }
                m_new = fmaxf(m_run, mx);
                const float neg_m = -m_new * p.scale_log2;
                for (int c = 0; c < nk16; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(lane_base + kColS + c, r);
                    tmem_wait_ld();
                    uint32_t phi[16], plo[16];
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int j0 = c + 2 * jj;
                        const float p0 = (j0 < nk) ? ex2_approx(fmaf(__uint_as_float(r[2 * jj]), p.scale_log2, neg_m)) : 0.f;
                        const float p1 = (j0 + 1 < nk) ? ex2_approx(fmaf(__uint_as_float(r[2 * jj + 1]), p.scale_log2, neg_m)) : 0.f;
                        l_add += p0 + p1;
                        float r0, r1;
                        phi[jj] = pack_pair(p0, p1, kBF16, r0, r1);
                        plo[jj] = kBF16 ? pack_bf16(r0, r1) : 0u;
                    }
                    tmem_st16(lane_base + kColS + c / 2, phi);
                    if (kBF16)
                        tmem_st16(lane_base + kColPlo + c / 2, plo);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncthreads();

            // ---- O_chunk = P V  (M = 128, N = 64, K = nk16; P from TMEM, V MN-major in smem)
            if (tid == 0) {
                tc_fence_after();
                const uint32_t idPV = idesc_f16(BM, kD, kBF16 ? 1u : 0u, 1u);
                for (int j = 0; j < nk16 / 16; ++j) {
                    const uint64_t bd = smem_desc_sw128(sVa + j * 2048, 16, 1024);
                    mma_ts(tmem + kColO, tmem + kColS + j * 8, bd, idPV, j > 0 ? 1u : 0u);
                }
                if (kBF16) {
                    for (int j = 0; j < nk16 / 16; ++j) {
                        const uint64_t bd = smem_desc_sw128(sVa + j * 2048, 16, 1024);
                        mma_ts(tmem + kColO, tmem + kColPlo + j * 8, bd, idPV, 1u);
                    }
                }
                mma_commit(bar_mma);
            }
            ok = mbar_wait_bounded(bar_mma, mma_phase, p.wait_ns);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) {
                    raise_error(p.err, RRA_ERR_TIMEOUT);
                    mbar_wait_bounded(bar_mma, mma_phase, kDrainNs);
                }
                failed = true;
                break;
            }
            mma_phase ^= 1;
            tc_fence_after();

            // ---- online merge: O = O * exp2(c (m_old - m_new)) + O_chunk
            if (warp_active) {
                const float alpha = ex2_approx((m_run - m_new) * p.scale_log2);
                uint32_t r[32];
                tmem_ld32(lane_base + kColO, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    o[j] = fmaf(o[j], alpha, __uint_as_float(r[j]));
                tmem_ld32(lane_base + kColO + 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    o[32 + j] = fmaf(o[32 + j], alpha, __uint_as_float(r[j]));
                l_run = fmaf(l_run, alpha, l_add);
                m_run = m_new;
            }
            tc_fence_before();
            __syncthreads();
        }
        if (failed)
            break;

        // ---- epilogue: normalise and store this thread's row
        if (tid < qrows) {
            const float inv = 1.f / l_run;
            const int64_t row = static_cast<int64_t>(seq0) + q0 + tid;
            const int64_t off = (row * H + h) * kD;
            if (p.out_dt == RRA_F32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + off);
#pragma unroll
                for (int j = 0; j < kD / 4; ++j)
                    dst[j] = make_float4(o[4 * j] * inv, o[4 * j + 1] * inv, o[4 * j + 2] * inv, o[4 * j + 3] * inv);
            } else if (p.out_dt == RRA_BF16) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + off);
#pragma unroll
                for (int j = 0; j < kD / 8; ++j) {
                    uint4 w;
                    w.x = pack_bf16(o[8 * j + 0] * inv, o[8 * j + 1] * inv);
                    w.y = pack_bf16(o[8 * j + 2] * inv, o[8 * j + 3] * inv);
                    w.z = pack_bf16(o[8 * j + 4] * inv, o[8 * j + 5] * inv);
                    w.w = pack_bf16(o[8 * j + 6] * inv, o[8 * j + 7] * inv);
                    dst[j] = w;
                }
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__half *>(p.out) + off);
#pragma unroll
                for (int j = 0; j < kD / 8; ++j) {
                    uint4 w;
                    __half2 t;
                    t = __floats2half2_rn(o[8 * j + 0] * inv, o[8 * j + 1] * inv);
                    w.x = *reinterpret_cast<uint32_t *>(&t);
                    t = __floats2half2_rn(o[8 * j + 2] * inv, o[8 * j + 3] * inv);
                    w.y = *reinterpret_cast<uint32_t *>(&t);
                    t = __floats2half2_rn(o[8 * j + 4] * inv, o[8 * j + 5] * inv);
                    w.z = *reinterpret_cast<uint32_t *>(&t);
                    t = __floats2half2_rn(o[8 * j + 6] * inv, o[8 * j + 7] * inv);
                    w.w = *reinterpret_cast<uint32_t *>(&t);
                    dst[j] = w;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- host side -----------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// Packed [capacity, H, 64] 16-bit tensor seen as 3-D (d, head, token); box = one head x 128 tokens.
bool make_tmap(CUtensorMap *map, const void *ptr, int64_t capacity, int H, bool bf16)
{
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr)
        return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(capacity)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD * 2), static_cast<cuuint64_t>(H) * kD * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kD), 1u, static_cast<cuuint32_t>(BM)};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                           const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <bool kBF16>
cudaError_t set_smem_attr(int bytes)
{
    static std::mutex mu;
    static int done_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && done_bytes[dev] >= bytes)
        return cudaSuccess;
    e = cudaFuncSetAttribute(attend_kernel<kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev < 64)
        done_bytes[dev] = bytes;
    return e;
}

}  // namespace

cudaError_t launch_attend(const AttendArgs &a, int num_sms, cudaStream_t stream)
{
    if (a.B == 0)
        return cudaSuccess;
    alignas(64) CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, a.q, a.capacity, a.H, a.in_bf16) || !make_tmap(&tk, a.k, a.capacity, a.H, a.in_bf16) ||
        !make_tmap(&tv, a.v, a.capacity, a.H, a.in_bf16))
        return cudaErrorInvalidValue;
    Params p;
    p.cu = a.cu;
    p.out = a.o;
    p.B = a.B;
    p.H = a.H;
    p.capacity = a.capacity;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out_dt = a.out_dt;
    p.err = a.err;
    p.wait_ns = a.wait_ns;

    int smem = kSmemFixed + (a.B + 1) * 4;
    if (smem < kSmemFloor)
        smem = kSmemFloor;
    const int64_t max_tiles = (static_cast<int64_t>(a.max_seqlen > 0 ? a.max_seqlen : 1) + BM - 1) / BM;
    int64_t grid = static_cast<int64_t>(a.B) * a.H * max_tiles;
    if (grid > 2LL * num_sms)
        grid = 2LL * num_sms;
    if (grid < 1)
        grid = 1;
    cudaError_t e = a.in_bf16 ? set_smem_attr<true>(smem) : set_smem_attr<false>(smem);
    if (e != cudaSuccess)
        return e;
    if (a.in_bf16)
        attend_kernel<true><<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(tq, tk, tv, p);
    else
        attend_kernel<false><<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace rra
