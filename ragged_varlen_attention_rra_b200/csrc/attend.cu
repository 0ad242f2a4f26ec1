// attend.cu -- bidirectional ragged attention on tcgen05 tensor cores (sm_100a).
//
// What it computes ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// sota2.com card, Abstract: a bidirectional attention kernel over the variable-length
// sequences left after token pruning): for every image b, head h and kept token i,
//     o_i = sum_j softmax_j(scale * q_i . k_j) v_j,   j over all L_b kept tokens of image b.
//
// How (B200-specific design, not the pages' Triton kernel):
//   * one persistent launch of two blocks per SM; each block walks a list of
//     (image, 128-row q-tile, head) work items that it derives from cu_seqlens on the device,
//     so the host never learns T;
//   * inside a block, warps specialise:
//       warp 0      TMA producer: Q tile and 128-key K/V chunks of one head, fetched straight
//                   from the packed [T, H, 64] layout (3-D tensor map, head = coordinate,
//                   128-byte swizzle) into two-slot rings, so the next item's loads overlap
//                   the current item's math;
//       warp 1      tensor-core issuer: S = Q K^T and O_chunk = P V as tcgen05.mma with fp32
//                   accumulators in TMEM (P comes from TMEM as the A operand);
//       warps 2..9  softmax: a pair of warps owns each quarter of the rows (TMEM lanes);
//                   within a 128-key chunk the two warps take alternate 32-key slices, so
//                   row max / row sum are thread-local plus one exchange per chunk between
//                   the two warps of a pair; keys are taken in chunks of 128 with an online
//                   softmax: O accumulates in TMEM across chunks, and when a row's running
//                   max rises the warps rescale that row of O in TMEM before the next PV MMA
//                   (each warp of a pair owns 32 of the 64 output columns), then rows are
//                   normalised and stored;
//   * for bf16 inputs P is split into a bf16 head and a bf16 remainder (two PV MMAs), which
//     keeps P at ~16 significant bits; fp16 P (11 bits) is used as is;
//   * key rows past the sequence end get probability 0 and the matching V rows are zeroed
//     in shared memory, so whatever bytes lie there (the next image, or uninitialised capacity
//     rows) never reach the output;
//   * every wait is bounded in time; on expiry the block records RRA_ERR_TIMEOUT, raises a
//     block-wide abort flag, drains the copies and MMAs it issued, frees TMEM and leaves.
#include <cuda.h>

#include <mutex>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int BM = 128;                 // query rows per tile (TMEM lanes)
constexpr int BN = 128;                 // keys per chunk
constexpr int kD = 64;                  // head dim
constexpr int kThreads = 320;           // 10 warps: producer, MMA, 8 x softmax
constexpr int kSoftmaxWarps = 8;
constexpr uint32_t kTmemCols = 256;
// S chunk, fp32 [128 x 128].  The P of each 32-key slice is written back over that slice's own
// S columns: bf16/fp16 head part in its first 16 columns, bf16 remainder in the next 16.
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 128;         // O chunk, fp32 [128 x 64]
constexpr uint32_t kTileBytes = 128 * 128;
constexpr int kStages = 2;              // ring depth of the Q slots and of the K/V chunk slots

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kStages * kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
constexpr uint32_t kOffRed = kOffBar + 256;             // row max / row sum exchange, 2 x 128 floats
constexpr uint32_t kOffTile = kOffRed + 2 * 128 * 4;    // tile_pre[B+1], then cu[B+1]
constexpr int kSmemFixed = 1024 /*align slack*/ + kOffTile;
constexpr int kSmemFloor = 80 * 1024;   // keeps at most two blocks (2 x 256 TMEM columns) per SM

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

struct Bars {
    uint64_t q_full[kStages], q_empty[kStages];
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full, p_full, o_full, o_free, drain;
    uint32_t tmem_slot;
    int abort;
    int warp_sums[kThreads / 32];
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b)
{
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// One decoded work item.
struct Item {
    int b, h, qt, seq0, L;
};

__device__ __forceinline__ Item decode_item(int item, int H, int B, const int32_t *tile_pre, const int32_t *cu)
{
    Item it;
    const int g = item / H;
    it.h = item - g * H;
    int lo = 0, hi = B;  // tile_pre[lo] <= g < tile_pre[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_pre[mid] <= g)
            lo = mid;
        else
            hi = mid;
    }
    it.b = lo;
    it.qt = g - tile_pre[lo];
    it.seq0 = cu[lo];
    it.L = cu[lo + 1] - it.seq0;
    return it;
}

// Bounded wait used by every role: returns false when the block is aborting or the wait ran
// out (which itself raises the abort flag and the timeout error).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Bars *bars, const Params &p)
{
    if (mbar_test_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (*reinterpret_cast<volatile int *>(&bars->abort))
            return false;
        if (p.wait_ns == 0 ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity))
            return true;
        if (global_timer_ns() - t0 >= p.wait_ns) {
            *reinterpret_cast<volatile int *>(&bars->abort) = 1;
            raise_error(p.err, RRA_ERR_TIMEOUT);
            return false;
        }
    }
}

// Warp-uniform version: every lane waits, and the warp proceeds only if all lanes saw the
// phase complete (so no lane can leave a loop that its warp-mates stay in).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, Bars *bars, const Params &p)
{
    const bool ok = wait_or_abort(bar, parity, bars, p);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Barrier between the two softmax warps that share a quarter of the rows (64 threads).
__device__ __forceinline__ void pair_sync(int quarter)
{
    asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, 2)
    attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bars = reinterpret_cast<Bars *>(base + kOffBar);
    int32_t *tile_pre = reinterpret_cast<int32_t *>(base + kOffTile);  // [B+1]
    int32_t *cu_s = tile_pre + (p.B + 1);                               // [B+1]
    float *red = reinterpret_cast<float *>(base + kOffRed);            // [2][128]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = p.B, H = p.H;

    if (tid == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->p_full, kSoftmaxWarps);   // one arrival per softmax warp
        mbar_init(&bars->o_full, 1);
        mbar_init(&bars->o_free, kSoftmaxWarps);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars->tmem_slot, kTmemCols);
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
            cu_s[b] = static_cast<int32_t>(s0);
            if (b == B - 1)
                cu_s[B] = static_cast<int32_t>(s1);
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
            bars->warp_sums[warp] = incl;
        __syncthreads();
        int before = carry;
        int chunk = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            before += (w < warp) ? bars->warp_sums[w] : 0;
            chunk += bars->warp_sums[w];
        }
        if (b < B)
            tile_pre[b + 1] = before + incl;
        carry += chunk;
        __syncthreads();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;
    const int total_items = tile_pre[B] * H;

    if (warp == 0) {
        // ================================================================ TMA producer
        // Empty-slot waits use the usual parity idiom: on a fresh barrier the phase "before"
        // phase 0 counts as complete, so waiting on parity (phase ^ 1) passes at once for the
        // first fill of each slot, then tracks the consumer's releases.
        uint32_t q_phase[kStages] = {0, 0}, kv_phase[kStages] = {0, 0};
        uint32_t q_issued = 0, kv_issued = 0;  // how many Q / KV slot fills were issued
        int qs = 0, ks = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
            const Item it = decode_item(item, H, B, tile_pre, cu_s);
            const int nkc = (it.L + BN - 1) / BN;
            // Q slot: free once the previous user of the slot has finished its last PV MMA
            ok = warp_wait(&bars->q_empty[qs], q_phase[qs] ^ 1u, bars, p);
            if (!ok)
                break;
            q_phase[qs] ^= 1u;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars->q_full[qs], kTileBytes);
                tma_load_3d(base + kOffQ + qs * kTileBytes, &tm_q, &bars->q_full[qs], 0, it.h, it.seq0 + it.qt * BM);
            }
            __syncwarp();
            ++q_issued;
            qs ^= 1;
            for (int kc = 0; kc < nkc; ++kc) {
                ok = warp_wait(&bars->kv_empty[ks], kv_phase[ks] ^ 1u, bars, p);
                if (!ok)
                    break;
                kv_phase[ks] ^= 1u;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars->kv_full[ks], 2 * kTileBytes);
                    tma_load_3d(base + kOffK + ks * kTileBytes, &tm_k, &bars->kv_full[ks], 0, it.h, it.seq0 + kc * BN);
                    tma_load_3d(base + kOffV + ks * kTileBytes, &tm_v, &bars->kv_full[ks], 0, it.h, it.seq0 + kc * BN);
                }
                __syncwarp();
                ++kv_issued;
                ks ^= 1;
            }
        }
        // drain: every issued fill has landed before the block may leave
        for (int s = 0; s < kStages; ++s) {
            const uint32_t nq = q_issued / kStages + (static_cast<uint32_t>(s) < q_issued % kStages ? 1u : 0u);
            if (nq > 0)
                mbar_wait_bounded(&bars->q_full[s], (nq - 1) & 1u, kDrainNs);
            const uint32_t nk = kv_issued / kStages + (static_cast<uint32_t>(s) < kv_issued % kStages ? 1u : 0u);
            if (nk > 0)
                mbar_wait_bounded(&bars->kv_full[s], (nk - 1) & 1u, kDrainNs);
        }
    } else if (warp == 1) {
        // ================================================================ tcgen05 issuer
        uint32_t q_ph[kStages] = {0, 0}, kv_ph[kStages] = {0, 0};
        uint32_t p_ph = 0, ofree_ph = 0, pv_ph = 0;
        uint32_t n_pv = 0;  // PV commits issued (each completes a phase of o_full)
        uint32_t n_items = 0;
        int qs = 0, ks = 0;
        const uint32_t idPV = idesc_f16(BM, kD, kBF16 ? 1u : 0u, 1u);
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
            const Item it = decode_item(item, H, B, tile_pre, cu_s);
            const int nkc = (it.L + BN - 1) / BN;
            ok = warp_wait(&bars->q_full[qs], q_ph[qs], bars, p);
            if (!ok)
                break;
            q_ph[qs] ^= 1u;
            const uint32_t sQa = smem_addr(base + kOffQ + qs * kTileBytes);
            for (int kc = 0; kc < nkc; ++kc) {
                const int nk = min(BN, it.L - kc * BN);
                const int nk16 = (nk + 15) & ~15;
                ok = warp_wait(&bars->kv_full[ks], kv_ph[ks], bars, p);
                if (!ok)
                    break;
                kv_ph[ks] ^= 1u;
                uint8_t *sV = base + kOffV + ks * kTileBytes;
                // zero V rows [nk, nk16): they enter the PV MMA with probability 0
                if (nk < nk16) {
                    for (int i = lane; i < (nk16 - nk) * 8; i += 32)
                        *reinterpret_cast<uint4 *>(sV + (nk + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                // S region (which holds the previous chunk's P) is free once that PV completed
                if (n_pv > 0) {
                    ok = warp_wait(&bars->o_full, pv_ph, bars, p);
                    if (!ok)
                        break;
                    pv_ph ^= 1u;
                }
                const uint32_t sKa = smem_addr(base + kOffK + ks * kTileBytes);
                const uint32_t sVa = smem_addr(sV);
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t idS = idesc_f16(BM, nk16, kBF16 ? 1u : 0u, 0u);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss(tmem + kColS, smem_desc_sw128(sQa + kk * 32, 16, 1024),
                               smem_desc_sw128(sKa + kk * 32, 16, 1024), idS, kk > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full);
                }
                __syncwarp();
                // P written (and O rescaled) by the softmax warps; before the first PV of an item
                // the previous item's O must have been read out by the epilogue
                ok = warp_wait(&bars->p_full, p_ph, bars, p);
                if (!ok)
                    break;
                p_ph ^= 1u;
                if (kc == 0 && n_items > 0) {
                    ok = warp_wait(&bars->o_free, ofree_ph, bars, p);
                    if (!ok)
                        break;
                    ofree_ph ^= 1u;
                }
                if (lane == 0) {
                    tc_fence_after();
                    // keys 16j..16j+15 live in slice j/2: head part at column 32(j/2) + 8(j%2),
                    // remainder 16 columns further
                    for (int j = 0; j < nk16 / 16; ++j)
                        mma_ts(tmem + kColO, tmem + kColS + 32 * (j >> 1) + 8 * (j & 1),
                               smem_desc_sw128(sVa + j * 2048, 16, 1024), idPV, (kc > 0 || j > 0) ? 1u : 0u);
                    if (kBF16)
                        for (int j = 0; j < nk16 / 16; ++j)
                            mma_ts(tmem + kColO, tmem + kColS + 32 * (j >> 1) + 8 * (j & 1) + 16,
                                   smem_desc_sw128(sVa + j * 2048, 16, 1024), idPV, 1u);
                    mma_commit(&bars->o_full);
                    mma_commit(&bars->kv_empty[ks]);
                    if (kc == nkc - 1)
                        mma_commit(&bars->q_empty[qs]);
                }
                __syncwarp();
                ++n_pv;
                ks ^= 1;
            }
            ++n_items;
            qs ^= 1;
        }
        // drain: every MMA this thread issued has completed
        if (lane == 0) {
            mma_commit(&bars->drain);
            mbar_wait_bounded(&bars->drain, 0, kDrainNs);
        }
        __syncwarp();
    } else {
        // ================================================================ softmax + epilogue
        const int q4 = warp & 3;                     // TMEM lane quarter of this warp
        const int hf = (warp - 2) >> 2;              // which of the pair: slices hf, hf+2, ...; O columns 32hf..
        const int row = q4 * 32 + lane;              // row of S / O owned by this thread
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        float *red_max = red;                        // [128]
        float *red_sum = red + 128;                  // [128]
        uint32_t s_ph = 0, o_ph = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
            const Item it = decode_item(item, H, B, tile_pre, cu_s);
            const int nkc = (it.L + BN - 1) / BN;
            const int q0 = it.qt * BM;
            const int qrows = min(BM, it.L - q0);
            const bool warp_active = q4 * 32 < qrows;
            float m_run = -INFINITY, l_run = 0.f;
            for (int kc = 0; kc < nkc; ++kc) {
                const int nk = min(BN, it.L - kc * BN);
                const int nk16 = (nk + 15) & ~15;
                ok = warp_wait(&bars->s_full, s_ph, bars, p);
                if (!ok)
                    break;
                s_ph ^= 1u;
                tc_fence_after();
                float m_new = m_run;
                if (warp_active) {
                    // pass 1: row max over this warp's valid keys, combined with the pair
                    float mx = -INFINITY;
                    for (int c = 32 * hf; c < nk16; c += 64) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + kColS + c, r);
                        tmem_wait_ld();
                        if (c + 32 <= nk) {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                mx = fmaxf(mx, __uint_as_float(r[j]));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (c + j < nk)
                                    mx = fmaxf(mx, __uint_as_float(r[j]));
                        }
                    }
                    if (hf == 1)
                        red_max[row] = mx;
                    pair_sync(q4);
                    if (hf == 0)
                        red_max[row] = fmaxf(mx, red_max[row]);
                    pair_sync(q4);
                    m_new = fmaxf(m_run, red_max[row]);
                }
                // later chunks: the previous PV has landed in O; rescale rows whose max rose
                if (kc > 0) {
                    ok = warp_wait(&bars->o_full, o_ph, bars, p);
                    if (!ok)
                        break;
                    o_ph ^= 1u;
                    tc_fence_after();
                    if (warp_active) {
                        const float alpha = ex2_approx((m_run - m_new) * p.scale_log2);
                        l_run *= alpha;
                        if (__any_sync(0xffffffffu, m_new > m_run)) {
                            uint32_t r[32];
                            tmem_ld32(lane_base + kColO + 32 * hf, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
                            tmem_st32(lane_base + kColO + 32 * hf, r);
                        }
                    }
                }
                if (warp_active) {
                    m_run = m_new;
                    const float neg_m = -m_new * p.scale_log2;
                    // pass 2: P = exp2(scale*log2e*(s - m)), row sum, P back over this slice's S
                    for (int c = 32 * hf; c < nk16; c += 64) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + kColS + c, r);
                        tmem_wait_ld();
                        if (c + 32 <= nk) {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                r[j] = __float_as_uint(ex2_approx(fmaf(__uint_as_float(r[j]), p.scale_log2, neg_m)));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                r[j] = __float_as_uint(
                                    (c + j < nk) ? ex2_approx(fmaf(__uint_as_float(r[j]), p.scale_log2, neg_m)) : 0.f);
                        }
                        uint32_t pp[32];
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            const float a = __uint_as_float(r[2 * jj]), b = __uint_as_float(r[2 * jj + 1]);
                            l_run += a + b;
                            if (kBF16) {
                                pp[jj] = pack_bf16(a, b);
                                const float ha = __uint_as_float(pp[jj] << 16);
                                const float hb = __uint_as_float(pp[jj] & 0xFFFF0000u);
                                pp[16 + jj] = pack_bf16(a - ha, b - hb);
                            } else {
                                pp[jj] = pack_f16(a, b);
                                pp[16 + jj] = 0u;
                            }
                        }
                        tmem_st32(lane_base + kColS + c, pp);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->p_full);
            }
            if (!ok)
                break;
            // epilogue: last PV landed; the pair adds its partial row sums, each warp normalises
            // and stores its 32 output columns, then O is released for the next item
            ok = warp_wait(&bars->o_full, o_ph, bars, p);
            if (!ok)
                break;
            o_ph ^= 1u;
            tc_fence_after();
            if (warp_active) {
                uint32_t r[32];
                tmem_ld32(lane_base + kColO + 32 * hf, r);
                tmem_wait_ld();
                if (hf == 1)
                    red_sum[row] = l_run;
                pair_sync(q4);
                if (hf == 0)
                    red_sum[row] = l_run + red_sum[row];
                pair_sync(q4);
                const float inv = 1.f / red_sum[row];
                if (row < qrows) {
                    const int t = it.seq0 + q0 + row;
                    const int64_t off = (static_cast<int64_t>(t) * H + it.h) * kD + 32 * hf;
                    if (p.out_dt == RRA_F32) {
                        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + off);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            dst[j] = make_float4(__uint_as_float(r[4 * j]) * inv, __uint_as_float(r[4 * j + 1]) * inv,
                                                 __uint_as_float(r[4 * j + 2]) * inv,
                                                 __uint_as_float(r[4 * j + 3]) * inv);
                    } else {
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + off);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                f[e] = __uint_as_float(r[8 * j + e]) * inv;
                            uint4 w;
                            if (p.out_dt == RRA_BF16) {
                                w.x = pack_bf16(f[0], f[1]);
                                w.y = pack_bf16(f[2], f[3]);
                                w.z = pack_bf16(f[4], f[5]);
                                w.w = pack_bf16(f[6], f[7]);
                            } else {
                                w.x = pack_f16(f[0], f[1]);
                                w.y = pack_f16(f[2], f[3]);
                                w.z = pack_f16(f[4], f[5]);
                                w.w = pack_f16(f[6], f[7]);
                            }
                            dst[j] = w;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->o_free);
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

    int smem = kSmemFixed + 2 * (a.B + 1) * 4;
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
