// linear.cu -- the dense parts of a transformer block on packed token rows, for the
// attention-vs-MLP latency split of a token-pruned ViT block ("Dispatch-Aware Ragged Attention
// for Pruned Vision Transformers", aissential.tech summary, "In practice": decompose attention
// vs. MLP latency contributions):
//   * linear_kernel: Y = act(X W^T + b) (+ R), X [M, K] and W [N, K] bf16 (an nn.Linear weight,
//     [out, in]), fp32 accumulation on tcgen05 tensor cores, bf16 out; act = identity or the
//     exact (erf) GELU; R an optional residual [M, N]; Y may be split column-wise into several
//     outputs (the Q, K, V of a fused QKV projection, each [M, N / n_outs]).
//   * layernorm_kernel: y = (x - mean) / sqrt(var + eps) * gamma + beta per row, fp32 statistics.
// Both may take their row count from a device word (cu_seqlens[B] of the pack that produced the
// rows), so that a whole block on packed rows is enqueued without the host knowing T.
//
// linear_kernel (B200 design):
//   * persistent: one block per SM walks 128 x 256 output tiles (128 x 128 when an output's width
//     is an odd multiple of 128), tile t of the block = block id +
//     t * grid; tiles are numbered along N first, so the blocks in flight share their X rows
//     (read from HBM once, then from L2) and W (a few MiB) stays in L2;
//   * a 4-stage ring of (X 128 x 64, W 256 x 64) bf16 tiles in 128-byte-swizzled shared memory,
//     filled by TMA (warp 0); one thread of warp 1 issues 4 tcgen05.mma (M 128, N 256, K 16) per
//     stage into one of two TMEM accumulators (2 x 256 columns), so the epilogue of a tile
//     overlaps the MMAs of the next;
//   * warps 4..19 are the epilogue: warp w reads TMEM lane quarter w % 4 and columns
//     [64 p, 64 p + 64) with p = (w - 4) / 4, adds the bias, applies the activation and the
//     residual in fp32, rounds to bf16, and passes each 32 x 32 block through its own 2 KiB of
//     shared memory, so that the global stores go out as whole 64-byte row segments, 8 rows per
//     instruction;
//   * every wait is bounded in time; on expiry the block records RRA_ERR_TIMEOUT, raises an abort
//     flag so every role leaves, drains what it issued and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int GM = 128;  // output rows per tile (TMEM lanes)
constexpr int GK = 64;   // K per ring stage: one 128-byte swizzle atom of bf16
constexpr int kLinStages = 4;
constexpr int kLinThreads = 640;  // 20 warps: producer, issuer, TMEM owner, idle, 16 x epilogue
constexpr int kEpiWarp0 = 4;
constexpr int kEpiWarps = 16;
constexpr uint32_t kXBytes = GM * GK * 2;  // 16 KiB
// per epilogue warp, a 32 x 32 bf16 block of the output on its way to global memory (2 KiB)
constexpr uint32_t kStageWarpBytes = 32 * 32 * 2;
static_assert(kEpiWarp0 + kEpiWarps == kLinThreads / 32, "warp roles");

// The output tile's width GN (TMEM columns of one accumulator): 256, or 128 for outputs whose
// width is an odd multiple of 128 (DeiT-S's 384, 1152, 1536).
template <int GN>
struct LinCfg {
    static constexpr int kEpiCols = GN / (kEpiWarps / 4);  // columns per epilogue warp (64 or 32)
    static constexpr uint32_t kWBytes = GN * GK * 2;
    static constexpr uint32_t kStageBytes = kXBytes + kWBytes;
    static constexpr uint32_t kTmemCols = 2 * GN;
    static constexpr uint32_t kOffBar = kLinStages * kStageBytes;
    static constexpr uint32_t kOffStage = kOffBar + 256;
    static constexpr int kSmem = 1024 + static_cast<int>(kOffStage + kEpiWarps * kStageWarpBytes);
    static_assert(kEpiCols % 32 == 0 && kSmem <= 232448, "linear tile configuration");
};
constexpr uint64_t kLinDrainNs = 2000000000ull;

struct LinBars {
    uint64_t full[kLinStages], empty[kLinStages];  // ring stage loaded / consumed by the MMAs
    uint64_t acc_full[2], acc_empty[2];            // accumulator computed / read out by the epilogue
    uint64_t drain;
    uint32_t tmem_slot;
    int abort;
};
static_assert(sizeof(LinBars) <= 256, "barrier block");

struct LinParams {
    int M, N, K;
    const int32_t *m_dev;      // device row count (rows [0, min(M, *m_dev)) are computed), or null
    const uint16_t *bias;      // [N] bf16, or null
    const uint16_t *residual;  // [M, N] bf16, or null
    uint16_t *outs[kLinearMaxOuts];
    int n_outs, out_ld;        // outs[j] holds columns [j out_ld, (j + 1) out_ld), rows out_ld apart
    int act;                   // 0: identity, 1: GELU (erf)
    int32_t *err;
    uint64_t wait_ns;
};

// Bounded wait of the whole warp: false when the block aborts or the wait runs out (which
// raises the abort flag and records the timeout).
__device__ __noinline__ bool lin_wait_slow(uint64_t *bar, uint32_t parity, LinBars *bars, const LinParams &p)
{
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

__device__ __forceinline__ bool lin_wait(uint64_t *bar, uint32_t parity, LinBars *bars, const LinParams &p)
{
    const bool ok = mbar_test_wait(bar, parity) || lin_wait_slow(bar, parity, bars, p);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// The erf GELU of the transformer MLP, x Phi(x) = x (1 + erf(x / sqrt 2)) / 2, with erfc from
// Abramowitz and Stegun, Handbook of Mathematical Functions, 7.1.28: for z >= 0,
// erfc(z) = (1 + a1 z + a2 z^2 + ... + a6 z^6)^-16 with |error| <= 3e-7 (their coefficients).
// With z = |x| / sqrt 2: Phi(x) = erfc(z) / 2 for x < 0 and 1 - erfc(z) / 2 for x >= 0, so the
// negative tail is formed directly, without cancellation.  Six fused multiply-adds, four squarings
// and one reciprocal (an overflowing power gives erfc = 0 in the far tail).  The fp32 roundings of
// the power add a relative error of about 4e-6 to erfc; the GELU's error stays below
// 5e-6 |x|, far under the bf16 rounding of the output.
__device__ __forceinline__ float gelu_erf(float x)
{
    const float z = fabsf(x) * 0.70710678118654752f;
    float q = fmaf(z, 4.30638e-5f, 2.765672e-4f);
    q = fmaf(q, z, 1.520143e-4f);
    q = fmaf(q, z, 9.2705272e-3f);
    q = fmaf(q, z, 4.22820123e-2f);
    q = fmaf(q, z, 7.05230784e-2f);
    q = fmaf(q, z, 1.0f);
    q = q * q;
    q = q * q;
    q = q * q;
    q = q * q;
    const float h = 0.5f * rcp_approx(q);  // erfc(z) / 2
    return x * (x < 0.f ? h : 1.f - h);
}

__device__ __forceinline__ void lin_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

template <int GN>
__global__ void __launch_bounds__(kLinThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, const LinParams p)
{
    using Cfg = LinCfg<GN>;
    constexpr int kEpiCols = Cfg::kEpiCols;
    constexpr uint32_t kLinStageBytes = Cfg::kStageBytes, kLinTmemCols = Cfg::kTmemCols;
    constexpr uint32_t kOffLinBar = Cfg::kOffBar, kOffLinStage = Cfg::kOffStage;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    LinBars *bars = reinterpret_cast<LinBars *>(base + kOffLinBar);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    pdl_trigger();
    if (tid == 0) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_w);
        for (int s = 0; s < kLinStages; ++s) {
            mbar_init(&bars->full[s], 1);   // the producer's arrival plus the TMA bytes
            mbar_init(&bars->empty[s], 1);  // the issuer's MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bars->acc_full[a], 1);
            mbar_init(&bars->acc_empty[a], kEpiWarps);  // one arrival per epilogue warp
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 2) {
        tmem_alloc(&bars->tmem_slot, kLinTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;
    pdl_wait();  // X, W, bias, residual and the row count may come from the previous kernel

    const int M = p.m_dev != nullptr ? max(0, min(p.M, *p.m_dev)) : p.M;
    const int tiles_n = p.N / GN;
    const int tiles = ((M + GM - 1) / GM) * tiles_n;
    const int nkb = p.K / GK;
    const int t_first = static_cast<int>(blockIdx.x), t_step = static_cast<int>(gridDim.x);

    if (warp == 0) {
        // ================================================================ TMA producer
        // Empty-stage waits use the parity idiom: on a fresh barrier the phase before phase 0
        // counts as complete, so the first fill of each stage passes at once.
        int s = 0;
        uint32_t ph = 0;
        uint32_t fills = 0;
        bool ok = true;
        for (int t = t_first; ok && t < tiles; t += t_step) {
            const int m0 = (t / tiles_n) * GM, n0 = (t % tiles_n) * GN;
            for (int kb = 0; kb < nkb; ++kb) {
                ok = lin_wait(&bars->empty[s], ((ph >> s) & 1u) ^ 1u, bars, p);
                if (!ok)
                    break;
                ph ^= 1u << s;
                if (lane == 0) {
                    uint8_t *st = base + s * kLinStageBytes;
                    mbar_arrive_expect_tx(&bars->full[s], kLinStageBytes);
                    tma_load_2d(st, &tm_x, &bars->full[s], kb * GK, m0);  // rows past M read as zeros
                    tma_load_2d(st + kXBytes, &tm_w, &bars->full[s], kb * GK, n0);
                }
                __syncwarp();
                ++fills;
                s = (s + 1 == kLinStages) ? 0 : s + 1;
            }
        }
        // drain: every issued fill has landed before the block may leave
        if (lane == 0)
            for (int st = 0; st < kLinStages; ++st) {
                const uint32_t n = fills / kLinStages + (static_cast<uint32_t>(st) < fills % kLinStages ? 1u : 0u);
                if (n > 0)
                    mbar_wait_bounded(&bars->full[st], (n - 1) & 1u, kLinDrainNs);
            }
        __syncwarp();
    } else if (warp == 1) {
        // ================================================================ tcgen05 issuer
        // Tile t of this block accumulates in TMEM buffer t % 2 (columns 256 (t % 2) ...); the
        // epilogue releases the buffer (acc_empty) once it has read the tile out.
        const uint32_t idesc = idesc_f16(GM, GN, 1u, 0u);
        const uint64_t d0 = smem_desc_sw128(smem_addr(base), 16, 1024);
        int s = 0, tl = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int t = t_first; ok && t < tiles; t += t_step, ++tl) {
            const int ab = tl & 1;
            ok = lin_wait(&bars->acc_empty[ab], ((tl >> 1) & 1u) ^ 1u, bars, p);
            if (!ok)
                break;
            tc_fence_after();
            for (int kb = 0; kb < nkb; ++kb) {
                ok = lin_wait(&bars->full[s], (ph >> s) & 1u, bars, p);
                if (!ok)
                    break;
                ph ^= 1u << s;
                if (lane == 0) {
                    tc_fence_after();
                    // stepping K by 16 inside the 128-byte swizzled rows adds 32 bytes (2 units)
                    const uint64_t xd = d0 + ((s * kLinStageBytes) >> 4);
                    const uint64_t wd = xd + (kXBytes >> 4);
#pragma unroll
                    for (int kk = 0; kk < GK / 16; ++kk)
                        mma_ss(tmem + GN * ab, xd + 2 * kk, wd + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&bars->empty[s]);
                }
                __syncwarp();
                s = (s + 1 == kLinStages) ? 0 : s + 1;
            }
            if (!ok)
                break;
            if (lane == 0)
                mma_commit(&bars->acc_full[ab]);
            __syncwarp();
        }
        // drain: every MMA this thread issued has completed
        if (lane == 0) {
            mma_commit(&bars->drain);
            mbar_wait_bounded(&bars->drain, 0, kLinDrainNs);
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0) {
        // ================================================================ epilogue
        const int q4 = warp & 3;
        const int part = (warp - kEpiWarp0) >> 2;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        int tl = 0;
        bool ok = true;
        for (int t = t_first; ok && t < tiles; t += t_step, ++tl) {
            const int ab = tl & 1;
            ok = lin_wait(&bars->acc_full[ab], (tl >> 1) & 1u, bars, p);
            if (!ok)
                break;
            tc_fence_after();
            const int m0 = (t / tiles_n) * GM, n0 = (t % tiles_n) * GN;
#pragma unroll 1
            for (int c = 0; c < kEpiCols; c += 32) {
                const int col = part * kEpiCols + c;
                uint32_t r[32];
                tmem_ld32(lane_addr + GN * ab + col, r);
                tmem_wait_ld_dep(r);
                const int n = n0 + col;
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    v[j] = __uint_as_float(r[j]);
                if (p.bias != nullptr) {
                    const uint4 *b4 = reinterpret_cast<const uint4 *>(p.bias + n);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 w = __ldg(b4 + q);
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            v[8 * q + 2 * e] += bf16_bits_to_float(ws[e] & 0xFFFFu);
                            v[8 * q + 2 * e + 1] += bf16_bits_to_float(ws[e] >> 16);
                        }
                    }
                }
                if (p.act == RRA_ACT_GELU) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] = gelu_erf(v[j]);
                }
                // the warp's 32 x 32 block goes through its own staging buffer: row r at 64 r bytes,
                // 16-byte piece q at (q ^ ((r >> 1) & 3)) -- an XOR that spreads the 32 rows of a
                // piece over all the banks; global memory sees whole 64-byte row segments, lane l
                // taking piece l % 4 of rows l / 4 + 8 i
                uint8_t *stg = base + kOffLinStage + (warp - kEpiWarp0) * kStageWarpBytes;
                auto piece = [&](int rr, int q) { return stg + rr * 64 + ((q ^ ((rr >> 1) & 3)) << 4); };
                if (p.residual != nullptr) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = (lane >> 2) + 8 * i, q = lane & 3;
                        const int grow = m0 + q4 * 32 + rr;
                        uint4 w = make_uint4(0, 0, 0, 0);
                        if (grow < M)
                            w = *reinterpret_cast<const uint4 *>(p.residual + static_cast<int64_t>(grow) * p.N + n + 8 * q);
                        *reinterpret_cast<uint4 *>(piece(rr, q)) = w;
                    }
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(piece(lane, q));
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            v[8 * q + 2 * e] += bf16_bits_to_float(ws[e] & 0xFFFFu);
                            v[8 * q + 2 * e + 1] += bf16_bits_to_float(ws[e] >> 16);
                        }
                    }
                    __syncwarp();
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(piece(lane, q)) =
                        make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                   pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                __syncwarp();
                const int oi = n / p.out_ld;
                uint16_t *obase = p.outs[oi] + (n - oi * p.out_ld);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = (lane >> 2) + 8 * i, q = lane & 3;
                    const int grow = m0 + q4 * 32 + rr;
                    if (grow < M)
                        *reinterpret_cast<uint4 *>(obase + static_cast<int64_t>(grow) * p.out_ld + 8 * q) =
                            *reinterpret_cast<const uint4 *>(piece(rr, q));
                }
                __syncwarp();  // the buffer is reused by the next block
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                lin_arrive(&bars->acc_empty[ab]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kLinTmemCols);
    }
}

// ---- layernorm ------------------------------------------------------------------------------

constexpr int kLnThreads = 256;  // 8 rows in flight per block, one warp each
constexpr int kLnMaxChunks = kLayerNormMaxC / (32 * 8);

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// One warp per row: the row's 16-byte chunks spread over the lanes (chunk c to lane c % 32), the
// mean, then the variance of (x - mean) (two passes over registers), each a warp reduction in fp32.
// kChunks = chunks per lane (C / 256 rounded up): a narrow row needs few registers, so more blocks
// fit on an SM and more rows are in flight -- the kernel streams each row once, so rows in flight
// set its bandwidth.
template <int kChunks>
__global__ void __launch_bounds__(kLnThreads, kChunks <= 4 ? 4 : 2)
    layernorm_kernel(const uint16_t *x, const uint16_t *gamma, const uint16_t *beta, uint16_t *y, int64_t M_max,
                     const int32_t *m_dev, int C, float eps)
{
    pdl_trigger();
    pdl_wait();
    const int64_t M = m_dev != nullptr ? max(int64_t{0}, min(M_max, static_cast<int64_t>(*m_dev))) : M_max;
    const int lane = threadIdx.x & 31;
    const int nch = C >> 3;
    const float inv_c = 1.f / static_cast<float>(C);
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * (kLnThreads / 32) + (threadIdx.x >> 5); row < M;
         row += static_cast<int64_t>(gridDim.x) * (kLnThreads / 32)) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * C);
        float v[kChunks][8];
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            const int c = lane + 32 * i;
            const uint4 w = c < nch ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                v[i][2 * e] = bf16_bits_to_float(ws[e] & 0xFFFFu);
                v[i][2 * e + 1] = bf16_bits_to_float(ws[e] >> 16);
                s += v[i][2 * e] + v[i][2 * e + 1];
            }
        }
        const float mean = warp_sum(s) * inv_c;
        float q = 0.f;
#pragma unroll
        for (int i = 0; i < kChunks; ++i)
            if (lane + 32 * i < nch) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float d = v[i][e] - mean;
                    q = fmaf(d, d, q);
                }
            }
        const float rstd = rsqrtf(warp_sum(q) * inv_c + eps);
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                const uint4 g = __ldg(reinterpret_cast<const uint4 *>(gamma) + c);
                const uint4 b = __ldg(reinterpret_cast<const uint4 *>(beta) + c);
                const uint32_t gs[4] = {g.x, g.y, g.z, g.w}, bs[4] = {b.x, b.y, b.z, b.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float y0 = (v[i][2 * e] - mean) * rstd * bf16_bits_to_float(gs[e] & 0xFFFFu) +
                                     bf16_bits_to_float(bs[e] & 0xFFFFu);
                    const float y1 = (v[i][2 * e + 1] - mean) * rstd * bf16_bits_to_float(gs[e] >> 16) +
                                     bf16_bits_to_float(bs[e] >> 16);
                    o[e] = pack_bf16x2(y0, y1);
                }
                reinterpret_cast<uint4 *>(y + row * C)[c] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

// ---- host side -----------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
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

// A row-major bf16 matrix [rows, K] seen as 2-D (k, row); box = 64 k x box_rows rows, 128-byte
// swizzle (one box row is one swizzle span).
bool make_tmap_2d(CUtensorMap *map, const void *ptr, int64_t rows, int K, int box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr)
        return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(GK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int GN>
cudaError_t set_linear_smem()
{
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && done[dev])
        return cudaSuccess;
    e = cudaFuncSetAttribute(linear_kernel<GN>, cudaFuncAttributeMaxDynamicSharedMemorySize, LinCfg<GN>::kSmem);
    if (e == cudaSuccess && dev < 64)
        done[dev] = true;
    return e;
}

template <int GN>
cudaError_t launch_linear_gn(const LinearArgs &a, int num_sms, cudaStream_t stream)
{
    alignas(64) CUtensorMap tx, tw;
    if (!make_tmap_2d(&tx, a.x, a.M, a.K, GM) || !make_tmap_2d(&tw, a.w, a.N, a.K, GN))
        return cudaErrorInvalidValue;
    LinParams p{};
    p.M = static_cast<int>(a.M);
    p.m_dev = a.m_dev;
    p.N = a.N;
    p.K = a.K;
    p.bias = static_cast<const uint16_t *>(a.bias);
    p.residual = static_cast<const uint16_t *>(a.residual);
    for (int j = 0; j < a.n_outs; ++j)
        p.outs[j] = static_cast<uint16_t *>(a.outs[j]);
    p.n_outs = a.n_outs;
    p.out_ld = a.N / a.n_outs;
    p.act = a.act;
    p.err = a.err;
    p.wait_ns = a.wait_ns;
    cudaError_t e = set_linear_smem<GN>();
    if (e != cudaSuccess)
        return e;
    const int64_t tiles = ((a.M + GM - 1) / GM) * (a.N / GN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    return launch_pdl(linear_kernel<GN>, dim3(grid), dim3(kLinThreads), LinCfg<GN>::kSmem, stream, tx, tw, p);
}

}  // namespace

cudaError_t launch_linear(const LinearArgs &a, int num_sms, cudaStream_t stream)
{
    if (a.M == 0)
        return cudaSuccess;
    // the widest tile that does not straddle two outputs
    return (a.N / a.n_outs) % 256 == 0 ? launch_linear_gn<256>(a, num_sms, stream)
                                       : launch_linear_gn<128>(a, num_sms, stream);
}

cudaError_t launch_layernorm(const void *x, const void *gamma, const void *beta, void *y, int64_t M,
                             const int32_t *m_dev, int C, float eps, int num_sms, cudaStream_t stream)
{
    if (M == 0)
        return cudaSuccess;
    const int64_t blocks_needed = (M + kLnThreads / 32 - 1) / (kLnThreads / 32);
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    const int chunks = (C / 8 + 31) / 32;
    auto go = [&](auto kernel) {
        return launch_pdl(kernel, dim3(grid), dim3(kLnThreads), 0, stream, static_cast<const uint16_t *>(x),
                          static_cast<const uint16_t *>(gamma), static_cast<const uint16_t *>(beta),
                          static_cast<uint16_t *>(y), M, m_dev, C, eps);
    };
    if (chunks <= 1)
        return go(layernorm_kernel<1>);
    if (chunks == 2)
        return go(layernorm_kernel<2>);
    if (chunks == 3)
        return go(layernorm_kernel<3>);
    if (chunks == 4)
        return go(layernorm_kernel<4>);
    return go(layernorm_kernel<kLnMaxChunks>);
}

}  // namespace rra
