// attend.cu -- bidirectional ragged attention on tcgen05 tensor cores (sm_100a).
//
// What it computes ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// sota2.com card, Abstract: a bidirectional attention kernel over the variable-length
// sequences left after token pruning): for every image b, head h and kept token i,
//     o_i = sum_j softmax_j(scale * q_i . k_j) v_j,   j over all L_b kept tokens of image b.
//
// How (B200-specific design, not the pages' Triton kernel):
//   * one persistent block per SM walks a list of (image, 128-row q-tile, head) work items
//     derived from cu_seqlens on the device, so the host never learns T; each item is taken
//     in steps of 128 keys;
//   * the block owns all 512 TMEM columns: an S buffer (fp32 [128 x 128]) and an O buffer
//     (fp32 [128 x 80]) for each of two softmax groups that work on alternate items, so one
//     group's QK^T and PV run on the tensor core while the other group's softmax runs;
//   * warps specialise:
//       warps 0..1  producer: Q tiles (2-slot ring) and 128-key K/V chunks (3-slot ring) of one
//                   head; on the packed path warp 0 fetches them straight from the [T, H, 64]
//                   layout with TMA (3-D tensor map, head = coordinate, 128-byte swizzle), on
//                   the single-launch path warps 0 and 1 gather them with cp.async;
//       warps 2..3  tensor-core issuers, one per softmax group: S = Q K^T (smem x smem) and
//                   O += P V (P from TMEM as the A operand), fp32 accumulation, completion
//                   signalled through mbarriers -- two issuing threads keep the tensor core busy
//                   with both groups' short instruction bursts at once;
//       warps 4..11 softmax: two groups of four warps take alternate items; in a group, thread
//                   r owns row r of its S and O buffers (TMEM lane r), so the row max and row sum
//                   need no exchange; it writes P back over its own S columns, rescales its row
//                   of O in TMEM when the running max rises, and finally normalises and stores
//                   the row -- while the other group's QK^T, softmax and PV run alongside;
//       warp 12     (single-launch path) builds each item's kept-row list ahead of the gathers;
//   * for bf16 inputs P is split into a bf16 head and a bf16 remainder (two PV MMAs), which
//     keeps P at ~16 significant bits; fp16 P (11 bits) is used as is;
//   * the PV MMA runs with N = 80: the 64 columns of V plus a constant tile whose first column
//     is all ones, so column 64 of O accumulates the row sum of exactly the P that was used --
//     the softmax warps never add up P themselves;
//   * key rows past the sequence end get probability 0 and the matching V rows are zeroed in
//     shared memory, so whatever bytes lie there (the next image, or uninitialised capacity
//     rows) never reach the output;
//   * every wait is bounded in time; on expiry the block records RRA_ERR_TIMEOUT, raises a
//     block-wide abort flag, drains the copies and MMAs it issued, frees TMEM and leaves.
//
// The same kernel body, instantiated with kFused, runs the whole pack -> attend -> unpack call
// in one launch (the pages' pipeline without its two copies through HBM): the block derives
// the kept counts of every image from the keep mask itself, the producer gathers the kept rows
// of the padded Q/K/V straight into the swizzled tiles with 16-byte cp.async (32 lanes, one
// coalesced 128-byte row segment per 8 lanes), and the epilogue writes each output row back to
// its padded position and zero-fills the pruned rows of its (image, head).
#include <cuda.h>

#include <mutex>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int BM = 128;                 // query rows per tile (TMEM lanes)
constexpr int BN = 128;                 // keys per step
constexpr int kD = 64;                  // head dim
constexpr int kThreads = 416;           // 13 warps: 2 x copier, 2 x MMA issuer, 8 x softmax, list builder
// producer warps: warp 0 fills the Q/K/V rings (TMA on the packed path; on the single-launch path
// warps 0 and 1 share the cp.async gathers), warp 12 (single-launch path) builds the kept-row
// lists ahead of them
constexpr int kCopyWarps = 2;
constexpr int kListWarp = 12;
constexpr int kMmaWarp0 = 2;            // warp 2 issues group 1's tensor-core work, warp 3 group 0's
constexpr int kSoftmaxWarp0 = 4;
constexpr int kSoftmaxWarps = 8;        // two groups of four, one per TMEM lane quarter each
constexpr int kGroupWarps = 4;
static_assert(kSoftmaxWarp0 + kSoftmaxWarps == kListWarp && kListWarp + 1 == kThreads / 32 &&
                  kSoftmaxWarps == 2 * kGroupWarps,
              "warp roles");
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S buffers at 0 and 128 (the P of each 32-key slice is written back over the
// slice's own S columns: 16 columns of packed head values, then 16 of bf16 remainders), O
// buffers of 80 columns (64 outputs, the row sum, 15 zeros) at 256 and 352.
constexpr uint32_t kColS0 = 0;
constexpr uint32_t kColO0 = 256;
constexpr uint32_t kOCols = 96;         // stride between the two O buffers
constexpr uint32_t kPvN = 80;
constexpr uint32_t kTileBytes = 128 * 128;
constexpr int kQStages = 2;
constexpr int kKVStages = 3;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQStages * kTileBytes;
constexpr uint32_t kOffV = kOffK + kKVStages * kTileBytes;
constexpr uint32_t kOffOnes = kOffV + kKVStages * kTileBytes;   // [128 keys x 64] MN-major, column 0 = 1
constexpr uint32_t kOffBar = kOffOnes + kTileBytes;
// fused: 4 slots, each the kept positions of one item's image (int16 [kFusedMaxN]), the byte
// offsets of those padded rows' first head (int32 [kFusedMaxN]) and the kept-bit mask
// (uint32 [kFusedMaxN / 32])
constexpr int kIdxSlots = 4;
constexpr uint32_t kIdxSlotBytes = kFusedMaxN * 2 + kFusedMaxN * 4 + kFusedMaxN / 8;
// the block's first work items, decoded once in the prologue (Item: 5 ints each)
constexpr int kItemTable = 64;
constexpr uint32_t kOffItems = kOffBar + 512;
constexpr uint32_t kOffIdx = kOffItems + kItemTable * 20;
// tile_pre[B+1], then cu[B+1]: after the list slots on the fused path, in their place otherwise
template <bool kFused>
constexpr uint32_t off_tile()
{
    return kFused ? kOffIdx + kIdxSlots * kIdxSlotBytes : kOffIdx;
}
template <bool kFused>
constexpr int smem_bytes(int B)
{
    return 1024 /*align slack*/ + static_cast<int>(off_tile<kFused>()) + 2 * (B + 1) * 4;
}

struct Params {
    const int32_t *cu;      // packed path: cu_seqlens in
    const uint8_t *mask;    // fused path: keep mask [B, N]
    const uint8_t *src[3];  // fused path: padded Q, K, V [B*N, H, 64]
    int32_t *cu_out;        // fused path: cu_seqlens out (may be null)
    void *out;
    int B, H, N;
    int64_t capacity;
    float scale_log2;
    int out_dt;
    int32_t *err;
    uint64_t wait_ns;
};

constexpr uint64_t kDrainNs = 2000000000ull;

struct Bars {
    uint64_t q_full[kQStages], q_empty[kQStages];
    // kv_full[slot][g]: the fill of a K/V slot for an item of softmax group g.  A slot carries
    // both groups' chunks, but each group's issuer waits only on its own barrier, whose phases
    // then advance one fill at a time from its point of view (a parity wait never sees a phase
    // two ahead or two behind).
    uint64_t kv_full[kKVStages][2], kv_empty[kKVStages];
    uint64_t s_full[2], p_full[2], s_free[2];
    uint64_t o_full[2], o_free[2];
    uint64_t idx_full[4], idx_free[4];  // fused: kept-row list slots, one per item in flight
    uint64_t drain[2];
    uint32_t tmem_slot;
    int abort;
    int warp_sums[2][kThreads / 32];
};
static_assert(sizeof(Bars) <= 512, "barrier block overflows its slot");
static_assert(smem_bytes<false>(kAttendMaxBatch) <= 232448, "packed path exceeds shared memory");
static_assert(smem_bytes<true>(kFusedMaxBatch) <= 232448, "single-launch path exceeds shared memory");

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

// Bit k of the result is set iff byte k of the 16-byte chunk is nonzero.
__device__ __forceinline__ uint32_t kept_bits16_(uint4 c)
{
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t t = (((w[i] & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w[i]) & 0x80808080u;
        m |= (((t >> 7) & 1u) | ((t >> 14) & 2u) | ((t >> 21) & 4u) | ((t >> 28) & 8u)) << (4 * i);
    }
    return m;
}

// Bits k (0..15) with lo <= s + k < hi.
__device__ __forceinline__ uint32_t range16_(int64_t s, int64_t lo, int64_t hi)
{
    const int64_t a = lo - s, b = hi - s;
    const int l = a < 0 ? 0 : (a > 16 ? 16 : static_cast<int>(a));
    const int h = b < 0 ? 0 : (b > 16 ? 16 : static_cast<int>(b));
    return h > l ? (((1u << h) - 1u) & ~((1u << l) - 1u)) : 0u;
}

// One decoded work item.
struct Item {
    int b, h, qt, seq0, L;
};
static_assert(sizeof(Item) == 20, "item table entry size");

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
__device__ __noinline__ bool wait_or_abort_slow(uint64_t *bar, uint32_t parity, Bars *bars, const Params &p)
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

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Bars *bars, const Params &p)
{
    return mbar_test_wait(bar, parity) || wait_or_abort_slow(bar, parity, bars, p);
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

template <bool kBF16>
__device__ __forceinline__ void pack_pair(uint32_t (&r)[32], int i, float p0, float p1)
{
    if constexpr (kBF16) {
        const uint32_t a = __float_as_uint(p0), b = __float_as_uint(p1);
        float l0, l1;
        sub2(l0, l1, p0, p1, __uint_as_float(a & 0xFFFF0000u), __uint_as_float(b & 0xFFFF0000u));
        r[2 * i] = __byte_perm(a, b, 0x7632);
        r[2 * i + 1] = __byte_perm(__float_as_uint(l0), __float_as_uint(l1), 0x7632);
    } else {
        r[2 * i] = pack_f16(p0, p1);
    }
}

// Exponentials of one 32-key slice of a row (keys c .. c+31, those >= nk masked to 0), packed
// in place and written back over the slice's own TMEM columns as the PV A operand: 16 columns of
// packed head values, then for bf16 16 columns of remainders.
//   bf16: head = the top 16 bits of each fp32 value (truncation), remainder = the exact
//         difference truncated the same way, so head + remainder carries p to a relative error
//         below 2^-14 and the split costs integer byte permutes only (no conversions);
//   fp16: p rounded to nearest fp16 (11 significant bits).
// Packed pairs land in r[2i] (head) and r[2i+1] (remainder).
template <bool kBF16>
__device__ __forceinline__ void softmax_slice(uint32_t (&r)[32], int c, int nk, float scale_log2, float neg_m,
                                              uint32_t taddr)
{
    if (c + 32 <= nk) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float x0, x1;
            fma2_scalar(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scale_log2, neg_m);
            pack_pair<kBF16>(r, i, ex2_approx(x0), ex2_approx(x1));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float x0, x1;
            fma2_scalar(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scale_log2, neg_m);
            pack_pair<kBF16>(r, i, c + 2 * i < nk ? ex2_approx(x0) : 0.f, c + 2 * i + 1 < nk ? ex2_approx(x1) : 0.f);
        }
    }
    tmem_st16_strided<0>(taddr, r);
    if constexpr (kBF16)
        tmem_st16_strided<1>(taddr + 16, r);
}

__device__ __forceinline__ float slice_max(const uint32_t (&r)[32], int c, int nk, float mx)
{
    // two independent chains of three-input maxima
    float t0 = mx, t1 = -INFINITY;
    if (c + 32 <= nk) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            t0 = fmax3(t0, __uint_as_float(r[j]), __uint_as_float(r[j + 1]));
            t1 = fmax3(t1, __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            t0 = fmax3(t0, c + j < nk ? __uint_as_float(r[j]) : -INFINITY,
                       c + j + 1 < nk ? __uint_as_float(r[j + 1]) : -INFINITY);
            t1 = fmax3(t1, c + j + 2 < nk ? __uint_as_float(r[j + 2]) : -INFINITY,
                       c + j + 3 < nk ? __uint_as_float(r[j + 3]) : -INFINITY);
        }
    }
    return fmaxf(t0, t1);
}

// Store 32 normalised output values (columns col0 .. col0+31 of one row) in the output type.
__device__ __forceinline__ void store_row(const Params &p, int64_t off, const uint32_t (&r)[32], int col0, float inv)
{
    if (p.out_dt == RRA_F32) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + off + col0);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(r[4 * j]) * inv, __uint_as_float(r[4 * j + 1]) * inv,
                                 __uint_as_float(r[4 * j + 2]) * inv, __uint_as_float(r[4 * j + 3]) * inv);
    } else {
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + off + col0);
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

// Fused path: copier warp w (of kCopyWarps) copies its share of one tile of up to 128 kept rows
// of one head from the padded tensor into the 128-byte-swizzled layout with 16-byte cp.async:
// row r of the tile is the image's kept row base + r.  The chunks go in groups of 32 (one per
// lane, 8 lanes per 128-byte row, so each row is one coalesced segment), group g to warp g % 2.
// Completion arrives on `bar` once per copier lane.
__device__ __forceinline__ void copy_tile_async(uint8_t *tile, const uint8_t *src, uint64_t *bar, const int32_t *offs,
                                                int base, int count, int w, int lane)
{
    // src points at this head's 128 bytes of the image's padded row 0; offs[] holds the byte
    // offsets of the kept rows from there.  Rows at or past `count` are not copied: their S
    // columns are masked, their V rows zeroed before use, or (Q) their output never stored.
    const uint32_t tile_s = smem_addr(tile);
    const int groups = (count * 8 + 31) >> 5;
#pragma unroll 4
    for (int grp = w; grp < groups; grp += kCopyWarps) {
        const int i = lane + 32 * grp;
        const int r = i >> 3, c = i & 7;
        if (r < count) {
            const uint8_t *gsrc = src + offs[base + r] + c * 16;
            const uint32_t d = tile_s + r * 128 + ((c ^ (r & 7)) << 4);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
        }
    }
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

template <bool kBF16, bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bars = reinterpret_cast<Bars *>(base + kOffBar);
    int32_t *tile_pre = reinterpret_cast<int32_t *>(base + off_tile<kFused>());  // [B+1]
    int32_t *cu_s = tile_pre + (p.B + 1);                               // [B+1]
    auto idx_list = [&](int slot) { return reinterpret_cast<int16_t *>(base + kOffIdx + slot * kIdxSlotBytes); };
    auto idx_offs = [&](int slot) {
        return reinterpret_cast<int32_t *>(base + kOffIdx + slot * kIdxSlotBytes + kFusedMaxN * 2);
    };
    auto idx_bits = [&](int slot) {
        return reinterpret_cast<uint32_t *>(base + kOffIdx + slot * kIdxSlotBytes + kFusedMaxN * 6);
    };

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = p.B, H = p.H;
    pdl_trigger();

    if (tid == 0) {
        if constexpr (!kFused) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        // full barriers: one TMA arrival with transaction bytes, or (fused) one cp.async
        // arrival per producer lane
        const uint32_t fills = kFused ? 32u * kCopyWarps : 1u;
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&bars->q_full[s], fills);
            mbar_init(&bars->q_empty[s], 1);
        }
        for (int s = 0; s < kKVStages; ++s) {
            mbar_init(&bars->kv_full[s][0], kFused ? 2u * fills : fills);
            mbar_init(&bars->kv_full[s][1], kFused ? 2u * fills : fills);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->p_full[s], kGroupWarps);  // one arrival per warp of softmax group s
            mbar_init(&bars->s_free[s], 1);
            mbar_init(&bars->o_full[s], 1);
            mbar_init(&bars->o_free[s], kGroupWarps);
        }
        for (int s = 0; s < kIdxSlots; ++s) {
            mbar_init(&bars->idx_full[s], 1);
            mbar_init(&bars->idx_free[s], kGroupWarps);
        }
        mbar_init(&bars->drain[0], 1);
        mbar_init(&bars->drain[1], 1);
        bars->abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars->tmem_slot, kTmemCols);
        tmem_relinquish();
    }

    // ---- constant ones tile: 128 key rows of 128 bytes in the 128-byte-swizzled layout, element 0
    // of every row = 1.0 (the 16-byte chunk c of row r sits at chunk c ^ (r % 8))
    {
        uint8_t *ones = base + kOffOnes;
        const uint32_t one = kBF16 ? 0x3F80u : 0x3C00u;
        for (int i = tid; i < 128 * 8; i += kThreads) {
            const int r = i >> 3, c = i & 7;
            const uint4 v = make_uint4(c == (r & 7) ? one : 0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(ones + r * 128 + c * 16) = v;
        }
        fence_proxy_async_smem();
    }

    // everything above is private to the block; the inputs may come from the previous kernel
    pdl_wait();

    // ---- work list: tile_pre[b] = number of 128-row query tiles of images < b; cu staged too.
    if constexpr (kFused) {
        // kept tokens per image, counted from 16-byte chunks of the flat mask into cu_s[b+1]
        const uintptr_t addr = reinterpret_cast<uintptr_t>(p.mask);
        const int off = static_cast<int>(addr & 15u);
        const uint4 *m16 = reinterpret_cast<const uint4 *>(addr - off);
        // a warp per image, six images per warp at a time: lane l loads 16-byte chunks l,
        // l + 32, ... of each image's byte range (coalesced), all loads of a round issued before
        // any is used; the counts are summed with one warp reduction per image
        constexpr int kImg = 6;
        for (int bw = warp * kImg; bw < B; bw += (kThreads / 32) * kImg) {
            int64_t lo[kImg], c0[kImg], c1[kImg];
            int cnt[kImg];
#pragma unroll
            for (int i = 0; i < kImg; ++i) {
                const int b = min(bw + i, B - 1);
                lo[i] = static_cast<int64_t>(b) * p.N;
                c0[i] = (off + lo[i]) >> 4;
                c1[i] = (off + lo[i] + p.N + 15) >> 4;
                cnt[i] = 0;
            }
            for (int k = 0; k * 32 < p.N / 16 + 2; ++k) {
                uint4 w[kImg];
#pragma unroll
                for (int i = 0; i < kImg; ++i) {
                    const int64_t j = c0[i] + lane + 32 * k;
                    w[i] = j < c1[i] ? __ldg(m16 + j) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int i = 0; i < kImg; ++i)
                    cnt[i] += __popc(kept_bits16_(w[i]) &
                                     range16_((c0[i] + lane + 32 * k) * 16 - off, lo[i], lo[i] + p.N));
            }
#pragma unroll
            for (int i = 0; i < kImg; ++i) {
                const int sum = __reduce_add_sync(0xffffffffu, cnt[i]);
                if (lane == 0 && bw + i < B)
                    cu_s[bw + i + 1] = sum;
            }
        }
        __syncthreads();
    }
    if (tid == 0)
        tile_pre[0] = 0;
    int carry_t = 0, carry_l = 0;
    for (int c0 = 0; c0 < B; c0 += kThreads) {
        const int b = c0 + tid;
        int tiles = 0, len = 0;
        if (b < B) {
            if constexpr (kFused) {
                len = cu_s[b + 1];
                tiles = (len + BM - 1) / BM;
            } else {
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
        }
        int it_incl = tiles, l_incl = len;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, it_incl, off);
            const int c = __shfl_up_sync(0xffffffffu, l_incl, off);
            if (lane >= off) {
                it_incl += a;
                l_incl += c;
            }
        }
        if (lane == 31) {
            bars->warp_sums[0][warp] = it_incl;
            bars->warp_sums[1][warp] = l_incl;
        }
        __syncthreads();
        int before_t = carry_t, before_l = carry_l, chunk_t = 0, chunk_l = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            before_t += (w < warp) ? bars->warp_sums[0][w] : 0;
            before_l += (w < warp) ? bars->warp_sums[1][w] : 0;
            chunk_t += bars->warp_sums[0][w];
            chunk_l += bars->warp_sums[1][w];
        }
        if (b < B) {
            tile_pre[b + 1] = before_t + it_incl;
            if constexpr (kFused)
                cu_s[b + 1] = before_l + l_incl;  // (reads of the count above happened before the barrier)
        }
        carry_t += chunk_t;
        carry_l += chunk_l;
        __syncthreads();
    }
    if constexpr (kFused) {
        if (tid == 0)
            cu_s[0] = 0;
        __syncthreads();
        if (blockIdx.x == 0 && p.cu_out != nullptr)
            for (int b = tid; b <= B; b += kThreads)
                p.cu_out[b] = cu_s[b];
        // images without kept tokens have no work item: their padded output rows are zeroed here
        const int out_vecs = (p.out_dt == RRA_F32 ? 4 * kD : 2 * kD) / 16;  // 16-byte vectors per head row
        for (int b = blockIdx.x; b < B; b += gridDim.x) {
            if (cu_s[b + 1] != cu_s[b])
                continue;
            uint4 *y = reinterpret_cast<uint4 *>(p.out) + static_cast<int64_t>(b) * p.N * H * out_vecs;
            for (int64_t i = tid; i < static_cast<int64_t>(p.N) * H * out_vecs; i += kThreads)
                y[i] = make_uint4(0, 0, 0, 0);
        }
    }

    // decode the block's first items once: every role walks the same list
    Item *items = reinterpret_cast<Item *>(base + kOffItems);
    {
        const int total = tile_pre[B] * H;
        for (int k = tid; k < kItemTable; k += kThreads) {
            const int item = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
            if (item < total)
                items[k] = decode_item(item, H, B, tile_pre, cu_s);
        }
    }
    auto item_at = [&](int k, int item) {
        return k < kItemTable ? items[k] : decode_item(item, H, B, tile_pre, cu_s);
    };

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;
    const int total_items = tile_pre[B] * H;
    // work items of this block, dealt round-robin: a block's items come from unrelated images,
    // which evens out the per-block cost
    const int item_first = static_cast<int>(blockIdx.x);
    const int item_end = total_items;
    const int item_step = static_cast<int>(gridDim.x);

    if (kFused && warp == kListWarp) {
        // ================================================================ kept-row lists
        // Item n's list goes to slot n % 4, free once the epilogue of item n-4 has used it (the
        // copier is done with a list before that epilogue can run); this warp runs up to four
        // items ahead of the copier.
        uint32_t idx_phase = 0;
        int cur_b = -1, prev_slot = 0, n = 0;
        bool ok = true;
        for (int item = item_first; ok && item < item_end; item += item_step, ++n) {
            const Item it = item_at(n, item);
            const int row_off = it.b * p.N;
            const int islot = n & (kIdxSlots - 1);
            int16_t *list = idx_list(islot);
            uint32_t *bits = idx_bits(islot);
            int32_t *offs = idx_offs(islot);
            const int nwords = (p.N + 31) / 32;
            ok = warp_wait(&bars->idx_free[islot], ((idx_phase >> islot) & 1u) ^ 1u, bars, p);
            if (!ok)
                break;
            idx_phase ^= 1u << islot;
            if (it.b == cur_b) {
                // same image as the previous item: copy its list
                const int16_t *pl = idx_list(prev_slot);
                const int32_t *po = idx_offs(prev_slot);
                const uint32_t *pb = idx_bits(prev_slot);
                for (int i = lane; i < it.L; i += 32) {
                    list[i] = pl[i];
                    offs[i] = po[i];
                }
                for (int i = lane; i < nwords; i += 32)
                    bits[i] = pb[i];
            } else {
                // kept positions of this image in order: mask bytes fetched 8 words of 32 at a
                // time (independent loads), then one ballot per word
                int running = 0;
                for (int w0 = 0; w0 < nwords; w0 += 8) {
                    bool keep[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int tok = (w0 + u) * 32 + lane;
                        keep[u] = tok < p.N && p.mask[row_off + tok] != 0;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const unsigned bal = __ballot_sync(0xffffffffu, keep[u]);
                        if (w0 + u < nwords) {
                            if (keep[u]) {
                                const int slot_i = running + __popc(bal & ((1u << lane) - 1u));
                                const int tok = (w0 + u) * 32 + lane;
                                list[slot_i] = static_cast<int16_t>(tok);
                                offs[slot_i] = tok * H * kD * 2;  // < 2^31 (checked on the host)
                            }
                            if (lane == 0)
                                bits[w0 + u] = bal;
                            running += __popc(bal);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->idx_full[islot]);
            cur_b = it.b;
            prev_slot = islot;
        }
    } else if (warp < (kFused ? kCopyWarps : 1)) {
        // ================================================================ producer
        // Empty-slot waits use the usual parity idiom: on a fresh barrier the phase "before"
        // phase 0 counts as complete, so waiting on parity (phase ^ 1) passes at once for the
        // first fill of each slot, then tracks the consumer's releases.
        uint32_t q_phase = 0, kv_phase = 0;  // one bit per slot
        uint32_t idxf_phase = 0, n_items = 0;
        uint32_t q_issued = 0;
        uint32_t kv_par = 0, kv_any = 0;  // per kv_full barrier (bit 2*slot+group): fill-count parity, any fill
        int qs = 0, ks = 0;
        bool ok = true;
        for (int item = item_first; ok && item < item_end; item += item_step) {
            const Item it = item_at(static_cast<int>(n_items), item);
            const int nkc = (it.L + BN - 1) / BN;
            const int row_off = it.b * p.N;  // fused: first padded row of this image
            const int islot = static_cast<int>(n_items & (kIdxSlots - 1));
            if constexpr (kFused) {
                // the kept-row list of this item (built by the list warp)
                ok = warp_wait(&bars->idx_full[islot], (idxf_phase >> islot) & 1u, bars, p);
                if (!ok)
                    break;
                idxf_phase ^= 1u << islot;
            }
            ok = warp_wait(&bars->q_empty[qs], ((q_phase >> qs) & 1u) ^ 1u, bars, p);
            if (!ok)
                break;
            q_phase ^= 1u << qs;
            // fused: this head's 128 bytes of the image's padded row 0 in Q, K, V
            const int64_t head0 = (static_cast<int64_t>(row_off) * H + it.h) * kD * 2;
            if constexpr (kFused) {
                const int q0 = it.qt * BM;
                copy_tile_async(base + kOffQ + qs * kTileBytes, p.src[0] + head0, &bars->q_full[qs], idx_offs(islot), q0,
                                min(BM, it.L - q0), warp, lane);
            } else {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars->q_full[qs], kTileBytes);
                    tma_load_3d(base + kOffQ + qs * kTileBytes, &tm_q, &bars->q_full[qs], 0, it.h, it.seq0 + it.qt * BM);
                }
            }
            __syncwarp();
            ++q_issued;
            qs = (qs + 1 == kQStages) ? 0 : qs + 1;
            for (int kc = 0; kc < nkc; ++kc) {
                ok = warp_wait(&bars->kv_empty[ks], ((kv_phase >> ks) & 1u) ^ 1u, bars, p);
                if (!ok)
                    break;
                kv_phase ^= 1u << ks;
                uint64_t *full = &bars->kv_full[ks][n_items & 1u];  // the owning group's barrier
                if constexpr (kFused) {
                    const int cnt = min(BN, it.L - kc * BN);
                    copy_tile_async(base + kOffK + ks * kTileBytes, p.src[1] + head0, full, idx_offs(islot), kc * BN,
                                    cnt, warp, lane);
                    copy_tile_async(base + kOffV + ks * kTileBytes, p.src[2] + head0, full, idx_offs(islot), kc * BN,
                                    cnt, warp, lane);
                } else {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(full, 2 * kTileBytes);
                        tma_load_3d(base + kOffK + ks * kTileBytes, &tm_k, full, 0, it.h, it.seq0 + kc * BN);
                        tma_load_3d(base + kOffV + ks * kTileBytes, &tm_v, full, 0, it.h, it.seq0 + kc * BN);
                    }
                }
                __syncwarp();
                {
                    const uint32_t bit = 1u << (2 * ks + (n_items & 1u));  // barrier kv_full[ks][group]
                    kv_par ^= bit;
                    kv_any |= bit;
                }
                ks = (ks + 1 == kKVStages) ? 0 : ks + 1;
            }
            ++n_items;
        }
        // drain: every issued fill has landed before the block may leave
        if constexpr (kFused)
            asm volatile("cp.async.wait_all;" ::: "memory");
        for (int s = 0; s < kQStages; ++s) {
            const uint32_t n = q_issued / kQStages + (static_cast<uint32_t>(s) < q_issued % kQStages ? 1u : 0u);
            if (n > 0)
                mbar_wait_bounded(&bars->q_full[s], (n - 1) & 1u, kDrainNs);
        }
        for (int s = 0; s < kKVStages; ++s)
            for (int gg = 0; gg < 2; ++gg) {
                const uint32_t bit = 1u << (2 * s + gg);
                if (kv_any & bit)  // the last fill has parity (count - 1) & 1
                    mbar_wait_bounded(&bars->kv_full[s][gg], (kv_par & bit) ? 0u : 1u, kDrainNs);
            }
    } else if (warp == kMmaWarp0 || warp == kMmaWarp0 + 1) {
        // ================================================================ tcgen05 issuers
        // One issuing thread per softmax group (warp 3: group 0, warp 2: group 1), so the two
        // groups' tensor-core work is issued concurrently.  Group g owns the items n = g, g+2, ...
        // of the block, S buffer g and O buffer g; for each 128-key chunk of its items its issuer
        // runs S = Q K^T, waits for the softmax to write P over S, then O += P V.  The Q/K/V rings
        // are filled in item order for both groups, so each issuer walks every item and, for the
        // other group's, only advances its ring positions and phase bits.
        const int g = kMmaWarp0 + 1 - warp;
        uint32_t q_ph = 0, kv_ph = 0, p_ph = 0, sfree_ph = 0, ofree_ph = 0;
        const uint32_t idPV = idesc_f16(BM, kPvN, kBF16 ? 1u : 0u, 1u);
        // shared-memory descriptors of the ring slots: stepping K inside a 128-byte swizzled row
        // adds 32 bytes (2 units) to the start address, stepping 16 key rows adds 2048 bytes (128
        // units), and a slot is 1024 units further.  V descriptors carry, as leading offset, the
        // distance to the ones tile that supplies PV columns 64..79.
        const uint64_t qdesc0 = smem_desc_sw128(smem_addr(base + kOffQ), 16, 1024);
        const uint64_t kdesc0 = smem_desc_sw128(smem_addr(base + kOffK), 16, 1024);
        const uint64_t vdesc0 = smem_desc_sw128(smem_addr(base + kOffV), kOffOnes - kOffV, 1024);
        auto slot_desc = [](uint64_t d0, int slot) { return d0 + static_cast<uint64_t>(slot) * (kTileBytes >> 4); };
        const uint32_t dS = tmem + kColS0 + 128 * g;
        const uint32_t dO = tmem + kColO0 + kOCols * g;
        int qs = 0, ks = 0, n = 0;
        bool s_busy = false, ok = true;
        for (int item = item_first; ok && item < item_end; item += item_step, ++n) {
            const int nkc = (item_at(n, item).L + BN - 1) / BN;
            if ((n & 1) != g) {
                // the other group's item: its Q slot is never ours (item n uses slot n % 2), and
                // its K/V chunks pass through the same slots but signal the other group's
                // barriers -- only the ring positions advance
                q_ph ^= 1u << qs;
                qs = (qs + 1 == kQStages) ? 0 : qs + 1;
                ks = (ks + nkc) % kKVStages;
                continue;
            }
            const int L = item_at(n, item).L;
            ok = warp_wait(&bars->q_full[qs], (q_ph >> qs) & 1u, bars, p);
            if (!ok)
                break;
            q_ph ^= 1u << qs;
            for (int kc = 0; kc < nkc; ++kc) {
                const int nk = min(BN, L - kc * BN);
                const int nk16 = (nk + 15) & ~15;
                ok = warp_wait(&bars->kv_full[ks][g], (kv_ph >> ks) & 1u, bars, p);
                if (!ok)
                    break;
                kv_ph ^= 1u << ks;
                uint8_t *sV = base + kOffV + ks * kTileBytes;
                // zero V rows [nk, nk16): they enter the PV MMA with probability 0
                if (nk < nk16) {
                    for (int i = lane; i < (nk16 - nk) * 8; i += 32)
                        *reinterpret_cast<uint4 *>(sV + (nk + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                // the S buffer holds the previous chunk's P until that chunk's PV has completed
                if (s_busy) {
                    ok = warp_wait(&bars->s_free[g], sfree_ph, bars, p);
                    if (!ok)
                        break;
                    sfree_ph ^= 1u;
                }
                if (lane == 0) {
                    tc_fence_after();
                    if constexpr (kFused)
                        fence_proxy_async_smem();  // Q/K/V arrived through cp.async (generic proxy)
                    const uint64_t qd = slot_desc(qdesc0, qs);
                    const uint64_t kd = slot_desc(kdesc0, ks);
                    const uint32_t idS = idesc_f16(BM, nk16, kBF16 ? 1u : 0u, 0u);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss(dS, qd + 2 * kk, kd + 2 * kk, idS, kk > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full[g]);
                    if (kc == nkc - 1)
                        mma_commit(&bars->q_empty[qs]);  // last read of this Q tile
                }
                __syncwarp();
                // P of this chunk in TMEM; before the first PV of an item, the group's previous
                // item must have been read out of O
                ok = warp_wait(&bars->p_full[g], p_ph, bars, p);
                if (!ok)
                    break;
                p_ph ^= 1u;
                if (kc == 0 && n >= 2) {
                    ok = warp_wait(&bars->o_free[g], ofree_ph, bars, p);
                    if (!ok)
                        break;
                    ofree_ph ^= 1u;
                }
                if (lane == 0) {
                    tc_fence_after();
                    const uint64_t vd = slot_desc(vdesc0, ks) - (static_cast<uint64_t>(ks) * (kTileBytes >> 4) << 16);
                    const int nj = nk16 >> 4;
                    // keys 16j..16j+15 live in slice j/2: head part at column 32(j/2) + 8(j%2),
                    // remainder (bf16) 16 columns further
#pragma unroll
                    for (int j = 0; j < BN / 16; ++j)
                        if (j < nj)
                            mma_ts(dO, dS + 32 * (j >> 1) + 8 * (j & 1), vd + 128 * j, idPV, (kc > 0 || j > 0) ? 1u : 0u);
                    if (kBF16) {
#pragma unroll
                        for (int j = 0; j < BN / 16; ++j)
                            if (j < nj)
                                mma_ts(dO, dS + 32 * (j >> 1) + 8 * (j & 1) + 16, vd + 128 * j, idPV, 1u);
                    }
                    mma_commit(&bars->o_full[g]);
                    mma_commit(&bars->s_free[g]);
                    mma_commit(&bars->kv_empty[ks]);
                }
                __syncwarp();
                s_busy = true;
                ks = (ks + 1 == kKVStages) ? 0 : ks + 1;
            }
            qs = (qs + 1 == kQStages) ? 0 : qs + 1;
        }
        // drain: every MMA this thread issued has completed
        if (lane == 0) {
            mma_commit(&bars->drain[g]);
            mbar_wait_bounded(&bars->drain[g], 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp >= kSoftmaxWarp0 && warp < kSoftmaxWarp0 + kSoftmaxWarps) {
        // ================================================================ softmax + epilogue
        // Group g (4 warps) takes items n = g, g+2, ...; thread r of the group owns row r of
        // S buffer g and O buffer g (its TMEM lane), so row max and row sum need no exchange.
        const int q4 = warp & 3;                     // TMEM lane quarter of this warp
        const int g = (warp - kSoftmaxWarp0) >> 2;   // softmax group
        const int row = q4 * 32 + lane;              // row of S / O owned by this thread
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        const uint32_t sbase = lane_base + kColS0 + 128 * g;
        const uint32_t obase = lane_base + kColO0 + kOCols * g;
        uint32_t s_ph = 0, o_ph = 0, idxf_ph = 0;
        bool ok = true;
        int n = 0;
        for (int item = item_first; ok && item < item_end; item += item_step, ++n) {
            if ((n & 1) != g)
                continue;
            const Item it = item_at(n, item);
            const int nkc = (it.L + BN - 1) / BN;
            const int q0 = it.qt * BM;
            const int qrows = min(BM, it.L - q0);
            const bool warp_active = q4 * 32 < qrows;
            float m_run = -INFINITY;
            for (int kc = 0; kc < nkc; ++kc) {
                const int nk = min(BN, it.L - kc * BN);
                const int nk16 = (nk + 15) & ~15;
                ok = warp_wait(&bars->s_full[g], s_ph, bars, p);
                if (!ok)
                    break;
                s_ph ^= 1u;
                tc_fence_after();
                // pass 1, row max: two 32-key slices per TMEM round trip (a rolled loop: every
                // slice runs the same code, which keeps the kernel's instruction footprint small)
                float m_new = m_run;
                if (warp_active) {
                    float mx = -INFINITY;
#pragma unroll 1
                    for (int c = 0; c < nk; c += 64) {
                        uint32_t ra[32], rb[32];
                        tmem_ld32(sbase + c, ra);
                        tmem_ld32(sbase + c + 32, rb);  // columns past the chunk are ignored below
                        tmem_wait_ld_dep(ra);
                        tmem_wait_ld_dep(rb);
                        mx = slice_max(ra, c, nk, mx);
                        if (c + 32 < nk)
                            mx = slice_max(rb, c + 32, nk, mx);
                    }
                    m_new = fmaxf(m_run, mx);
                }
                // later chunks: the previous PV has landed in O; rescale rows whose max rose
                // (before any P of this chunk is handed over, so no PV of it can start earlier)
                if (kc > 0) {
                    ok = warp_wait(&bars->o_full[g], o_ph, bars, p);
                    if (!ok)
                        break;
                    o_ph ^= 1u;
                    tc_fence_after();
                    if (warp_active && __any_sync(0xffffffffu, m_new > m_run)) {
                        const float alpha = ex2_approx((m_run - m_new) * p.scale_log2);
#pragma unroll 1
                        for (uint32_t c = 0; c < kPvN; c += 16) {
                            uint32_t o[16];
                            tmem_ld16(obase + c, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                            tmem_st16(obase + c, o);
                        }
                    }
                }
                m_run = m_new;
                const float neg_m = -m_new * p.scale_log2;
                // pass 2: P = exp2(scale*log2e*(s - m)), one 32-key slice per round trip
                if (warp_active) {
#pragma unroll 1
                    for (int c = 0; c < nk16; c += 32) {
                        uint32_t ra[32];
                        tmem_ld32(sbase + c, ra);
                        tmem_wait_ld_dep(ra);
                        softmax_slice<kBF16>(ra, c, nk, p.scale_log2, neg_m, sbase + c);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->p_full[g]);
            }
            if (!ok)
                break;
            // epilogue: the last PV has landed; normalise by the row sum (O column 64) and store
            ok = warp_wait(&bars->o_full[g], o_ph, bars, p);
            if (!ok)
                break;
            o_ph ^= 1u;
            const int islot = n & (kIdxSlots - 1);
            if constexpr (kFused) {
                ok = warp_wait(&bars->idx_full[islot], (idxf_ph >> islot) & 1u, bars, p);
                if (!ok)
                    break;
                idxf_ph ^= 1u << islot;
            }
            tc_fence_after();
            if (warp_active) {
                uint32_t sum[1];
                tmem_ld1(obase + 64, sum);
                tmem_wait_ld();
                const float inv = 1.f / __uint_as_float(sum[0]);
                int64_t out_row = static_cast<int64_t>(it.seq0) + q0 + row;
                if constexpr (kFused)
                    out_row = static_cast<int64_t>(it.b) * p.N + idx_list(islot)[q0 + (row < qrows ? row : 0)];
                const int64_t off = (out_row * H + it.h) * kD;
#pragma unroll 1
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t r[32];
                    tmem_ld32(obase + 32 * h2, r);
                    tmem_wait_ld_dep(r);
                    if (row < qrows)
                        store_row(p, off, r, 32 * h2, inv);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->o_free[g]);
            if constexpr (kFused) {
                if (it.qt == 0) {
                    // pruned rows of this (image, head) in the padded output become zero: 16-byte
                    // stores, consecutive threads along a row
                    const uint32_t *bits = idx_bits(islot);
                    const int lg = p.out_dt == RRA_F32 ? 4 : 3;  // log2 of 16-byte vectors per head row
                    const int nvec = p.N << lg;
                    for (int i = q4 * 32 + lane; i < nvec; i += kGroupWarps * 32) {
                        const int tok = i >> lg;
                        if (!((bits[tok >> 5] >> (tok & 31)) & 1u))
                            reinterpret_cast<uint4 *>(p.out)[(((static_cast<int64_t>(it.b) * p.N + tok) * H + it.h) << lg) +
                                                             (i & ((1 << lg) - 1))] = make_uint4(0, 0, 0, 0);
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->idx_free[islot]);
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

template <bool kBF16, bool kFused>
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
    e = cudaFuncSetAttribute(attend_kernel<kBF16, kFused>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev < 64)
        done_bytes[dev] = bytes;
    return e;
}

template <bool kFused>
cudaError_t launch_variant(bool bf16, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           const Params &p, int64_t grid, int smem, cudaStream_t stream)
{
    cudaError_t e = bf16 ? set_smem_attr<true, kFused>(smem) : set_smem_attr<false, kFused>(smem);
    if (e != cudaSuccess)
        return e;
    const dim3 g(static_cast<unsigned>(grid)), blk(kThreads);
    return bf16 ? launch_pdl(attend_kernel<true, kFused>, g, blk, smem, stream, tq, tk, tv, p)
                : launch_pdl(attend_kernel<false, kFused>, g, blk, smem, stream, tq, tk, tv, p);
}

int64_t grid_for(int B, int H, int max_seqlen, int num_sms)
{
    const int64_t max_tiles = (static_cast<int64_t>(max_seqlen > 0 ? max_seqlen : 1) + BM - 1) / BM;
    int64_t grid = static_cast<int64_t>(B) * H * max_tiles;
    if (grid > num_sms)
        grid = num_sms;  // one block per SM: it owns all 512 TMEM columns
    return grid < 1 ? 1 : grid;
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
    Params p{};
    p.cu = a.cu;
    p.out = a.o;
    p.B = a.B;
    p.H = a.H;
    p.capacity = a.capacity;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out_dt = a.out_dt;
    p.err = a.err;
    p.wait_ns = a.wait_ns;
    const int smem = smem_bytes<false>(a.B);
    return launch_variant<false>(a.in_bf16, tq, tk, tv, p, grid_for(a.B, a.H, a.max_seqlen, num_sms), smem, stream);
}

cudaError_t launch_fused(const FusedArgs &a, int num_sms, cudaStream_t stream)
{
    if (a.B == 0) {
        if (a.cu_out != nullptr)
            return cudaMemsetAsync(a.cu_out, 0, sizeof(int32_t), stream);
        return cudaSuccess;
    }
    const int64_t rows = static_cast<int64_t>(a.B) * a.N;
    alignas(64) CUtensorMap unused{};  // the single-launch path copies with cp.async, not TMA
    Params p{};
    p.src[0] = static_cast<const uint8_t *>(a.q);
    p.src[1] = static_cast<const uint8_t *>(a.k);
    p.src[2] = static_cast<const uint8_t *>(a.v);
    p.mask = a.mask;
    p.cu_out = a.cu_out;
    p.out = a.y;
    p.B = a.B;
    p.H = a.H;
    p.N = a.N;
    p.capacity = rows;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out_dt = a.out_dt;
    p.err = a.err;
    p.wait_ns = a.wait_ns;
    const int smem = smem_bytes<true>(a.B);
    return launch_variant<true>(a.in_bf16, unused, unused, unused, p, grid_for(a.B, a.H, a.N, num_sms), smem, stream);
}

}  // namespace rra
