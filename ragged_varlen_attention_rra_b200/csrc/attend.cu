// attend.cu -- bidirectional ragged attention on tcgen05 tensor cores (sm_100a).
//
// What it computes ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// sota2.com card, Abstract: a bidirectional attention kernel over the variable-length
// sequences left after token pruning): for every image b, head h and kept token i,
//     o_i = sum_j softmax_j(scale * q_i . k_j) v_j,   j over all L_b kept tokens of image b.
//
// How (B200-specific design, not the pages' Triton kernel):
//   * one persistent block per SM walks a list of work items derived from cu_seqlens on the
//     device, so the host never learns T: (image, 128-row q-tile, head) when some image keeps
//     more than 64 tokens; otherwise (tile of 128 consecutive rows of the packed token space,
//     head), each tile holding the rows of several images, every query row attending only to its
//     own image's keys (a per-row key range, i.e. a block-diagonal mask); keys come in steps of
//     128;
//   * the block owns all 512 TMEM columns, 256 for each of two softmax groups that work on
//     alternate items: S (fp32 [128 x 128]), P (16-bit [128 x 128]) and O (fp32 [128 x 64]).  P
//     apart from S lets the next chunk's S = Q K^T run while this chunk's O += P V does, and one
//     group's tensor-core work runs while the other group's softmax does;
//   * warps specialise:
//       warps 0..1  producer: Q tiles (2-slot ring) and 128-key K/V chunks (4-slot ring) of one
//                   head; on the packed path warp 0 fetches them straight from the [T, H, 64]
//                   layout with TMA (3-D tensor map, head = coordinate, 128-byte swizzle), on
//                   the single-launch path warps 0 and 1 gather them with cp.async;
//       warps 2..3  tensor-core issuers, one per softmax group: S = Q K^T (smem x smem) and
//                   O += P V (P from TMEM as the A operand), fp32 accumulation, completion
//                   signalled through mbarriers;
//       warps 4..11 softmax: two groups of four warps take alternate items; in a group, thread
//                   r owns row r of its S, P and O (TMEM lane r), so the row max and row sum
//                   need no exchange (the row sum is kept in a register); it rescales its row of O
//                   in TMEM when the running max rises, and finally normalises and stores the row;
//       warp 12     (single-launch path) builds each item's kept-row list ahead of the gathers;
//       warps 13-14 prepare each V tile as soon as it lands (zero tail; for bf16 inputs an
//                   in-place conversion to fp16), each owning two of the four K/V slots;
//       warp 15     (single-launch path) clears the block's share of pruned padded rows while
//                   the rest of the block computes, one bulk copy per row from zeroed shared
//                   memory;
//   * P is rounded to fp16 (11 significant bits) and meets an fp16 V: for bf16 inputs every V
//     tile is converted in shared memory, exactly for |v| in [2^-14, 65504] and with an
//     absolute error below 2^-25 under it; a tile holding a finite |v| >= 65536 keeps bf16 and
//     meets a bf16 P;
//   * key rows past the sequence end get probability 0 and the matching V rows are zeroed in
//     shared memory, so whatever bytes lie there (the next image, or uninitialised capacity
//     rows) never reach the output;
//   * every wait is bounded in time; on expiry the block records RRA_ERR_TIMEOUT, raises a
//     block-wide abort flag, drains the copies and MMAs it issued, frees TMEM and leaves.
//
// The same kernel body, instantiated with kFused, runs the whole pack -> attend -> unpack call
// in one launch (the pages' pipeline without its two copies through HBM): the block derives
// the kept counts of every image from the keep mask itself (a warp or a thread per image,
// whichever needs fewer memory round trips), the producer gathers the kept rows
// of the padded Q/K/V straight into the swizzled tiles with 16-byte cp.async (32 lanes, one
// coalesced 128-byte row segment per 8 lanes), and the epilogue writes each output row back to
// its padded position.
#include <cuda.h>

#include <mutex>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int BM = 128;                 // query rows per tile (TMEM lanes)
constexpr int BN = 128;                 // keys per step
constexpr int kD = 64;                  // head dim
constexpr int kThreads = 512;           // 16 warps: 2 x copier, 2 x MMA issuer, 8 x softmax, list, 2 x V, zero-fill
// producer warps: warp 0 fills the Q/K/V rings (TMA on the packed path; on the single-launch path
// warps 0 and 1 share the cp.async gathers), warp 12 (single-launch path) builds the kept-row
// lists ahead of them, warps 13 and 14 prepare the V tiles for their PVs as soon as they land
// (alternate fills), warp 15 (single-launch path) zero-fills the block's share of pruned rows
constexpr int kCopyWarps = 2;
constexpr int kListWarp = 12;
constexpr int kVWarp0 = 13;
constexpr int kVWarps = 2;
constexpr int kZeroWarp = 15;
constexpr int kMmaWarp0 = 2;            // warp 2 issues group 1's tensor-core work, warp 3 group 0's
constexpr int kSoftmaxWarp0 = 4;
constexpr int kSoftmaxWarps = 8;        // two groups of four, one per TMEM lane quarter each
constexpr int kGroupWarps = 4;
static_assert(kSoftmaxWarp0 + kSoftmaxWarps == kListWarp && kListWarp + 1 == kVWarp0 && kVWarp0 + kVWarps == kZeroWarp &&
                  kZeroWarp + 1 == kThreads / 32 && kSoftmaxWarps == 2 * kGroupWarps,
              "warp roles");
constexpr uint32_t kTmemCols = 512;
// TMEM columns: 256 per softmax group g, at 256 g: S (fp32 [128 x 128]) in columns 0..127, P
// (16-bit [128 x 128], two keys per column) in 128..191, O (fp32 [128 x 64]) in 192..255.  With P
// apart from S, the next chunk's S = Q K^T can be computed while this chunk's O += P V runs.
constexpr uint32_t kGroupCols = 256;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColP = 128;
constexpr uint32_t kColO = 192;
constexpr uint32_t kTileBytes = 128 * 128;
constexpr int kQStages = 2;
constexpr int kKVStages = 4;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQStages * kTileBytes;
constexpr uint32_t kOffV = kOffK + kKVStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kKVStages * kTileBytes;
// fused: 4 slots, each the padded row index (b * N + n, int32) of every key row of one item, in
// packed order
constexpr int kIdxSlots = 4;
constexpr uint32_t kIdxSlotBytes = kFusedMaxN * 4;
// short-sequence tiling: used when no image has more than kShortMax kept tokens; a tile's keys
// then span at most 128 + 2 * (kShortMax - 1) <= 2 * BN rows
constexpr int kShortMax = 64;
// the block's first work items, decoded once in the prologue (Item: 6 ints each)
constexpr int kItemTable = 56;
constexpr uint32_t kBarBytes = 640;
constexpr uint32_t kOffItems = kOffBar + kBarBytes;
constexpr uint32_t kOffIdx = kOffItems + kItemTable * 24;
// fused: a block of zero bytes, the source of the bulk stores that clear pruned output rows
constexpr uint32_t kZeroBytes = 4096;
constexpr uint32_t kOffZero = kOffIdx + kIdxSlots * kIdxSlotBytes;
// tile_pre[B+1], then cu[B+1]: after the list slots and the zero block on the fused path, in
// their place otherwise
template <bool kFused>
constexpr uint32_t off_tile()
{
    return kFused ? kOffZero + kZeroBytes : kOffIdx;
}
template <bool kFused>
constexpr int smem_bytes(int B)
{
    return 1024 /*align slack*/ + static_cast<int>(off_tile<kFused>()) + 2 * (B + 1) * 4;
}

struct Params {
    const int32_t *cu;      // packed path: cu_seqlens in
    const uint8_t *mask;    // fused path: keep mask [B, N]
    const uint8_t *src[3];  // fused path: padded Q, K, V [B*N, H, 64]; packed path: V [capacity, H, 64] in src[2]
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
    // per softmax group: S of a chunk computed / its P written (and S read) / its PV completed /
    // its V tile ready for the PV (zero tail, fp16 or bf16 as v_fmt of its slot says) / O read out
    uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
    // v_ready[slot][g]: the V warp has prepared the slot's V tile of a chunk of group g (one
    // barrier per slot and group, like kv_full: the V warp may run a few chunks ahead of a group,
    // but never more than one fill of the same slot)
    uint64_t v_ready[kKVStages][2];
    uint64_t idx_full[4], idx_free[4];  // fused: kept-row list slots, one per item in flight
    uint64_t drain[2];
    uint32_t tmem_slot;
    int abort;
    int v_fmt[kKVStages];  // per K/V slot: 0 = its V tile (and so the chunk's P) is fp16, 1 = bf16
    int warp_sums[3][kThreads / 32];
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block overflows its slot");
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

// One decoded work item: the query rows [q0, q0 + nq) of the packed token space (one head), and
// the key rows [k0, k0 + nk) they attend to -- every kept token of each image that owns one of the
// query rows (images are contiguous in the packed space, so this is one range).  b0 is the image
// of row q0.
//   per-image tiling (some image longer than kShortMax): item = (image b, 128-row q-tile qt, h),
//     q0 = cu[b] + 128 qt, k0 = cu[b], nk = L_b: one image per item;
//   short-sequence tiling: item = (tile t of the packed space, h), q0 = 128 t: the tile's rows
//     may belong to several images, each query row attending only to its own image's keys.
struct Item {
    int b0, h, q0, nq, k0, nk;
};
static_assert(sizeof(Item) == 24, "item table entry size");

// Largest b in [lo, hi) with cu[b] <= p (cu non-decreasing, cu[lo] <= p): the image owning packed
// row p (an empty image shares its start with the next one, which is then the one returned).
__device__ __forceinline__ int image_of_row(const int32_t *cu, int lo, int hi, int p)
{
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= p)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

__device__ __forceinline__ Item decode_item(int item, int H, int B, bool short_tiles, int T, const int32_t *tile_pre,
                                            const int32_t *cu)
{
    Item it;
    const int g = item / H;
    it.h = item - g * H;
    if (short_tiles) {
        it.q0 = g * BM;
        it.nq = min(BM, T - it.q0);
        it.b0 = image_of_row(cu, 0, B, it.q0);
        const int b1 = image_of_row(cu, it.b0, B, it.q0 + it.nq - 1);
        it.k0 = cu[it.b0];
        it.nk = cu[b1 + 1] - it.k0;
    } else {
        int lo = 0, hi = B;  // tile_pre[lo] <= g < tile_pre[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tile_pre[mid] <= g)
                lo = mid;
            else
                hi = mid;
        }
        const int qt = g - tile_pre[lo];
        it.b0 = lo;
        it.k0 = cu[lo];
        it.nk = cu[lo + 1] - it.k0;
        it.q0 = it.k0 + qt * BM;
        it.nq = min(BM, it.nk - qt * BM);
    }
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

// Two fp32 probabilities packed as two 16-bit values (low half = the first), fp16 or bf16, round
// to nearest.
__device__ __forceinline__ uint32_t pack_p(float a, float b, bool f16)
{
    return f16 ? pack_f16(a, b) : pack_bf16(a, b);
}

// Exponentials of one 32-key slice of a row (keys c .. c+31; keys not set in `keys` masked to 0),
// packed as 16 columns of 16-bit pairs and written to the row's P columns at `taddr`; returns the
// slice's sum of the fp32 values.  `full` (warp-uniform) says every lane's keys cover the slice.
__device__ __forceinline__ float softmax_slice(const uint32_t (&r)[32], uint32_t keys, bool full, bool f16,
                                               float scale_log2, float neg_m, uint32_t taddr)
{
    uint32_t pk[16];
    float s0 = 0.f, s1 = 0.f;
    if (full) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float x0, x1;
            fma2_scalar(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scale_log2, neg_m);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            s0 += p0;
            s1 += p1;
            pk[i] = pack_p(p0, p1, f16);
        }
    } else {
        // masked keys enter the exponential as -inf (2^-inf = +0): a select per element, never a
        // branch, so lanes with different key ranges do not diverge (and garbage S is dropped)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float x0, x1;
            fma2_scalar(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), scale_log2, neg_m);
            x0 = ((keys >> (2 * i)) & 1u) ? x0 : -INFINITY;
            x1 = ((keys >> (2 * i + 1)) & 1u) ? x1 : -INFINITY;
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            s0 += p0;
            s1 += p1;
            pk[i] = pack_p(p0, p1, f16);
        }
    }
    tmem_st16(taddr, pk);
    return s0 + s1;
}

// P = 0 for a whole 32-key slice (no key of the slice belongs to any row of the warp).
__device__ __forceinline__ void zero_p16(uint32_t taddr)
{
    uint32_t z[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        z[i] = 0u;
    tmem_st16(taddr, z);
}

// Bit k set: key c + k of the slice lies in the row's range [lo, hi).
__device__ __forceinline__ uint32_t key_bits(int c, int lo, int hi)
{
    const int a = max(lo - c, 0), b = min(hi - c, 32);
    if (b <= a)
        return 0u;
    return (b == 32 ? 0xffffffffu : ((1u << b) - 1u)) & ~((1u << a) - 1u);
}

// Running max over the keys c .. c+31 of a row that are set in `keys`.
__device__ __forceinline__ float slice_max(const uint32_t (&r)[32], uint32_t keys, bool full, float mx)
{
    // two independent chains of three-input maxima
    float t0 = mx, t1 = -INFINITY;
    if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            t0 = fmax3(t0, __uint_as_float(r[j]), __uint_as_float(r[j + 1]));
            t1 = fmax3(t1, __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            t0 = fmax3(t0, ((keys >> j) & 1u) ? __uint_as_float(r[j]) : -INFINITY,
                       ((keys >> (j + 1)) & 1u) ? __uint_as_float(r[j + 1]) : -INFINITY);
            t1 = fmax3(t1, ((keys >> (j + 2)) & 1u) ? __uint_as_float(r[j + 2]) : -INFINITY,
                       ((keys >> (j + 3)) & 1u) ? __uint_as_float(r[j + 3]) : -INFINITY);
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

// Two bf16 values -> two fp16 values, round to nearest (exact for |v| in [2^-14, 65504]; smaller
// magnitudes round to fp16's subnormal grid, an absolute error below 2^-25).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w)
{
    const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    return *reinterpret_cast<const uint32_t *>(&h);
}

// A K/V slot's V tile before its PV, by one whole warp: rows [nk, nk16) are zeroed (they meet
// P = 0 and must not hold NaN), and bf16 values are converted in place to fp16, so that P can be
// rounded to fp16 (11 significant bits) rather than bf16 (8).  A value outside fp16's range (a
// finite |v| >= 65536, or an infinity) becomes an fp16 infinity; if any does, the tile is put back
// to its original bf16 bytes from global memory (row r of the tile is row rows[base + r], or
// row0 + r when rows is null, of the tensor at vsrc) and stays bf16, and so does the P that meets
// it.  Rows are 128 contiguous bytes in the swizzled layout, so rows [0, nk) are the first
// 128 nk bytes.  Returns true when the tile (and the chunk's P) is fp16.
template <bool kBF16>
__device__ __noinline__ bool prepare_v(uint8_t *sV, int nk, int lane, const uint8_t *vsrc, int64_t row_bytes,
                                       const int32_t *rows, int base, int64_t row0)
{
    const int nk16 = (nk + 15) & ~15;
    for (int i = lane; i < (nk16 - nk) * 8; i += 32)
        *reinterpret_cast<uint4 *>(sV + nk * 128 + i * 16) = make_uint4(0, 0, 0, 0);
    bool fp16 = true;
    if constexpr (kBF16) {
        uint4 *v = reinterpret_cast<uint4 *>(sV);
        const int n16 = nk * 8;  // 16-byte chunks of rows [0, nk)
        uint32_t infs = 0;
        for (int i0 = lane; i0 < n16; i0 += 128) {
            uint4 w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                w[u] = i0 + 32 * u < n16 ? v[i0 + 32 * u] : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint4 h;
                h.x = bf16x2_to_f16x2(w[u].x);
                h.y = bf16x2_to_f16x2(w[u].y);
                h.z = bf16x2_to_f16x2(w[u].z);
                h.w = bf16x2_to_f16x2(w[u].w);
                infs |= __vcmpeq2(h.x & 0x7FFF7FFFu, 0x7C007C00u) | __vcmpeq2(h.y & 0x7FFF7FFFu, 0x7C007C00u) |
                        __vcmpeq2(h.z & 0x7FFF7FFFu, 0x7C007C00u) | __vcmpeq2(h.w & 0x7FFF7FFFu, 0x7C007C00u);
                if (i0 + 32 * u < n16)
                    v[i0 + 32 * u] = h;
            }
        }
        if (__any_sync(0xffffffffu, infs != 0u)) {
            // rare: an infinity or a value beyond fp16's range -- the original bf16 tile again
            __syncwarp();
            for (int i = lane; i < n16; i += 32) {
                const int r = i >> 3, c = i & 7;
                const int64_t grow = rows != nullptr ? static_cast<int64_t>(rows[base + r]) : row0 + r;
                v[r * 8 + (c ^ (r & 7))] = __ldg(reinterpret_cast<const uint4 *>(vsrc + grow * row_bytes) + c);
            }
            fp16 = false;
        }
    }
    fence_proxy_async_smem();  // generic-proxy writes, read next by the tensor core
    __syncwarp();
    return fp16;
}

// Fused path: copier warp w (of kCopyWarps) copies its share of one tile of up to 128 kept rows
// of one head from the padded tensor into the 128-byte-swizzled layout with 16-byte cp.async:
// row r of the tile is padded row rows[base + r].  The chunks go in groups of 32 (one per lane,
// 8 lanes per 128-byte row, so each row is one coalesced segment), group g to warp g % kCopyWarps.
// Completion arrives on `bar` once per copier lane.  Kept out of line: inlined, its unrolled loop
// sat in the middle of the block's hot code and cost instruction-cache hits even on calls that
// take the TMA path (measured: the single launch 3 % faster at config 5 r = 1, 10 % at r = 0.7).
__device__ __noinline__ void copy_tile_async(uint8_t *tile, const uint8_t *src, int64_t row_bytes, uint64_t *bar,
                                                const int32_t *rows, int base, int count, int w, int lane)
{
    // src points at this head's 128 bytes of padded row 0.  Rows at or past `count` are not
    // copied: their S columns are masked, their V rows zeroed before use, or (Q) their output
    // never stored.
    const uint32_t tile_s = smem_addr(tile);
    const int groups = (count * 8 + 31) >> 5;
#pragma unroll 4
    for (int grp = w; grp < groups; grp += kCopyWarps) {
        const int i = lane + 32 * grp;
        const int r = i >> 3, c = i & 7;
        if (r < count) {
            const uint8_t *gsrc = src + static_cast<int64_t>(rows[base + r]) * row_bytes + c * 16;
            const uint32_t d = tile_s + r * 128 + ((c ^ (r & 7)) << 4);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
        }
    }
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Fused path: one tile of up to 128 kept rows of one head, as copy_tile_async does, but when the
// rows are consecutive padded rows (every token of the range kept, e.g. an unpruned image) copier
// lane 0 of warp 0 moves the whole 128-row box with one TMA load of the padded tensor instead
// (rows past `count` land too and are masked like the gathered case's stale rows).  Either way each
// copier lane arrives once on `bar`; the TMA bytes are added to the phase's transaction count.
__device__ __forceinline__ void gather_tile(uint8_t *tile, const CUtensorMap *tm, int h, const uint8_t *src,
                                            int64_t row_bytes, uint64_t *bar, const int32_t *rows, int base,
                                            int count, int w, int lane)
{
    const int r0 = rows[base];
    if (rows[base + count - 1] - r0 == count - 1) {  // the list is increasing: consecutive rows
        if (w == 0 && lane == 0) {
            mbar_expect_tx(bar, kTileBytes);
            tma_load_3d(tile, tm, bar, 0, h, r0);
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
        return;
    }
    copy_tile_async(tile, src, row_bytes, bar, rows, base, count, w, lane);
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
    auto idx_list = [&](int slot) { return reinterpret_cast<int32_t *>(base + kOffIdx + slot * kIdxSlotBytes); };

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = p.B, H = p.H;
    pdl_trigger();

    if (tid == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
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
            mbar_init(&bars->v_ready[s][0], 1);
            mbar_init(&bars->v_ready[s][1], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->p_full[s], kGroupWarps);  // one arrival per warp of softmax group s
            mbar_init(&bars->pv_done[s], 1);
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

    // everything above is private to the block; the inputs may come from the previous kernel
    pdl_wait();

    // ---- work list: tile_pre[b] = number of 128-row query tiles of images < b; cu staged too.
    if constexpr (kFused) {
        // kept tokens per image, counted from 16-byte chunks of the flat mask into cu_s[b+1], by
        // whichever of two layouts takes fewer dependent memory round trips (a block-uniform
        // choice): a warp per image (lanes over the image's chunks, coalesced, six images per warp
        // at a time, one warp reduction each) for few or long images; a thread per image (all of
        // its chunks, up to kCntBatch, loaded before any is counted) for many short ones
        const uintptr_t addr = reinterpret_cast<uintptr_t>(p.mask);
        const int off = static_cast<int>(addr & 15u);
        const uint4 *m16 = reinterpret_cast<const uint4 *>(addr - off);
        constexpr int kImg = 6, kCntBatch = 16;
        const int chunks = p.N / 16 + 2;  // 16-byte chunks an image's bytes can touch, at most
        const int rounds_warp = (B + (kThreads / 32) * kImg - 1) / ((kThreads / 32) * kImg) * ((chunks + 31) / 32);
        const int rounds_thread = (B + kThreads - 1) / kThreads * ((chunks + kCntBatch - 1) / kCntBatch);
        if (rounds_thread < rounds_warp) {
            for (int b = tid; b < B; b += kThreads) {
                const int64_t lo = static_cast<int64_t>(b) * p.N, hi = lo + p.N;
                const int64_t c0 = (off + lo) >> 4, c1 = (off + hi + 15) >> 4;
                int cnt = 0;
                for (int64_t j0 = c0; j0 < c1; j0 += kCntBatch) {
                    uint4 w[kCntBatch];
#pragma unroll
                    for (int i = 0; i < kCntBatch; ++i)
                        w[i] = j0 + i < c1 ? __ldg(m16 + j0 + i) : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int i = 0; i < kCntBatch; ++i)
                        cnt += __popc(kept_bits16_(w[i]) & range16_((j0 + i) * 16 - off, lo, hi));
                }
                cu_s[b + 1] = cnt;
            }
        } else {
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
                for (int k = 0; k * 32 < chunks; ++k) {
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
        }
        __syncthreads();
    }
    if (tid == 0)
        tile_pre[0] = 0;
    int carry_t = 0, carry_l = 0, lmax = 0;  // lmax: longest sequence, or kShortMax + 1 if any image is malformed
    for (int c0 = 0; c0 < B; c0 += kThreads) {
        const int b = c0 + tid;
        int tiles = 0, len = 0;
        if (b < B) {
            if constexpr (kFused) {
                len = cu_s[b + 1];
                tiles = (len + BM - 1) / BM;
                lmax = max(lmax, len);
            } else {
                const int64_t s0 = p.cu[b], s1 = p.cu[b + 1];
                cu_s[b] = static_cast<int32_t>(s0);
                if (b == B - 1)
                    cu_s[B] = static_cast<int32_t>(s1);
                if (s0 < 0 || s1 < s0 || s1 > p.capacity) {
                    if (blockIdx.x == 0)
                        raise_error(p.err, RRA_ERR_BAD_SEQLENS);
                    lmax = kShortMax + 1;  // malformed: per-image tiles, which skip this image
                } else {
                    tiles = static_cast<int>((s1 - s0 + BM - 1) / BM);
                    // the packed space must start at row 0 for the short-sequence tiling
                    lmax = max(lmax, (b == 0 && s0 != 0) ? kShortMax + 1 : static_cast<int>(s1 - s0));
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
        const int wmax = __reduce_max_sync(0xffffffffu, lmax);
        if (lane == 31) {
            bars->warp_sums[0][warp] = it_incl;
            bars->warp_sums[1][warp] = l_incl;
            bars->warp_sums[2][warp] = wmax;
        }
        __syncthreads();
        int before_t = carry_t, before_l = carry_l, chunk_t = 0, chunk_l = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            before_t += (w < warp) ? bars->warp_sums[0][w] : 0;
            before_l += (w < warp) ? bars->warp_sums[1][w] : 0;
            chunk_t += bars->warp_sums[0][w];
            chunk_l += bars->warp_sums[1][w];
            lmax = max(lmax, bars->warp_sums[2][w]);
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
    }

    // tiling: when no image is longer than kShortMax, 128-row tiles of the packed space (several
    // images per tile); otherwise one image per tile
    const int T = cu_s[B];
    const bool short_tiles = lmax <= kShortMax && T > 0;
    const int total_items = (short_tiles ? (T + BM - 1) / BM : tile_pre[B]) * H;

    // decode the block's first items once: every role walks the same list
    Item *items = reinterpret_cast<Item *>(base + kOffItems);
    for (int k = tid; k < kItemTable; k += kThreads) {
        const int item = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
        if (item < total_items)
            items[k] = decode_item(item, H, B, short_tiles, T, tile_pre, cu_s);
    }
    auto item_at = [&](int k, int item) {
        return k < kItemTable ? items[k] : decode_item(item, H, B, short_tiles, T, tile_pre, cu_s);
    };

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_slot;
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
        int cur_k0 = -1, cur_nk = -1, prev_slot = 0, n = 0;
        bool ok = true;
        const int nwords = (p.N + 31) / 32;
        for (int item = item_first; ok && item < item_end; item += item_step, ++n) {
            const Item it = item_at(n, item);
            const int islot = n & (kIdxSlots - 1);
            int32_t *list = idx_list(islot);
            ok = warp_wait(&bars->idx_free[islot], ((idx_phase >> islot) & 1u) ^ 1u, bars, p);
            if (!ok)
                break;
            idx_phase ^= 1u << islot;
            if (it.k0 == cur_k0 && it.nk == cur_nk) {
                // same key rows as the previous item (another head or q-tile): copy its list
                const int32_t *pl = idx_list(prev_slot);
                for (int i = lane; i < it.nk; i += 32)
                    list[i] = pl[i];
            } else {
                // the padded rows of the kept tokens of every image of the item, in packed order:
                // per image, mask bytes fetched 8 words of 32 at a time (independent loads), then
                // one ballot per word
                int running = 0;
                for (int b = it.b0; b < B && cu_s[b] < it.k0 + it.nk; ++b) {
                    const int row_off = b * p.N;
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
                            if (keep[u]) {
                                const int slot_i = running + __popc(bal & ((1u << lane) - 1u));
                                list[slot_i] = row_off + (w0 + u) * 32 + lane;  // < B * N < 2^31
                            }
                            running += __popc(bal);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->idx_full[islot]);
            cur_k0 = it.k0;
            cur_nk = it.nk;
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
            const int nkc = (it.nk + BN - 1) / BN;
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
            // fused: this head's 128 bytes of padded row 0 in Q, K, V; one padded row is H * 128 bytes
            const int64_t head0 = static_cast<int64_t>(it.h) * kD * 2;
            const int64_t row_bytes = static_cast<int64_t>(H) * kD * 2;
            if constexpr (kFused) {
                gather_tile(base + kOffQ + qs * kTileBytes, &tm_q, it.h, p.src[0] + head0, row_bytes,
                            &bars->q_full[qs], idx_list(islot), it.q0 - it.k0, it.nq, warp, lane);
            } else {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars->q_full[qs], kTileBytes);
                    tma_load_3d(base + kOffQ + qs * kTileBytes, &tm_q, &bars->q_full[qs], 0, it.h, it.q0);
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
                    const int cnt = min(BN, it.nk - kc * BN);
                    gather_tile(base + kOffK + ks * kTileBytes, &tm_k, it.h, p.src[1] + head0, row_bytes, full,
                                idx_list(islot), kc * BN, cnt, warp, lane);
                    gather_tile(base + kOffV + ks * kTileBytes, &tm_v, it.h, p.src[2] + head0, row_bytes, full,
                                idx_list(islot), kc * BN, cnt, warp, lane);
                } else {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(full, 2 * kTileBytes);
                        tma_load_3d(base + kOffK + ks * kTileBytes, &tm_k, full, 0, it.h, it.k0 + kc * BN);
                        tma_load_3d(base + kOffV + ks * kTileBytes, &tm_v, full, 0, it.h, it.k0 + kc * BN);
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
        // of the block and TMEM columns [256 g, 256 g + 256).  Per chunk kc of an item: S = Q K^T
        // into S; once the softmax has turned S(kc) into P(kc) (p_full), S(kc+1) is issued at once
        // -- S and P are separate, so it overlaps O += P(kc) V(kc) -- then that PV, once the V
        // warp has prepared V(kc).
        // The Q/K/V rings are filled in item order for both groups, so each issuer walks every
        // item and, for the other group's, only advances its ring positions.
        const int g = kMmaWarp0 + 1 - warp;
        uint32_t q_ph = 0, kv_ph = 0, p_ph = 0, ofree_ph = 0;
        // shared-memory descriptors of the ring slots: stepping K inside a 128-byte swizzled row
        // adds 32 bytes (2 units) to the start address, stepping 16 key rows adds 2048 bytes (128
        // units), and a slot is 1024 units further
        const uint64_t qdesc0 = smem_desc_sw128(smem_addr(base + kOffQ), 16, 1024);
        const uint64_t kdesc0 = smem_desc_sw128(smem_addr(base + kOffK), 16, 1024);
        const uint64_t vdesc0 = smem_desc_sw128(smem_addr(base + kOffV), 16, 1024);
        auto slot_desc = [](uint64_t d0, int slot) { return d0 + static_cast<uint64_t>(slot) * (kTileBytes >> 4); };
        const uint32_t dS = tmem + kGroupCols * g + kColS;
        const uint32_t dP = tmem + kGroupCols * g + kColP;
        const uint32_t dO = tmem + kGroupCols * g + kColO;
        // S(kc) = Q K(kc)^T into S: one MMA per 16 of the 64 head dims
        auto issue_qk = [&](int qs, int ks, int nk, bool last) {
            if (lane == 0) {
                tc_fence_after();
                if constexpr (kFused)
                    fence_proxy_async_smem();  // Q/K/V arrived through cp.async (generic proxy)
                const uint64_t qd = slot_desc(qdesc0, qs);
                const uint64_t kd = slot_desc(kdesc0, ks);
                const uint32_t idS = idesc_f16(BM, (nk + 15) & ~15, kBF16 ? 1u : 0u, 0u);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss(dS, qd + 2 * kk, kd + 2 * kk, idS, kk > 0 ? 1u : 0u);
                mma_commit(&bars->s_full[g]);
                if (last)
                    mma_commit(&bars->q_empty[qs]);  // last read of this Q tile
            }
            __syncwarp();
        };
        uint32_t v_ph = 0;
        int qs = 0, ks = 0, n = 0;
        bool ok = true;
        for (int item = item_first; ok && item < item_end; item += item_step, ++n) {
            const Item it = item_at(n, item);
            const int nkc = (it.nk + BN - 1) / BN;
            if ((n & 1) != g) {
                // the other group's item: its Q slot is never ours (item n uses slot n % 2), and
                // its K/V chunks pass through the same slots but signal the other group's
                // barriers -- only the ring positions advance
                q_ph ^= 1u << qs;
                qs = (qs + 1 == kQStages) ? 0 : qs + 1;
                ks = (ks + nkc) % kKVStages;
                continue;
            }
            ok = warp_wait(&bars->q_full[qs], (q_ph >> qs) & 1u, bars, p);
            if (!ok)
                break;
            q_ph ^= 1u << qs;
            ok = warp_wait(&bars->kv_full[ks][g], (kv_ph >> ks) & 1u, bars, p);
            if (!ok)
                break;
            kv_ph ^= 1u << ks;
            issue_qk(qs, ks, min(BN, it.nk), nkc == 1);
            for (int kc = 0; kc < nkc; ++kc) {
                const int nk = min(BN, it.nk - kc * BN);
                const int ks_next = (ks + 1 == kKVStages) ? 0 : ks + 1;
                // P(kc) written (and S(kc) read) by the softmax
                ok = warp_wait(&bars->p_full[g], p_ph, bars, p);
                if (!ok)
                    break;
                p_ph ^= 1u;
                if (kc + 1 < nkc) {
                    ok = warp_wait(&bars->kv_full[ks_next][g], (kv_ph >> ks_next) & 1u, bars, p);
                    if (!ok)
                        break;
                    kv_ph ^= 1u << ks_next;
                    issue_qk(qs, ks_next, min(BN, it.nk - (kc + 1) * BN), kc + 1 == nkc - 1);
                }
                // before the first PV of an item, the group's previous item must have been read out of O
                if (kc == 0 && n >= 2) {
                    ok = warp_wait(&bars->o_free[g], ofree_ph, bars, p);
                    if (!ok)
                        break;
                    ofree_ph ^= 1u;
                }
                // V(kc) prepared by the V warp (zero tail; fp16 unless out of its range)
                ok = warp_wait(&bars->v_ready[ks][g], (v_ph >> ks) & 1u, bars, p);
                if (!ok)
                    break;
                v_ph ^= 1u << ks;
                const bool fp16 = !kBF16 || bars->v_fmt[ks] == 0;
                if (lane == 0) {
                    tc_fence_after();
                    const uint64_t vd = slot_desc(vdesc0, ks);
                    const uint32_t idPV = idesc_f16(BM, kD, fp16 ? 0u : 1u, 1u);
                    const int nj = ((nk + 15) & ~15) >> 4;
                    // keys 16j .. 16j+15: P columns 8j .. 8j+7 (two 16-bit values per column)
#pragma unroll
                    for (int j = 0; j < BN / 16; ++j)
                        if (j < nj)
                            mma_ts(dO, dP + 8 * j, vd + 128 * j, idPV, (kc > 0 || j > 0) ? 1u : 0u);
                    mma_commit(&bars->pv_done[g]);
                    mma_commit(&bars->kv_empty[ks]);
                }
                __syncwarp();
                ks = ks_next;
            }
            qs = (qs + 1 == kQStages) ? 0 : qs + 1;
        }
        // drain: every MMA this thread issued has completed
        if (lane == 0) {
            mma_commit(&bars->drain[g]);
            mbar_wait_bounded(&bars->drain[g], 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp >= kVWarp0 && warp < kVWarp0 + kVWarps) {
        // ================================================================ V tiles
        // V warp v owns the K/V ring slots s = v (mod 2): it waits for every fill of those slots in
        // production order and prepares each as soon as it has landed -- zero the V rows past the
        // chunk's keys and, for bf16 inputs, convert the tile to fp16 in place when it fits -- then
        // records the slot's format and tells the owning group (its issuer before the PV, its
        // softmax before writing P).  A slot is refilled only after that chunk's PV, which follows
        // this warp's v_ready, so no fill of its slots can land before it has looked at the last
        // one (a warp that also watched slots another warp prepares could be lapped there).
        static_assert(kKVStages % kVWarps == 0, "each V warp owns whole ring slots");
        const int vw = warp - kVWarp0;
        uint32_t kv_ph = 0;  // bit 2*slot + group: parity of kv_full[slot][group] waits
        int ks = 0, n = 0;
        bool ok = true;
        for (int item = item_first; ok && item < item_end; item += item_step, ++n) {
            const Item it = item_at(n, item);
            const int nkc = (it.nk + BN - 1) / BN;
            const int gi = n & 1;
            for (int kc = 0; kc < nkc; ++kc) {
                if (ks % kVWarps == vw) {
                    const uint32_t bit = 1u << (2 * ks + gi);
                    ok = warp_wait(&bars->kv_full[ks][gi], (kv_ph & bit) ? 1u : 0u, bars, p);
                    if (!ok)
                        break;
                    kv_ph ^= bit;
                    // where the tile's rows came from, should it have to be restored as bf16
                    const uint8_t *vsrc = p.src[2] + static_cast<int64_t>(it.h) * kD * 2;
                    const int32_t *rows = kFused ? idx_list(n & (kIdxSlots - 1)) : nullptr;
                    const bool fp16 = prepare_v<kBF16>(base + kOffV + ks * kTileBytes, min(BN, it.nk - kc * BN), lane,
                                                       vsrc, static_cast<int64_t>(H) * kD * 2, rows, kc * BN,
                                                       static_cast<int64_t>(it.k0) + kc * BN);
                    if (lane == 0) {
                        bars->v_fmt[ks] = fp16 ? 0 : 1;
                        mbar_arrive(&bars->v_ready[ks][gi]);
                    }
                    __syncwarp();
                }
                ks = (ks + 1 == kKVStages) ? 0 : ks + 1;
            }
        }
    } else if (kFused && warp == kZeroWarp) {
        // ================================================================ pruned rows
        // The block's contiguous share of the B*N padded rows: every pruned one becomes zero bytes
        // (all heads), concurrently with the attention work, which never writes those rows.  Each
        // lane clears its own pruned rows with bulk copies from a zeroed block of shared memory
        // (the copy engine moves the bytes; the warp only issues), then waits for them to land.
        uint8_t *zero = base + kOffZero;
        for (uint32_t i = 16u * lane; i < kZeroBytes; i += 16u * 32u)
            *reinterpret_cast<uint4 *>(zero + i) = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();  // the zeros are visible to the copy engine
        __syncwarp();
        const int64_t rows = static_cast<int64_t>(B) * p.N;
        const int64_t share = (rows + gridDim.x - 1) / gridDim.x;
        const int64_t r0 = static_cast<int64_t>(blockIdx.x) * share;
        const int64_t r1 = min(rows, r0 + share);
        const uint32_t row_bytes = static_cast<uint32_t>(H) * (p.out_dt == RRA_F32 ? 4u : 2u) * kD;
        for (int64_t t = r0 + lane; t < r1; t += 32) {
            if (p.mask[t] != 0)
                continue;
            uint8_t *y = static_cast<uint8_t *>(p.out) + t * row_bytes;
            for (uint32_t o = 0; o < row_bytes; o += kZeroBytes)
                bulk_store(y + o, zero, min(kZeroBytes, row_bytes - o));
        }
        bulk_commit();
        bulk_wait_all();
    } else if (warp >= kSoftmaxWarp0 && warp < kSoftmaxWarp0 + kSoftmaxWarps) {
        // ================================================================ softmax + epilogue
        // Group g (4 warps) takes items n = g, g+2, ...; thread r of the group owns row r of the
        // group's S, P and O (its TMEM lane), so the row max and row sum need no exchange.  Per
        // chunk: the row max of S; once the previous chunk's PV has completed, O and the row sum
        // are rescaled if the max rose; then P = exp2(scale log2(e) (s - max)) goes to P, rounded
        // to the 16-bit type of the chunk's V tile, and its fp32 values are added to the row sum.
        const int q4 = warp & 3;                     // TMEM lane quarter of this warp
        const int g = (warp - kSoftmaxWarp0) >> 2;   // softmax group
        const int row = q4 * 32 + lane;              // row of S / P / O owned by this thread
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + kGroupCols * g;
        const uint32_t sbase = lane_base + kColS;
        const uint32_t pbase = lane_base + kColP;
        const uint32_t obase = lane_base + kColO;
        uint32_t s_ph = 0, pv_ph = 0, v_ph = 0, idxf_ph = 0;
        bool ok = true;
        int n = 0, ks = 0;  // ks: K/V ring slot of the item's first chunk
        for (int item = item_first; ok && item < item_end; item += item_step, ++n) {
            const Item it = item_at(n, item);
            const int nkc = (it.nk + BN - 1) / BN;
            if ((n & 1) != g) {
                ks = (ks + nkc) % kKVStages;
                continue;
            }
            const int qrows = it.nq;
            const bool warp_active = q4 * 32 < qrows;
            // this row's keys, relative to k0: every kept token of its own image
            // (rows past the tile's last query row keep the whole range in per-image tiling: their
            // output is never stored, and whole-slice ranges keep the unmasked path)
            int klo = 0, khi = it.nk;
            if (short_tiles) {
                if (row < qrows) {
                    const int b = image_of_row(cu_s, it.b0, B, it.q0 + row);
                    klo = cu_s[b] - it.k0;
                    khi = cu_s[b + 1] - it.k0;
                } else {
                    khi = 0;
                }
            }
            float m_run = -INFINITY, l_run = 0.f;
            for (int kc = 0; kc < nkc; ++kc) {
                const int nk = min(BN, it.nk - kc * BN);
                const int nk16 = (nk + 15) & ~15;
                // the row's keys inside this chunk, [lo, hi), and their union over the warp
                int lo = max(klo - kc * BN, 0), hi = min(khi - kc * BN, nk);
                if (hi <= lo)
                    lo = hi = 0;
                const int wlo = __reduce_min_sync(0xffffffffu, hi > lo ? lo : BN);
                const int whi = __reduce_max_sync(0xffffffffu, hi);
                ok = warp_wait(&bars->s_full[g], s_ph, bars, p);
                if (!ok)
                    break;
                s_ph ^= 1u;
                tc_fence_after();
                // pass 1, row max: two 32-key slices per TMEM round trip
                float m_new = m_run;
                if (warp_active) {
                    float mx = -INFINITY;
#pragma unroll 1
                    for (int c = wlo & ~31; c < whi; c += 64) {
                        uint32_t ra[32], rb[32];
                        tmem_ld32(sbase + c, ra);
                        tmem_ld32(sbase + c + 32, rb);  // columns past the chunk are ignored below
                        tmem_wait_ld_dep(ra);
                        tmem_wait_ld_dep(rb);
                        const uint32_t ka = key_bits(c, lo, hi), kb = key_bits(c + 32, lo, hi);
                        mx = slice_max(ra, ka, __all_sync(0xffffffffu, ka == 0xffffffffu), mx);
                        if (c + 32 < whi)
                            mx = slice_max(rb, kb, __all_sync(0xffffffffu, kb == 0xffffffffu), mx);
                    }
                    m_new = fmaxf(m_run, mx);
                }
                // later chunks: the previous chunk's PV has completed (P is free again and O holds
                // every earlier chunk); rescale O and the row sum where the running max rose
                if (kc > 0) {
                    ok = warp_wait(&bars->pv_done[g], pv_ph, bars, p);
                    if (!ok)
                        break;
                    pv_ph ^= 1u;
                    tc_fence_after();
                    if (warp_active && __any_sync(0xffffffffu, m_new > m_run)) {
                        const float alpha = ex2_approx((m_run - m_new) * p.scale_log2);
                        l_run *= alpha;
#pragma unroll 1
                        for (uint32_t c = 0; c < kD; c += 16) {
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
                // the chunk's V format (fp16 unless its bf16 tile exceeds fp16's range)
                const int kslot = (ks + kc) % kKVStages;
                ok = warp_wait(&bars->v_ready[kslot][g], (v_ph >> kslot) & 1u, bars, p);
                if (!ok)
                    break;
                v_ph ^= 1u << kslot;
                const bool p_f16 = !kBF16 || bars->v_fmt[kslot] == 0;
                // pass 2: P = exp2(scale*log2e*(s - m)), one 32-key slice per round trip, 16 P
                // columns per slice; slices outside the warp's keys get P = 0 without being read
                if (warp_active) {
                    float lsum = 0.f;
#pragma unroll 1
                    for (int c = 0; c < nk16; c += 32) {
                        if (c + 32 <= wlo || c >= whi) {
                            zero_p16(pbase + (c >> 1));
                            continue;
                        }
                        uint32_t ra[32];
                        tmem_ld32(sbase + c, ra);
                        tmem_wait_ld_dep(ra);
                        const uint32_t kk = key_bits(c, lo, hi);
                        lsum += softmax_slice(ra, kk, __all_sync(0xffffffffu, kk == 0xffffffffu), p_f16, p.scale_log2,
                                              neg_m, pbase + (c >> 1));
                    }
                    l_run += lsum;
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->p_full[g]);
            }
            if (!ok)
                break;
            ks = (ks + nkc) % kKVStages;
            // epilogue: the last PV has completed; normalise by the row sum and store
            ok = warp_wait(&bars->pv_done[g], pv_ph, bars, p);
            if (!ok)
                break;
            pv_ph ^= 1u;
            const int islot = n & (kIdxSlots - 1);
            if constexpr (kFused) {
                ok = warp_wait(&bars->idx_full[islot], (idxf_ph >> islot) & 1u, bars, p);
                if (!ok)
                    break;
                idxf_ph ^= 1u << islot;
            }
            tc_fence_after();
            if (warp_active) {
                const float inv = 1.f / l_run;
                int64_t out_row = static_cast<int64_t>(it.q0) + row;
                if constexpr (kFused)  // the padded row of this packed row
                    out_row = idx_list(islot)[it.q0 - it.k0 + (row < qrows ? row : 0)];
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
    p.src[2] = static_cast<const uint8_t *>(a.v);  // read back only to restore a bf16 V tile
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
    // the padded tensors seen as [B*N, H, 64]: the TMA box of a tile whose kept rows are consecutive
    alignas(64) CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, a.q, rows, a.H, a.in_bf16) || !make_tmap(&tk, a.k, rows, a.H, a.in_bf16) ||
        !make_tmap(&tv, a.v, rows, a.H, a.in_bf16))
        return cudaErrorInvalidValue;
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
    return launch_variant<true>(a.in_bf16, tq, tk, tv, p, grid_for(a.B, a.H, a.N, num_sms), smem, stream);
}

}  // namespace rra
