// mask.cu -- Threshold-l2 token selection, the step in front of the pack -> attend -> unpack
// pipeline ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers", aissential.tech
// summary, Summary: the DeiT models are pruned with Threshold-l2, EViT and other methods).
//
// Each image is scored by a thread-block cluster of up to eight CTAs, so every SM takes part even
// at small batches (one CTA per image once the batch alone fills the GPU): CTA r of the cluster
// owns a contiguous slice of the image's tokens, and a warp computes the squared norms of four
// tokens at a time from coalesced 16-byte loads of their embedding rows.  The squared norm is
// first accumulated in plain double, one addition per input of its square (exact in fp32: at most
// 22 significant bits, and bf16 inputs are range-checked against overflow and underflow); that sum is
// provably exact, in any order, when every square is a multiple of 2^q and the total stays below
// 2^(q+52), which a token checks from the smallest exponent among its inputs -- true for almost
// every token of realistic embeddings.  A token that fails the check (a tiny, subnormal, infinite
// or NaN input) is recomputed in double-double arithmetic: each addition an error-free two-sum
// whose rounding error is carried in a second double, the warp's partials combined the same way,
// the pair normalised to (hi, lo) = (RN(S), S - RN(S)).  Either way the result is a function of
// the exact sum S alone, so the selection does not depend on the order of the additions and
// equals the exact selection whenever every token's squares lie within 2^96 of one another (any
// realistic embedding; beyond that, only tokens whose exact scores agree to ~2^-96 relative could
// be ordered differently).  A token's (hi, lo) becomes a 128-bit key whose unsigned order is the
// score order (0 = not a candidate, then NaN, then the finite scores, then +infinity).  Each CTA
// writes its keys to its own shared memory; the threads then send them, one (token, CTA) pair
// each, to the other CTAs of the cluster (distributed shared memory), and one cluster barrier
// publishes them.  Each CTA then ranks its own tokens: a candidate's rank is the number of
// candidates that beat it (a higher key, or an equal key and a lower index), and it is kept when
// that rank is below k_b -- N comparisons per token, no sort.  The comparisons run on the keys
// rounded to fp32 (a monotone rounding: a higher fp32 key is a higher score), one lane per token
// against broadcast reads of all N keys, the key range split over the warps when a CTA has few
// tokens; only a token whose fp32 key another token shares is settled on the full keys.  In
// threshold mode a token's own key decides, and no keys are exchanged.
#include <cuda_fp16.h>

#include <mutex>

#include "rra_device.cuh"
#include "rra_internal.h"

namespace rra {

namespace {

constexpr int kMaskThreads = 256;
constexpr int kMaskWarps = kMaskThreads / 32;
constexpr int kMaxCluster = 8;  // portable cluster size
constexpr int kChunksPerPass = 2;  // 16-byte loads in flight per lane and token
constexpr int kTokPerWarp = 4;     // tokens a warp scores at once

struct Key {
    unsigned long long hi, lo;
};

template <bool kBF16>
__device__ __forceinline__ double widen(uint32_t bits16)
{
    if constexpr (kBF16)
        return static_cast<double>(__uint_as_float(bits16 << 16));
    else
        return static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(bits16))));
}

// s + e == a + b exactly (Knuth's two-sum; explicit round-to-nearest operations, no contraction).
__device__ __forceinline__ void two_sum(double a, double b, double &s, double &e)
{
    s = __dadd_rn(a, b);
    const double bb = __dsub_rn(s, a);
    e = __dadd_rn(__dsub_rn(a, __dsub_rn(s, bb)), __dsub_rn(b, bb));
}

// (hi, lo) += (h2, l2)
__device__ __forceinline__ void dd_add(double &hi, double &lo, double h2, double l2)
{
    double s, e;
    two_sum(hi, h2, s, e);
    hi = s;
    lo = __dadd_rn(lo, __dadd_rn(e, l2));
}

// Unsigned 64-bit image of a double whose order is the numeric order (for the low part, which
// may be negative).
__device__ __forceinline__ unsigned long long ordered_bits(double d)
{
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(d));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ bool key_greater(const Key &a, const Key &b)
{
    return a.hi > b.hi || (a.hi == b.hi && a.lo > b.lo);
}

// A key rounded to fp32, in the same (non-strict) order: -2 not a candidate, -1 NaN, else RN(S)
// rounded to fp32 (a monotone map of RN(S), so a higher fp32 key means a higher exact score).
__device__ __forceinline__ float key_float(const Key &k)
{
    if (k.hi == 0ull)
        return -2.0f;
    if (k.hi == 1ull)
        return -1.0f;
    return __double2float_rn(__longlong_as_double(static_cast<long long>(k.hi - 2ull)));
}

constexpr float kPadKeyF = -3.0f;  // fp32 key of the padding past N: below every token's

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_size()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// Store a key into the shared memory of CTA `rank` of this cluster, at the address that `local`
// has in this CTA.
__device__ __forceinline__ void st_cluster_key(const Key *local, uint32_t rank, const Key &k)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
    asm volatile("st.shared::cluster.v2.u64 [%0], {%1, %2};" ::"r"(remote), "l"(k.hi), "l"(k.lo) : "memory");
}

__device__ __forceinline__ void st_cluster_f32(const float *local, uint32_t rank, float v)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The two 16-bit values of w widened exactly to fp32 (low half first).
template <bool kBF16>
__device__ __forceinline__ float2 widen2(uint32_t w)
{
    if constexpr (kBF16)
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    else
        return __half22float2(*reinterpret_cast<const __half2 *>(&w));
}

// True when the plain double accumulation of the squares was exact, so `acc` is the exact sum;
// sqmin is the smallest fp32 square seen.  Required: every square exact in fp32 -- it has at most
// 16 (bf16) or 22 (fp16) significant bits, so it is exact unless it overflows (an input of 2^64
// or more, or an infinite or NaN one: `acc` is then infinite or NaN and the final test fails) or
// leaves fp32's normal range at the bottom (a zero or subnormal sqmin: refused; a zero input goes
// to the slow path, which is exact for it too); and every square a multiple of 2^q, q = twice
// the last-bit exponent of the smallest input, while the sum stays below 2^(q+52) -- then every
// partial sum, in any order, is an integer multiple of 2^q below 2^(q+53), representable exactly,
// so no addition rounded (the factor-2 margin covers the rounding of `acc` itself when the
// condition fails).  The smallest input has the smallest square; its exponent e is half the
// square's exponent, rounded down, and its last bit is 2^(e-7) for bf16 and at least 2^(e-10) for
// fp16 (a subnormal fp16's is 2^-24, coarser, which only makes the test stricter).
template <bool kBF16>
__device__ __forceinline__ bool fast_sum_exact(double acc, float sqmin)
{
    const int e2 = static_cast<int>(__float_as_uint(sqmin) >> 23);  // biased exponent, sign 0
    if (e2 == 0)
        return false;
    const int e = (e2 - 127) >> 1;  // arithmetic shift: rounds down for negative exponents
    const int q = 2 * (e - (kBF16 ? 7 : 10));
    return acc < __hiloint2double((q + 52 + 1023) << 20, 0);  // 2^(q+52), a normal double here
}

// Key of a token that the fast path cannot settle: the squared norm in double-double arithmetic
// (exact squares, error-free two-sum), normalised to (RN(S), S - RN(S)), with NaN / infinite
// classes.  The whole warp calls it (warp-uniform condition); lane 0's result is used.
template <bool kBF16>
__device__ __noinline__ Key slow_key(const uint16_t *xrow, int nchunks, int lane)
{
    const uint4 *row = reinterpret_cast<const uint4 *>(xrow);
    double hi = 0.0, lo = 0.0;
    bool nan = false, inf = false;
    for (int j = lane; j < nchunks; j += 32) {
        const uint4 v = __ldg(row + j);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double d = widen<kBF16>((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu));
            nan |= isnan(d);
            inf |= isinf(d);
            double s, e;
            two_sum(hi, __dmul_rn(d, d), s, e);  // the square is exact in double
            hi = s;
            lo = __dadd_rn(lo, e);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const double h2 = __shfl_xor_sync(0xffffffffu, hi, off);
        const double l2 = __shfl_xor_sync(0xffffffffu, lo, off);
        dd_add(hi, lo, h2, l2);
    }
    nan = __any_sync(0xffffffffu, nan);
    inf = __any_sync(0xffffffffu, inf);
    if (nan)
        return {1ull, 0ull};
    if (inf)
        return {0x7FF0000000000000ull + 2ull, ordered_bits(0.0)};
    const double h = __dadd_rn(hi, lo);  // (h, l) = (RN(S), S - RN(S)): canonical
    double l = __dsub_rn(lo, __dsub_rn(h, hi));
    if (l == 0.0)
        l = 0.0;  // one zero
    return {static_cast<unsigned long long>(__double_as_longlong(h)) + 2ull, ordered_bits(l)};
}

template <bool kBF16>
__global__ void __launch_bounds__(kMaskThreads, 4) l2_mask_kernel(const uint16_t *__restrict__ x, int N, int C,
                                                                const int32_t *__restrict__ k_keep, double thr_sq,
                                                                const uint8_t *prev, uint8_t *mask)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int N4 = (N + 3) & ~3;
    Key *keys = reinterpret_cast<Key *>(sm);                  // [N]: the keys of every token of the image
    float *keyf = reinterpret_cast<float *>(keys + N);        // [N4]: the same keys rounded to fp32, padded
    uint32_t *cnt = reinterpret_cast<uint32_t *>(keyf + N4);  // [n1 - n0]: rank counts of this CTA's tokens
    const uint32_t cs = cluster_size();
    const uint32_t rank = cluster_rank();
    const int b = static_cast<int>(blockIdx.x / cs);
    const int per_cta = (N + static_cast<int>(cs) - 1) / static_cast<int>(cs);
    const int n0 = static_cast<int>(rank) * per_cta;
    const int n1 = min(N, n0 + per_cta);
    const int T = max(0, n1 - n0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = static_cast<int64_t>(b) * N;
    const int nchunks = C / 8;
    for (int i = threadIdx.x; i < T; i += kMaskThreads)
        cnt[i] = 0u;
    if (threadIdx.x < N4 - N)
        keyf[N + threadIdx.x] = kPadKeyF;
    pdl_trigger();
    pdl_wait();  // the embeddings and the previous stage's mask may come from the previous kernel

    // ---- scores of this CTA's tokens: a warp takes kTokPerWarp tokens at a time (n, n + 8, ...,
    // all their loads of a pass in flight together) and writes their keys to this CTA's shared
    // memory
    for (int nb = n0 + warp; nb < n1; nb += kTokPerWarp * kMaskWarps) {
        // candidacy of the group's tokens (lane t: token t), loaded alongside the embeddings
        const int nl = nb + lane * kMaskWarps;
        const bool cand_l = lane < kTokPerWarp && nl < n1 && nl >= 1 && (prev == nullptr || prev[row0 + nl] != 0);
        double acc[kTokPerWarp];
        float sqmin[kTokPerWarp];  // smallest square
#pragma unroll
        for (int t = 0; t < kTokPerWarp; ++t) {
            acc[t] = 0.0;
            sqmin[t] = __uint_as_float(0x7F800000u);
        }
        for (int j0 = 0; j0 < nchunks; j0 += 32 * kChunksPerPass) {
            uint4 v[kTokPerWarp][kChunksPerPass];
#pragma unroll
            for (int t = 0; t < kTokPerWarp; ++t) {
                const int n = nb + t * kMaskWarps;
                const uint4 *row = reinterpret_cast<const uint4 *>(x + (row0 + n) * C);
#pragma unroll
                for (int u = 0; u < kChunksPerPass; ++u) {
                    const int j = j0 + lane + 32 * u;
                    v[t][u] = (n < n1 && j < nchunks) ? __ldg(row + j) : make_uint4(0u, 0u, 0u, 0u);  // padding: not accumulated
                }
            }
#pragma unroll
            for (int t = 0; t < kTokPerWarp; ++t) {
#pragma unroll
                for (int u = 0; u < kChunksPerPass; ++u) {
                    const int j = j0 + lane + 32 * u;
                    const uint32_t w[4] = {v[t][u].x, v[t][u].y, v[t][u].z, v[t][u].w};
                    if (j < nchunks) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = widen2<kBF16>(w[i]);
                            // exact fp32 squares (checked by fast_sum_exact), exact widening, one
                            // rounded-to-nearest double addition each
                            const float sx = __fmul_rn(f.x, f.x), sy = __fmul_rn(f.y, f.y);
                            sqmin[t] = fminf(sqmin[t], fminf(sx, sy));
                            acc[t] = __dadd_rn(acc[t], static_cast<double>(sx));
                            acc[t] = __dadd_rn(acc[t], static_cast<double>(sy));
                        }
                    }
                }
            }
        }
        const uint32_t cand_bits = __ballot_sync(0xffffffffu, cand_l);
#pragma unroll
        for (int t = 0; t < kTokPerWarp; ++t) {
            const int n = nb + t * kMaskWarps;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                acc[t] = __dadd_rn(acc[t], __shfl_xor_sync(0xffffffffu, acc[t], off));
                sqmin[t] = fminf(sqmin[t], __shfl_xor_sync(0xffffffffu, sqmin[t], off));
            }
            Key k;
            if (!fast_sum_exact<kBF16>(acc[t], sqmin[t]) && n < n1)
                k = slow_key<kBF16>(x + (row0 + n) * C, nchunks, lane);  // warp-uniform, rare
            else
                k = {static_cast<unsigned long long>(__double_as_longlong(acc[t])) + 2ull, ordered_bits(0.0)};
            if (lane == 0 && n < n1) {
                if (((cand_bits >> t) & 1u) == 0u)
                    k = {0ull, 0ull};
                keys[n] = k;
                keyf[n] = key_float(k);
            }
        }
    }
    __syncthreads();  // this CTA's keys are complete

    if (k_keep == nullptr) {
        // ---- threshold mode: each token's own key decides (exact S >= t: RN(S) > t, or
        // RN(S) == t and S - RN(S) >= 0); NaN and non-candidates never pass
        for (int n = n0 + static_cast<int>(threadIdx.x); n < n1; n += kMaskThreads) {
            const Key kn = keys[n];
            uint8_t keep = 0;
            if (n == 0) {
                keep = 1;  // CLS
            } else if (kn.hi > 1ull) {
                const double h = __longlong_as_double(static_cast<long long>(kn.hi - 2ull));
                keep = (h > thr_sq || (h == thr_sq && kn.lo >= 0x8000000000000000ull)) ? 1 : 0;
            }
            mask[row0 + n] = keep;
        }
        return;  // no shared memory of another CTA was touched
    }

    // ---- the other CTAs of the cluster receive this CTA's keys (one store per thread and item)
    for (int i = static_cast<int>(threadIdx.x); i < T * static_cast<int>(cs - 1); i += kMaskThreads) {
        const int n = n0 + i % T;
        uint32_t r = static_cast<uint32_t>(i / T);
        r += r >= rank ? 1u : 0u;
        st_cluster_key(keys + n, r, keys[n]);
        st_cluster_f32(keyf + n, r, keyf[n]);
    }
    cluster_sync_all();  // every key of the image is now in this CTA's shared memory

    // ---- ranks of this CTA's tokens: lane = token (32 per group), the N keys split into S slices
    // across warps when the CTA has few groups; fp32 keys first (gt | eq << 16 per token), the
    // 128-bit keys only for tokens whose fp32 key is shared
    const int G = (T + 31) / 32;
    const int S = G >= kMaskWarps ? 1 : kMaskWarps / max(G, 1);
    const int Q = N4 / 4;
    const float4 *kf4 = reinterpret_cast<const float4 *>(keyf);
    for (int it = warp; it < G * S; it += kMaskWarps) {
        const int g = it / S, s = it % S;
        const int n = n0 + g * 32 + lane;
        const float fn = n < n1 ? keyf[n] : 0.0f;
        uint32_t c = 0u;
        const int qe = (s + 1) * Q / S;
#pragma unroll 4
        for (int q = s * Q / S; q < qe; ++q) {
            const float4 f = kf4[q];  // the same address across the warp: a broadcast
            c += (f.x > fn ? 1u : 0u) + (f.x == fn ? 0x10000u : 0u);
            c += (f.y > fn ? 1u : 0u) + (f.y == fn ? 0x10000u : 0u);
            c += (f.z > fn ? 1u : 0u) + (f.z == fn ? 0x10000u : 0u);
            c += (f.w > fn ? 1u : 0u) + (f.w == fn ? 0x10000u : 0u);
        }
        if (n < n1)
            atomicAdd(cnt + (n - n0), c);
    }
    __syncthreads();

    const int kb = k_keep[b];
    for (int g = warp; g < G; g += kMaskWarps) {
        const int n = n0 + g * 32 + lane;
        const bool valid = n < n1;
        const Key kn = valid ? keys[n] : Key{0ull, 0ull};
        const uint32_t c = valid ? cnt[n - n0] : 0u;
        const bool cand = valid && n != 0 && kn.hi != 0ull;
        // rank = candidates with a higher key or an equal key and a lower index; with no other
        // token at the same fp32 key that is the count of higher fp32 keys (the rounding is
        // monotone), otherwise the tied tokens are compared on their full keys
        int r = static_cast<int>(c & 0xFFFFu);
        uint32_t tied = __ballot_sync(0xffffffffu, cand && (c >> 16) > 1u);
        while (tied != 0u) {
            const int src = __ffs(tied) - 1;
            tied &= tied - 1u;
            const int nt = n0 + g * 32 + src;
            const Key kt = keys[nt];
            const float ft = keyf[nt];
            int e = 0;
            for (int m = lane; m < N; m += 32) {
                if (m != nt && keyf[m] == ft) {
                    const Key km = keys[m];
                    e += (key_greater(km, kt) || (km.hi == kt.hi && km.lo == kt.lo && m < nt)) ? 1 : 0;
                }
            }
            e = __reduce_add_sync(0xffffffffu, e);
            if (lane == src)
                r += e;
        }
        if (valid)
            mask[row0 + n] = (n == 0 || (cand && r < kb)) ? 1 : 0;
    }
}

// CTAs per image: enough for about two CTAs per SM over the batch (one CTA per image once the
// batch alone fills the GPU, where clusters would only limit how many CTAs can be resident), at
// least 16 tokens per CTA, at most the portable cluster size; a power of two.
// Clusters of 1, 2, 4 and 8 CTAs that can be resident at once, for this kernel at a given
// shared-memory size, from the occupancy query (which knows the GPU's actual GPC layout);
// -1 where a size cannot be used.  Queried once per device and size, then cached.
static_assert(kMaxCluster == 8, "cluster sizes 1, 2, 4, 8 are queried");

// Shared memory of the kernel: the 128-bit keys [N], the fp32 keys [N rounded up to 4] and the
// rank counts of one CTA's tokens (at most N).
constexpr int mask_smem_bytes(int N)
{
    return N * static_cast<int>(sizeof(Key)) + ((N + 3) & ~3) * 4 + N * 4;
}

template <bool kBF16>
struct ClusterFit {
    int smem = -1;
    int act[4] = {0, 0, 0, 0};
};

template <bool kBF16>
const int *max_active_clusters(int smem)
{
    static std::mutex mu;
    static ClusterFit<kBF16> cache[64][4];  // per device: the last four shared-memory sizes seen
    static int next[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &c : cache[dev])
        if (c.smem == smem)
            return c.act;
    ClusterFit<kBF16> &c = cache[dev][next[dev]];
    next[dev] = (next[dev] + 1) & 3;
    for (int i = 0; i < 4; ++i) {
        const int cs = 1 << i;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(cs));
        cfg.blockDim = dim3(kMaskThreads);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, l2_mask_kernel<kBF16>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = -1;
        }
        c.act[i] = n;
    }
    c.smem = smem;
    return c.act;
}

// Cluster size (CTAs per image): the fewest waves of clusters (one image per cluster), then the
// largest size (more SMs per image), keeping at least 16 tokens per CTA.
template <bool kBF16>
int cluster_for(int B, int N, int smem)
{
    const int *act = max_active_clusters<kBF16>(smem);
    int best = 1;
    int64_t best_waves = -1;
    for (int i = 0; i < 4; ++i) {
        const int cs = 1 << i;
        if (cs > 1 && N < 16 * cs)
            break;
        if (act == nullptr || act[i] <= 0)
            continue;
        const int64_t waves = (static_cast<int64_t>(B) + act[i] - 1) / act[i];
        if (best_waves < 0 || waves <= best_waves) {
            best_waves = waves;
            best = cs;
        }
    }
    return best;
}

template <bool kBF16>
cudaError_t set_mask_smem(int bytes)
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
    e = cudaFuncSetAttribute(l2_mask_kernel<kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev < 64)
        done_bytes[dev] = bytes;
    return e;
}

template <bool kBF16>
cudaError_t launch_mask_variant(const uint16_t *x, int B, int N, int C, const int32_t *k_keep, double thr_sq,
                                const uint8_t *prev, uint8_t *mask, int num_sms, cudaStream_t stream)
{
    const int smem = mask_smem_bytes(N);
    cudaError_t e = set_mask_smem<kBF16>(smem);
    if (e != cudaSuccess)
        return e;
    (void)num_sms;
    const int cs = cluster_for<kBF16>(B, N, smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(B) * cs);
    cfg.blockDim = dim3(kMaskThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, l2_mask_kernel<kBF16>, x, N, C, k_keep, thr_sq, prev, mask);
}

}  // namespace

static_assert(mask_smem_bytes(kMaskMaxN) <= 227 * 1024, "keys exceed shared memory at the largest N");

cudaError_t launch_l2_mask(const void *x, int B, int N, int C, bool bf16, const int32_t *k_keep, double thr_sq,
                           const uint8_t *prev, uint8_t *mask, int num_sms, cudaStream_t stream)
{
    if (B == 0)
        return cudaSuccess;
    const auto *xs = static_cast<const uint16_t *>(x);
    return bf16 ? launch_mask_variant<true>(xs, B, N, C, k_keep, thr_sq, prev, mask, num_sms, stream)
                : launch_mask_variant<false>(xs, B, N, C, k_keep, thr_sq, prev, mask, num_sms, stream);
}

}  // namespace rra
