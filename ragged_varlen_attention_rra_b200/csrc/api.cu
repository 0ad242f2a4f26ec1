// api.cu -- the extern "C" boundary of librra.so (declared in include/rra.h): argument
// validation, per-device attributes and kernel launches.  No call allocates or synchronises,
// except rra_get_device_error, which reads the device error word back.
#include <atomic>
#include <mutex>

#include "../../include/rra.h"
#include "rra_internal.h"

namespace {

std::atomic<uint64_t> g_wait_ns{2000000000ull};

int num_sms_of_current_device(int *out)
{
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev] > 0) {
        *out = cache[dev];
        return 0;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return -1;
    if (dev < 64)
        cache[dev] = n;
    *out = n;
    return 0;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int elem_size(rra_dtype dt)
{
    switch (dt) {
    case RRA_F16:
    case RRA_BF16: return 2;
    case RRA_F32: return 4;
    default: return 0;
    }
}

constexpr int64_t kMaxRows = 0x7fffffffLL;

// True when the byte ranges [a, a+na) and [b, b+nb) do not intersect (empty ranges never do).
inline bool disjoint(const void *a, uint64_t na, const void *b, uint64_t nb)
{
    if (a == nullptr || b == nullptr || na == 0 || nb == 0)
        return true;
    const uint64_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 + na <= b0 || b0 + nb <= a0;
}

}  // namespace

extern "C" {

rra_status rra_pack(const uint8_t *keep_mask, int B, int N, int H, int d, rra_dtype dt, int n_tensors,
                    const void *const *src, void *const *dst, int64_t capacity, int32_t *cu_seqlens,
                    int32_t *dev_error, rra_stream_t stream)
{
    if (keep_mask == nullptr || src == nullptr || dst == nullptr || cu_seqlens == nullptr)
        return RRA_ERR_INVALID_ARG;
    if (B < 0 || N < 1 || H < 1 || d < 1 || capacity < 1 || n_tensors < 1 || n_tensors > 3)
        return RRA_ERR_INVALID_ARG;
    const int es = elem_size(dt);
    if (es == 0)
        return RRA_ERR_UNSUPPORTED;
    const int64_t row_bytes = static_cast<int64_t>(H) * d * es;
    if (row_bytes % 16 != 0 || row_bytes > 8192)
        return RRA_ERR_UNSUPPORTED;
    if (B > 65535 || static_cast<int64_t>(B) * N > kMaxRows || capacity > kMaxRows)
        return RRA_ERR_UNSUPPORTED;
    for (int i = 0; i < n_tensors; ++i) {
        if (src[i] == nullptr || dst[i] == nullptr)
            return RRA_ERR_INVALID_ARG;
        if (!aligned16(src[i]) || !aligned16(dst[i]))
            return RRA_ERR_INVALID_ARG;
    }
    {
        // outputs (packed rows, cu_seqlens) must not overlap the inputs (mask, padded rows) or each other
        const uint64_t mask_b = static_cast<uint64_t>(B) * N, cu_b = 4ull * (B + 1);
        const uint64_t src_b = mask_b * row_bytes, dst_b = static_cast<uint64_t>(capacity) * row_bytes;
        for (int i = 0; i < n_tensors; ++i) {
            if (!disjoint(dst[i], dst_b, keep_mask, mask_b) || !disjoint(dst[i], dst_b, cu_seqlens, cu_b) ||
                !disjoint(cu_seqlens, cu_b, src[i], src_b))
                return RRA_ERR_INVALID_ARG;
            for (int j = 0; j < n_tensors; ++j)
                if (!disjoint(dst[i], dst_b, src[j], src_b) || (j != i && !disjoint(dst[i], dst_b, dst[j], dst_b)))
                    return RRA_ERR_INVALID_ARG;
        }
        if (!disjoint(cu_seqlens, cu_b, keep_mask, mask_b))
            return RRA_ERR_INVALID_ARG;
    }
    int sms = 0;
    if (num_sms_of_current_device(&sms) != 0)
        return RRA_ERR_CUDA;
    const cudaError_t e = rra::launch_pack(keep_mask, B, N, row_bytes, n_tensors, src, dst, capacity, cu_seqlens,
                                           dev_error, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA;
}

rra_status rra_attend(const void *q, const void *k, const void *v, void *o, const int32_t *cu_seqlens, int B, int H,
                      int d, int max_seqlen, int64_t capacity, float softmax_scale, rra_dtype in_dt,
                      rra_dtype out_dt, void *workspace, size_t ws_bytes, int32_t *dev_error,
                      rra_stream_t stream)
{
    (void)workspace;
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || cu_seqlens == nullptr)
        return RRA_ERR_INVALID_ARG;
    if (B < 0 || H < 1 || capacity < 1 || max_seqlen < 0)
        return RRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return RRA_ERR_INVALID_ARG;
    if (d != 64 || (in_dt != RRA_F16 && in_dt != RRA_BF16) || (out_dt != in_dt && out_dt != RRA_F32))
        return RRA_ERR_UNSUPPORTED;
    if (B > rra::kAttendMaxBatch || H > 65535 || capacity > kMaxRows)
        return RRA_ERR_UNSUPPORTED;
    if (ws_bytes < rra_attend_workspace_size(B, H, max_seqlen))
        return RRA_ERR_INVALID_ARG;
    if (!(softmax_scale == softmax_scale))
        return RRA_ERR_INVALID_ARG;
    {
        const uint64_t rows = static_cast<uint64_t>(capacity) * H * d;
        const uint64_t in_b = rows * 2, out_b = rows * (out_dt == RRA_F32 ? 4 : 2), cu_b = 4ull * (B + 1);
        if (!disjoint(o, out_b, q, in_b) || !disjoint(o, out_b, k, in_b) || !disjoint(o, out_b, v, in_b) ||
            !disjoint(o, out_b, cu_seqlens, cu_b))
            return RRA_ERR_INVALID_ARG;
    }
    int sms = 0;
    if (num_sms_of_current_device(&sms) != 0)
        return RRA_ERR_CUDA;
    rra::AttendArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.cu = cu_seqlens;
    a.B = B;
    a.H = H;
    a.max_seqlen = max_seqlen;
    a.capacity = capacity;
    a.scale = softmax_scale > 0.f ? softmax_scale : 0.125f;  // 1/sqrt(64)
    a.in_bf16 = in_dt == RRA_BF16;
    a.out_dt = static_cast<int>(out_dt);
    a.err = dev_error;
    a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    const cudaError_t e = rra::launch_attend(a, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA;
}

rra_status rra_pack_attend_unpack(const uint8_t *keep_mask, const void *q, const void *k, const void *v, void *y,
                                  int32_t *cu_seqlens, int B, int N, int H, int d, float softmax_scale,
                                  rra_dtype in_dt, rra_dtype out_dt, int32_t *dev_error, rra_stream_t stream)
{
    if (keep_mask == nullptr || q == nullptr || k == nullptr || v == nullptr || y == nullptr)
        return RRA_ERR_INVALID_ARG;
    if (B < 0 || N < 1 || H < 1)
        return RRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y))
        return RRA_ERR_INVALID_ARG;
    if (d != 64 || (in_dt != RRA_F16 && in_dt != RRA_BF16) || (out_dt != in_dt && out_dt != RRA_F32))
        return RRA_ERR_UNSUPPORTED;
    if (B > rra::kFusedMaxBatch || N > rra::kFusedMaxN || H > 65535 || static_cast<int64_t>(B) * N > kMaxRows)
        return RRA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(N) * H * d * 2 > kMaxRows)  // byte offsets inside one image are 32-bit
        return RRA_ERR_UNSUPPORTED;
    if (!(softmax_scale == softmax_scale))
        return RRA_ERR_INVALID_ARG;
    {
        const uint64_t mask_b = static_cast<uint64_t>(B) * N, elems = mask_b * H * d, cu_b = 4ull * (B + 1);
        const uint64_t in_b = elems * 2, out_b = elems * (out_dt == RRA_F32 ? 4 : 2);
        const void *ins[4] = {q, k, v, keep_mask};
        const uint64_t in_sz[4] = {in_b, in_b, in_b, mask_b};
        for (int i = 0; i < 4; ++i)
            if (!disjoint(y, out_b, ins[i], in_sz[i]) || !disjoint(cu_seqlens, cu_b, ins[i], in_sz[i]))
                return RRA_ERR_INVALID_ARG;
        if (!disjoint(y, out_b, cu_seqlens, cu_b))
            return RRA_ERR_INVALID_ARG;
    }
    int sms = 0;
    if (num_sms_of_current_device(&sms) != 0)
        return RRA_ERR_CUDA;
    rra::FusedArgs a;
    a.mask = keep_mask;
    a.q = q;
    a.k = k;
    a.v = v;
    a.y = y;
    a.cu_out = cu_seqlens;
    a.B = B;
    a.N = N;
    a.H = H;
    a.scale = softmax_scale > 0.f ? softmax_scale : 0.125f;  // 1/sqrt(64)
    a.in_bf16 = in_dt == RRA_BF16;
    a.out_dt = static_cast<int>(out_dt);
    a.err = dev_error;
    a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    const cudaError_t e = rra::launch_fused(a, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA;
}

rra_status rra_l2_mask(const void *x, int B, int N, int C, rra_dtype dt, const int32_t *k_keep, double threshold_sq,
                       const uint8_t *prev_mask, uint8_t *keep_mask, rra_stream_t stream)
{
    if (x == nullptr || keep_mask == nullptr)
        return RRA_ERR_INVALID_ARG;
    if (B < 0 || N < 1 || C < 1 || !aligned16(x))
        return RRA_ERR_INVALID_ARG;
    if ((dt != RRA_F16 && dt != RRA_BF16) || C % 8 != 0)
        return RRA_ERR_UNSUPPORTED;
    if (B > 65535 || N > rra::kMaskMaxN || static_cast<int64_t>(B) * N * C > (int64_t{1} << 40))
        return RRA_ERR_UNSUPPORTED;
    if (k_keep == nullptr && threshold_sq != threshold_sq)
        return RRA_ERR_INVALID_ARG;
    {
        const uint64_t mask_b = static_cast<uint64_t>(B) * N;
        if (!disjoint(keep_mask, mask_b, x, mask_b * C * 2) || !disjoint(keep_mask, mask_b, k_keep, 4ull * B) ||
            (prev_mask != keep_mask && !disjoint(keep_mask, mask_b, prev_mask, mask_b)))
            return RRA_ERR_INVALID_ARG;
    }
    if (B == 0)
        return RRA_OK;
    int sms = 0;
    if (num_sms_of_current_device(&sms) != 0)
        return RRA_ERR_CUDA;
    const cudaError_t e = rra::launch_l2_mask(x, B, N, C, dt == RRA_BF16, k_keep, threshold_sq, prev_mask, keep_mask,
                                              sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA;
}

rra_status rra_linear(const void *x, const void *w, const void *bias, const void *residual, void *const *outs,
                      int n_outs, int64_t M, const int32_t *m_dev, int N, int K, rra_activation act,
                      int32_t *dev_error, rra_stream_t stream)
{
    if (x == nullptr || w == nullptr || outs == nullptr || n_outs < 1 || n_outs > rra::kLinearMaxOuts)
        return RRA_ERR_INVALID_ARG;
    if (M < 0 || N < 1 || K < 1 || M > kMaxRows || (act != RRA_ACT_NONE && act != RRA_ACT_GELU))
        return RRA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(bias) || !aligned16(residual))
        return RRA_ERR_INVALID_ARG;
    if (K % 64 != 0 || N % n_outs != 0 || (N / n_outs) % 128 != 0)
        return RRA_ERR_UNSUPPORTED;
    const uint64_t out_b = static_cast<uint64_t>(M) * (N / n_outs) * 2;
    const uint64_t x_b = static_cast<uint64_t>(M) * K * 2, w_b = static_cast<uint64_t>(N) * K * 2;
    const uint64_t res_b = static_cast<uint64_t>(M) * N * 2;
    for (int j = 0; j < n_outs; ++j) {
        if (outs[j] == nullptr || !aligned16(outs[j]))
            return RRA_ERR_INVALID_ARG;
        if (!disjoint(outs[j], out_b, x, x_b) || !disjoint(outs[j], out_b, w, w_b) ||
            !disjoint(outs[j], out_b, bias, 2ull * N))
            return RRA_ERR_INVALID_ARG;
        // the residual may be the single output itself, element for element
        if (!(n_outs == 1 && residual == outs[0]) && !disjoint(outs[j], out_b, residual, res_b))
            return RRA_ERR_INVALID_ARG;
        for (int i = 0; i < j; ++i)
            if (!disjoint(outs[j], out_b, outs[i], out_b))
                return RRA_ERR_INVALID_ARG;
    }
    if (M == 0)
        return RRA_OK;
    int sms = 0;
    if (num_sms_of_current_device(&sms) != 0)
        return RRA_ERR_CUDA;
    rra::LinearArgs a{};
    a.x = x;
    a.w = w;
    a.bias = bias;
    a.residual = residual;
    for (int j = 0; j < n_outs; ++j)
        a.outs[j] = outs[j];
    a.n_outs = n_outs;
    a.M = M;
    a.m_dev = m_dev;
    a.N = N;
    a.K = K;
    a.act = static_cast<int>(act);
    a.err = dev_error;
    a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    const cudaError_t e = rra::launch_linear(a, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA;
}

rra_status rra_layernorm(const void *x, const void *gamma, const void *beta, void *y, int64_t M,
                         const int32_t *m_dev, int C, float eps, rra_stream_t stream)
{
    if (x == nullptr || gamma == nullptr || beta == nullptr || y == nullptr)
        return RRA_ERR_INVALID_ARG;
    if (M < 0 || M > kMaxRows || C < 1 || !(eps > 0.f))
        return RRA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(beta) || !aligned16(y))
        return RRA_ERR_INVALID_ARG;
    if (C % 8 != 0 || C > rra::kLayerNormMaxC)
        return RRA_ERR_UNSUPPORTED;
    const uint64_t row_b = static_cast<uint64_t>(M) * C * 2;
    if (!disjoint(y, row_b, x, row_b) || !disjoint(y, row_b, gamma, 2ull * C) || !disjoint(y, row_b, beta, 2ull * C))
        return RRA_ERR_INVALID_ARG;
    if (M == 0)
        return RRA_OK;
    int sms = 0;
    if (num_sms_of_current_device(&sms) != 0)
        return RRA_ERR_CUDA;
    const cudaError_t e =
        rra::launch_layernorm(x, gamma, beta, y, M, m_dev, C, eps, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA;
}

size_t rra_attend_workspace_size(int B, int H, int max_seqlen)
{
    (void)B;
    (void)H;
    (void)max_seqlen;
    return 0;
}

rra_status rra_unpack(const void *packed, const int32_t *cu_seqlens, const uint8_t *keep_mask, int B, int N, int H,
                      int d, rra_dtype dt, int fill_mode, int64_t capacity, void *dst, int32_t *dev_error,
                      rra_stream_t stream)
{
    if (packed == nullptr || cu_seqlens == nullptr || keep_mask == nullptr || dst == nullptr)
        return RRA_ERR_INVALID_ARG;
    if (B < 0 || N < 1 || H < 1 || d < 1 || capacity < 1 || (fill_mode != 0 && fill_mode != 1))
        return RRA_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(dst))
        return RRA_ERR_INVALID_ARG;
    const int es = elem_size(dt);
    if (es == 0)
        return RRA_ERR_UNSUPPORTED;
    const int64_t row_bytes = static_cast<int64_t>(H) * d * es;
    if (row_bytes % 16 != 0 || row_bytes > 8192)
        return RRA_ERR_UNSUPPORTED;
    if (B > 65535 || static_cast<int64_t>(B) * N > kMaxRows || capacity > kMaxRows)
        return RRA_ERR_UNSUPPORTED;
    {
        const uint64_t mask_b = static_cast<uint64_t>(B) * N;
        const uint64_t dst_b = mask_b * row_bytes;
        if (!disjoint(dst, dst_b, packed, static_cast<uint64_t>(capacity) * row_bytes) ||
            !disjoint(dst, dst_b, cu_seqlens, 4ull * (B + 1)) || !disjoint(dst, dst_b, keep_mask, mask_b))
            return RRA_ERR_INVALID_ARG;
    }
    int sms = 0;
    if (num_sms_of_current_device(&sms) != 0)
        return RRA_ERR_CUDA;
    const cudaError_t e = rra::launch_unpack(packed, cu_seqlens, keep_mask, B, N, row_bytes, fill_mode, capacity,
                                             dst, dev_error, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RRA_OK : RRA_ERR_CUDA;
}

rra_status rra_get_device_error(const int32_t *dev_error, rra_stream_t stream, int32_t *host_out)
{
    if (dev_error == nullptr || host_out == nullptr)
        return RRA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(host_out, dev_error, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return RRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return RRA_ERR_CUDA;
    return RRA_OK;
}

const char *rra_status_string(rra_status status)
{
    switch (status) {
    case RRA_OK: return "RRA_OK";
    case RRA_ERR_INVALID_ARG: return "RRA_ERR_INVALID_ARG";
    case RRA_ERR_UNSUPPORTED: return "RRA_ERR_UNSUPPORTED";
    case RRA_ERR_CUDA: return "RRA_ERR_CUDA";
    case RRA_ERR_CAPACITY: return "RRA_ERR_CAPACITY";
    case RRA_ERR_TIMEOUT: return "RRA_ERR_TIMEOUT";
    case RRA_ERR_BAD_SEQLENS: return "RRA_ERR_BAD_SEQLENS";
    default: return "RRA_ERR_UNKNOWN";
    }
}

void rra_set_wait_timeout_ns(uint64_t timeout_ns) { g_wait_ns.store(timeout_ns, std::memory_order_relaxed); }

int rra_version(void) { return 100; }

}  // extern "C"
