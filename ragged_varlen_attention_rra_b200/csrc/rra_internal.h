// rra_internal.h -- launchers shared between the kernel files and the C-ABI layer.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

namespace rra {

// Launch `kernel` with programmatic stream serialization: it may start while the previous kernel
// in the stream finishes, and must call pdl_wait() before touching memory that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}


cudaError_t launch_pack(const uint8_t *mask, int B, int N, int64_t row_bytes, int n_tensors,
                        const void *const *src, void *const *dst, int64_t capacity, int32_t *cu, int32_t *err,
                        int num_sms, cudaStream_t stream);

cudaError_t launch_unpack(const void *packed, const int32_t *cu, const uint8_t *mask, int B, int N,
                          int64_t row_bytes, int fill_mode, int64_t capacity, void *dst, int32_t *err, int num_sms,
                          cudaStream_t stream);

struct AttendArgs {
    const void *q, *k, *v;
    void *o;
    const int32_t *cu;
    int B, H, max_seqlen;
    int64_t capacity;
    float scale;
    bool in_bf16;
    int out_dt;  // rra_dtype of o
    int32_t *err;
    uint64_t wait_ns;
};

// Largest B rra_attend accepts (its per-block tile and cu_seqlens tables live in shared memory
// next to the 128 KiB of Q/K/V rings).
constexpr int kAttendMaxBatch = 8192;

cudaError_t launch_attend(const AttendArgs &a, int num_sms, cudaStream_t stream);

struct FusedArgs {
    const uint8_t *mask;
    const void *q, *k, *v;
    void *y;
    int32_t *cu_out;
    int B, N, H;
    float scale;
    bool in_bf16;
    int out_dt;
    int32_t *err;
    uint64_t wait_ns;
};

// Largest N and B the single-launch path accepts (its kept-row lists and per-image tables live
// in shared memory next to the Q/K/V rings).
constexpr int kFusedMaxN = 1024;
constexpr int kFusedMaxBatch = 4096;

cudaError_t launch_fused(const FusedArgs &a, int num_sms, cudaStream_t stream);

// Largest N rra_l2_mask accepts (one 16-byte key per token in shared memory).
constexpr int kMaskMaxN = 4096;

cudaError_t launch_l2_mask(const void *x, int B, int N, int C, bool bf16, const int32_t *k_keep, double thr_sq,
                           const uint8_t *prev, uint8_t *mask, int num_sms, cudaStream_t stream);

// Dense parts of a transformer block on packed rows (linear.cu).
constexpr int kLinearMaxOuts = 4;     // a fused projection's outputs (Q, K, V)
constexpr int kLayerNormMaxC = 2048;  // row width rra_layernorm accepts (8 16-byte chunks per lane)

struct LinearArgs {
    const void *x, *w, *bias, *residual;
    void *outs[kLinearMaxOuts];
    int n_outs;
    int64_t M;
    const int32_t *m_dev;
    int N, K, act;
    int32_t *err;
    uint64_t wait_ns;
};

cudaError_t launch_linear(const LinearArgs &a, int num_sms, cudaStream_t stream);

cudaError_t launch_layernorm(const void *x, const void *gamma, const void *beta, void *y, int64_t M,
                             const int32_t *m_dev, int C, float eps, int num_sms, cudaStream_t stream);

}  // namespace rra
