/*
 * rra.h -- C ABI of the ragged varlen attention library (librra.so) for token-pruned ViTs.
 *
 * The library implements the pack -> attend -> unpack pipeline of "Dispatch-Aware Ragged
 * Attention for Pruned Vision Transformers" (sota2.com paper card, Abstract; aissential.tech
 * summary, Method) as hand-written CUDA kernels for sm_100a (B200):
 *
 *   rra_pack    keep mask -> per-image kept counts -> cu_seqlens, and a gather of the kept
 *               token rows of up to three padded tensors into a packed, padding-free layout
 *               (the summary's "two-phase token packer": index computation, then gather);
 *   rra_attend  bidirectional (non-causal) softmax(Q K^T * scale) V, independently per image
 *               and head, over the variable-length sequences described by cu_seqlens
 *               (the card's "lightweight bidirectional ... attention kernel");
 *   rra_unpack  scatter of packed rows back to the padded layout, pruned rows zero-filled
 *               (the card's "pack-attend-unpack pipeline").
 *
 * Layouts (all row-major, C-contiguous):
 *   keep_mask   uint8  [B, N]        nonzero = the token survives pruning
 *   padded      dtype  [B, N, H, d]  one row = H*d elements
 *   packed      dtype  [capacity, H, d]; image b occupies rows cu_seqlens[b] .. cu_seqlens[b+1)-1,
 *               its kept tokens in ascending original index order
 *   cu_seqlens  int32  [B+1]         cu[0] = 0, cu[b+1] = cu[b] + L_b (the varlen convention)
 *
 * Conventions shared by every call:
 *   - All pointers except the host arrays `src`/`dst` of rra_pack and `host_out` are DEVICE
 *     pointers owned by the caller.  No call allocates, frees or synchronises: each only
 *     enqueues kernels on `stream` (NULL = the legacy default stream), so the whole sequence
 *     can be captured into a CUDA graph and replayed with new data in the same buffers.
 *   - Synchronous errors (bad arguments, unsupported shapes, launch failures) are returned
 *     before anything is enqueued, except RRA_ERR_CUDA from a failed launch.
 *   - Data-dependent errors found by a kernel (more kept tokens than `capacity`, malformed
 *     cu_seqlens, a bounded wait that ran out) are written to `dev_error`, an int32 device
 *     word the caller zeroes before use: the first error code wins, later ones are dropped.
 *     `dev_error` may be NULL, in which case those errors are not reported -- the kernels
 *     still never read or write outside the buffers described here.
 *   - Device pointers must be 16-byte aligned (the kernels move 16-byte vectors).
 *   - No output may overlap an input of the same call, nor another output: blocks read the
 *     inputs of an image while other blocks write the outputs of that image, so an in-place
 *     call would race.  Every call compares the byte ranges its sizes describe and returns
 *     RRA_ERR_INVALID_ARG, before any launch, when two of them intersect.  The one exception
 *     is rra_l2_mask, whose keep_mask may be exactly the same buffer as prev_mask.
 */
#ifndef RRA_H
#define RRA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *rra_stream_t;

typedef enum {
    RRA_OK = 0,
    RRA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer           */
    RRA_ERR_UNSUPPORTED = 2,   /* shape or dtype outside what the kernels implement          */
    RRA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed                */
    RRA_ERR_CAPACITY = 4,      /* device: more kept tokens than the packed buffer's capacity */
    RRA_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel ran out             */
    RRA_ERR_BAD_SEQLENS = 6    /* device: cu_seqlens decreasing, past capacity, or not
                                  matching the keep mask                                     */
} rra_status;

typedef enum { RRA_F16 = 0, RRA_BF16 = 1, RRA_F32 = 2 } rra_dtype;

/*
 * rra_pack -- the token packer (aissential.tech summary, Method: "two-phase fused token packer";
 * sota2.com card, Abstract: pruning drops uninformative patches before attention).
 *
 * Phase 1: L_b = number of nonzero bytes of keep_mask[b, :]; cu_seqlens[b+1] = sum_{b'<=b} L_b'.
 * Phase 2: for every kept (b, n) and every tensor i < n_tensors,
 *          dst[i][cu_seqlens[b] + rank(b, n)] = src[i][b, n]   (a byte copy of one row),
 *          rank(b, n) = number of kept n' < n of image b.
 * Rows of dst at or beyond T = cu_seqlens[B] are not written.
 *
 *   keep_mask   device uint8 [B, N]
 *   B, N        images and padded tokens per image (B >= 0, N >= 1)
 *   H, d        heads and head dim; one row is H*d elements of `dt` and must be a multiple
 *               of 16 bytes
 *   dt          element type of src/dst (any of rra_dtype; the copy is bitwise)
 *   n_tensors   1..3 (typically Q, K, V)
 *   src         HOST array of n_tensors device pointers, each [B, N, H, d]
 *   dst         HOST array of n_tensors device pointers, each [capacity, H, d]
 *   capacity    rows available in each dst (B*N always suffices); if T > capacity, rows at or
 *               beyond capacity are not written and RRA_ERR_CAPACITY is raised on dev_error;
 *               cu_seqlens still receives the true counts
 *   cu_seqlens  device int32 [B+1], written
 *   dev_error   device int32 or NULL
 *   stream      CUDA stream
 */
rra_status rra_pack(const uint8_t *keep_mask, int B, int N, int H, int d, rra_dtype dt,
                    int n_tensors, const void *const *src, void *const *dst, int64_t capacity,
                    int32_t *cu_seqlens, int32_t *dev_error, rra_stream_t stream);

/*
 * rra_attend -- bidirectional ragged attention (sota2.com card, Abstract: a bidirectional
 * attention kernel over the variable-length post-pruning sequences; aissential.tech summary,
 * Method: the "specialized bidirectional ... attention kernel" fed by the packer).
 *
 * For every image b with L_b = cu_seqlens[b+1] - cu_seqlens[b], head h and i < L_b:
 *     o[cu_seqlens[b]+i, h, :] = sum_j softmax_j(scale * q_i . k_j) v_j,   j over all L_b tokens.
 * Inputs are fp16 or bf16, products and sums are accumulated in fp32, the output is written
 * in out_dt (in_dt or RRA_F32).  Rows of o outside [0, T) are not written.
 *
 *   q, k, v        device [capacity, H, d] in in_dt (RRA_F16 or RRA_BF16)
 *   o              device [capacity, H, d] in out_dt
 *   cu_seqlens     device int32 [B+1], non-decreasing, cu_seqlens[B] <= capacity; an image
 *                  that breaks this is skipped and RRA_ERR_BAD_SEQLENS raised on dev_error
 *   B, H, d        images, heads, head dim (d must be 64)
 *   max_seqlen     host upper bound on any L_b, used only to size the launch (longer
 *                  sequences are still computed correctly); pass N if unsure
 *   capacity       rows of q/k/v/o
 *   softmax_scale  <= 0 selects 1/sqrt(d)
 *   workspace      reserved (may be NULL); ws_bytes must be >= rra_attend_workspace_size()
 *   dev_error      device int32 or NULL
 */
rra_status rra_attend(const void *q, const void *k, const void *v, void *o,
                      const int32_t *cu_seqlens, int B, int H, int d, int max_seqlen,
                      int64_t capacity, float softmax_scale, rra_dtype in_dt, rra_dtype out_dt,
                      void *workspace, size_t ws_bytes, int32_t *dev_error, rra_stream_t stream);

/* Bytes of device workspace rra_attend needs for these sizes (currently always 0). */
size_t rra_attend_workspace_size(int B, int H, int max_seqlen);

/*
 * rra_unpack -- scatter back to the padded layout (sota2.com card, Abstract: the
 * "pack-attend-unpack pipeline").
 *
 * For every (b, n): if keep_mask[b, n] != 0, dst[b, n] = packed[cu_seqlens[b] + rank(b, n)]
 * (a byte copy of one row); otherwise the row is set to zero bytes (fill_mode 0) or left
 * untouched (fill_mode 1).  A kept row whose source row is at or beyond `capacity`, or beyond
 * cu_seqlens[b+1], is left untouched and RRA_ERR_BAD_SEQLENS / RRA_ERR_CAPACITY is raised.
 *
 *   packed      device [capacity, H, d] in dt
 *   cu_seqlens  device int32 [B+1] (as written by rra_pack for the same mask)
 *   keep_mask   device uint8 [B, N]
 *   dst         device [B, N, H, d] in dt
 */
rra_status rra_unpack(const void *packed, const int32_t *cu_seqlens, const uint8_t *keep_mask,
                      int B, int N, int H, int d, rra_dtype dt, int fill_mode, int64_t capacity,
                      void *dst, int32_t *dev_error, rra_stream_t stream);

/*
 * rra_pack_attend_unpack -- the whole pack -> attend -> unpack call of one pruning stage in a
 * single launch (sota2.com card, Abstract: the pack-attend-unpack pipeline; aissential.tech
 * summary, Method: the "fused token packer" feeding the attention kernel).
 *
 * Same result as rra_pack (Q, K, V) + rra_attend + rra_unpack (fill_mode 0) with
 * softmax_scale, byte for byte in y and cu_seqlens, but the kept rows are gathered from the
 * padded tensors straight into the attention tiles and each output row is written straight to
 * its padded position, so no packed buffers exist.
 *
 *   keep_mask   device uint8 [B, N], nonzero = keep
 *   q, k, v     device [B, N, H, d] in in_dt (RRA_F16 or RRA_BF16), d must be 64
 *   y           device [B, N, H, d] in out_dt (in_dt or RRA_F32): kept rows receive the attention
 *               output, pruned rows are set to zero bytes
 *   cu_seqlens  device int32 [B+1] written with the running kept counts, or NULL
 *   B, N, H, d  B <= 4096, N <= 1024, N*H*d*2 < 2^31
 *   softmax_scale <= 0 selects 1/sqrt(d)
 *   dev_error   device int32 or NULL (only RRA_ERR_TIMEOUT can be raised)
 */
rra_status rra_pack_attend_unpack(const uint8_t *keep_mask, const void *q, const void *k, const void *v, void *y,
                                  int32_t *cu_seqlens, int B, int N, int H, int d, float softmax_scale,
                                  rra_dtype in_dt, rra_dtype out_dt, int32_t *dev_error, rra_stream_t stream);

/*
 * rra_l2_mask -- Threshold-l2 token selection, the step in front of the pipeline (aissential.tech
 * summary, Summary: the DeiT models are pruned with Threshold-l2, EViT and other methods; the
 * pages name the method only).  For every image b:
 *   score(n)   = squared l2 norm of x[b, n, :], the exact sum of the squares of the (exactly
 *                widened) 16-bit inputs: each square is exact in double precision and the sum is
 *                carried in double-double arithmetic, normalised to (RN(S), S - RN(S)), which is a
 *                function of the exact sum S alone -- so the order of the additions cannot matter,
 *                and the selection is the exact one whenever a token's squares lie within 2^96 of
 *                one another (otherwise only tokens whose exact scores agree to about 2^-96
 *                relative can be ordered differently); a score with a NaN term ranks below every
 *                other, one with an infinite term (and no NaN) above every finite one;
 *   candidates = tokens n >= 1 with prev_mask[b, n] != 0 (every n >= 1 when prev_mask is NULL),
 *                which makes the masks of successive stages nested (EViT-like schedules);
 *   keep_mask[b, 0] = 1 (the CLS token is always kept);
 *   with k_keep:  keep_mask[b, n] = 1 for the k_keep[b] best candidates -- higher score first,
 *                 lower n first among equal scores, k clamped to [0, number of candidates];
 *   without:      keep_mask[b, n] = 1 for the candidates with score >= threshold_sq, compared
 *                 exactly (a NaN score never passes);
 *   every other keep_mask[b, n] = 0.
 *
 *   x             device [B, N, C] in dt (RRA_F16 or RRA_BF16), 16-byte aligned, C a multiple of 8
 *   k_keep        device int32 [B], or NULL for threshold mode
 *   threshold_sq  threshold on the squared norm (threshold mode only)
 *   prev_mask     device uint8 [B, N] or NULL; may be the same buffer as keep_mask
 *   keep_mask     device uint8 [B, N], written
 *   B <= 65535, 1 <= N <= 4096
 */
rra_status rra_l2_mask(const void *x, int B, int N, int C, rra_dtype dt, const int32_t *k_keep,
                       double threshold_sq, const uint8_t *prev_mask, uint8_t *keep_mask,
                       rra_stream_t stream);

/*
 * The dense parts of a transformer block, on the same packed token rows the path produces, for
 * the attention-vs-MLP latency split of a token-pruned ViT block (aissential.tech summary, "In
 * practice": decompose attention vs. MLP latency contributions).  A block on packed rows x [T, C]:
 *   h = LayerNorm1(x); [q | k | v] = h Wqkv^T + bqkv (rra_linear, three outputs); a = the
 *   ragged attention of q, k, v over cu_seqlens (rra_attend); x1 = x + a Wo^T + bo; h2 =
 *   LayerNorm2(x1); m = GELU(h2 W1^T + b1); y = x1 + m W2^T + b2.
 */
typedef enum { RRA_ACT_NONE = 0, RRA_ACT_GELU = 1 } rra_activation;

/*
 * rra_linear -- Y = act(X W^T + bias) (+ residual): the projection and MLP layers, on tcgen05
 * tensor cores with fp32 accumulation and one rounding to bf16 per output element.
 *   x         device bf16 [M, K], row-major
 *   w         device bf16 [N, K] (an nn.Linear weight: one row per output feature)
 *   bias      device bf16 [N], or NULL
 *   residual  device bf16 [M, N], or NULL; added after the activation.  It may be exactly the
 *             buffer of the single output (n_outs = 1: each element is read, then written, by
 *             the same thread); otherwise it must not overlap an output
 *   act       RRA_ACT_NONE or RRA_ACT_GELU (the exact GELU, x (1 + erf(x / sqrt 2)) / 2)
 *   outs      host array of n_outs (1..4) device bf16 pointers: outs[j] is [M, N / n_outs] and
 *             receives columns [j N / n_outs, (j + 1) N / n_outs) of Y (n_outs = 3 splits a fused
 *             QKV projection into packed Q, K and V)
 *   M >= 0 rows of buffer; K a positive multiple of 64; N / n_outs a positive multiple of 128
 *   m_dev     device int32 or NULL: when given, only rows [0, min(M, *m_dev)) are computed and
 *             written -- on packed rows, cu_seqlens[B] of the pack, so the host need not know T
 *   dev_error device int32 word for a bounded wait that ran out (RRA_ERR_TIMEOUT), or NULL
 * Outputs must not overlap x, w, bias or each other (RRA_ERR_INVALID_ARG).  Its shapes and
 * layouts are this library's; the pages define none for the dense layers.
 */
rra_status rra_linear(const void *x, const void *w, const void *bias, const void *residual,
                      void *const *outs, int n_outs, int64_t M, const int32_t *m_dev, int N, int K,
                      rra_activation act, int32_t *dev_error, rra_stream_t stream);

/*
 * rra_layernorm -- y = (x - mean) / sqrt(var + eps) * gamma + beta over each row of x, with
 * the mean and the (biased) variance of the row in fp32 and one rounding to bf16 per output.
 *   x, y          device bf16 [M, C]; y must not overlap x
 *   gamma, beta   device bf16 [C]
 *   C a positive multiple of 8, at most 2048; eps > 0
 *   M, m_dev      rows of buffer, and an optional device row count as for rra_linear
 */
rra_status rra_layernorm(const void *x, const void *gamma, const void *beta, void *y, int64_t M,
                         const int32_t *m_dev, int C, float eps, rra_stream_t stream);

/*
 * rra_get_device_error -- copy the device error word to *host_out.  This SYNCHRONISES `stream`
 * (it is the only call that does) and so must not be used inside stream capture.
 */
rra_status rra_get_device_error(const int32_t *dev_error, rra_stream_t stream, int32_t *host_out);

/* Human-readable name of a status code (static string, never NULL). */
const char *rra_status_string(rra_status status);

/*
 * Debugging knob for the bounded waits inside rra_attend and rra_linear: the time, in nanoseconds of the
 * GPU global timer, after which a wait for an asynchronous copy or tensor-core operation gives
 * up, raises RRA_ERR_TIMEOUT and ends its block after draining the work it issued.  The default
 * is 2e9 (two seconds); 0 makes every wait that is not already complete give up at once.
 * Applies to launches enqueued after the call, process-wide.
 */
void rra_set_wait_timeout_ns(uint64_t timeout_ns);

/* Library version: major*10000 + minor*100 + patch. */
int rra_version(void);

#ifdef __cplusplus
}
#endif
#endif /* RRA_H */
