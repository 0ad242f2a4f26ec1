/*
 * rra_oracle.c -- plain, slow, float64 CPU oracle for the pack -> attend -> unpack path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code, header, table or helper with the CUDA path.
 *
 * Source of what is computed: "Dispatch-Aware Ragged Attention for Pruned Vision Transformers"
 *   - sota2.com paper card, Abstract: token pruning drops uninformative patches; the kept
 *     tokens of each image form a variable-length sequence; attention over them is
 *     bidirectional (non-causal); the system is a pack-attend-unpack pipeline.
 *   - aissential.tech summary, Method: a two-phase token packer (index computation, then a
 *     gather) feeds the ragged attention kernel, whose output is unpacked to the padded layout.
 * The pages give no formula beyond "attention", so the oracle is the plain definition of
 * softmax(Q K^T * scale) V restricted to the kept tokens of one image and one head.
 *
 * Readings where the pages are silent:
 *   - keep mask: one byte per (image, token); nonzero = keep;
 *   - kept tokens keep their original order (stable ascending index), images in batch order;
 *   - cu_seqlens[0] = 0, cu_seqlens[b+1] = cu_seqlens[b] + L_b (varlen descriptor);
 *   - packed layout [T, H, d], T = sum L_b, rows token-major with heads interleaved;
 *   - unpack writes +0.0 bytes to pruned rows (fill_mode 0) or leaves them untouched (1);
 *   - scale defaults to 1/sqrt(d).
 *
 * Everything is scalar loops in IEEE double; 16-bit inputs are widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1, ORACLE_F32 = 2, ORACLE_F64 = 3 };

/* IEEE 754 binary16 -> double, exact: value = (-1)^s * 2^(e-15) * (1 + m/1024), subnormals
 * m * 2^-24. */
static double half_bits_to_double(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = (m != 0) ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return s ? -v : v;
}

/* bfloat16 is the top half of an IEEE binary32 word; widening is exact. */
static double bfloat_bits_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void *base, int dtype, int64_t idx)
{
    switch (dtype) {
    case ORACLE_F16: return half_bits_to_double(((const uint16_t *)base)[idx]);
    case ORACLE_BF16: return bfloat_bits_to_double(((const uint16_t *)base)[idx]);
    case ORACLE_F32: return (double)((const float *)base)[idx];
    default: return ((const double *)base)[idx];
    }
}

/* Phase 1 of the packer (aissential.tech summary, Method): per-image kept counts and their
 * running sum.  Returns T = cu[B]. */
int64_t rra_oracle_cu_seqlens(const uint8_t *mask, int B, int N, int32_t *cu)
{
    int64_t run = 0;
    cu[0] = 0;
    for (int b = 0; b < B; ++b) {
        for (int n = 0; n < N; ++n)
            if (mask[(int64_t)b * N + n] != 0)
                run += 1;
        cu[b + 1] = (int32_t)run;
    }
    return run;
}

/* rank[b*N+n] = number of kept tokens n' < n of image b, or -1 when (b, n) is pruned. */
void rra_oracle_rank(const uint8_t *mask, int B, int N, int32_t *rank)
{
    for (int b = 0; b < B; ++b) {
        int32_t r = 0;
        for (int n = 0; n < N; ++n) {
            if (mask[(int64_t)b * N + n] != 0)
                rank[(int64_t)b * N + n] = r++;
            else
                rank[(int64_t)b * N + n] = -1;
        }
    }
}

/* Phase 2 of the packer: copy the bytes of every kept row (b, n) of src [B, N, row] to packed
 * row cu[b] + rank(b, n) of dst [capacity, row].  Rows that would land at or beyond
 * `capacity` are not written.  Returns T. */
int64_t rra_oracle_pack(const uint8_t *mask, int B, int N, int64_t row_bytes,
                        const uint8_t *src, uint8_t *dst, int64_t capacity, int32_t *cu)
{
    int64_t T = rra_oracle_cu_seqlens(mask, B, N, cu);
    for (int b = 0; b < B; ++b) {
        int64_t r = 0;
        for (int n = 0; n < N; ++n) {
            if (mask[(int64_t)b * N + n] == 0)
                continue;
            int64_t out_row = (int64_t)cu[b] + r;
            r += 1;
            if (out_row >= capacity)
                continue;
            memcpy(dst + out_row * row_bytes, src + ((int64_t)b * N + n) * row_bytes, (size_t)row_bytes);
        }
    }
    return T;
}

/* One output row of the ragged attention (sota2.com card, Abstract: bidirectional attention
 * over the kept tokens of one image): for packed token t of image b (cu[b] <= t < cu[b+1])
 * and head h,
 *     s_j = scale * sum_k q[t,h,k] * k[cu[b]+j,h,k]     for j = 0..L_b-1  (no causal mask)
 *     m   = max_j s_j,   p_j = exp(s_j - m)
 *     o[k] = sum_j p_j * v[cu[b]+j,h,k] / sum_j p_j
 * q/k/v are packed [cap, H, d] in `dtype`; out is d doubles. */
static void attend_row(const void *q, const void *k, const void *v, int dtype,
                       int64_t seq_start, int64_t L, int64_t t, int h, int H, int d,
                       double scale, double *s, double *out)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
            acc += load_elem(q, dtype, (t * H + h) * (int64_t)d + c) *
                   load_elem(k, dtype, ((seq_start + j) * H + h) * (int64_t)d + c);
        s[j] = acc * scale;
        if (s[j] > m)
            m = s[j];
    }
    double denom = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        s[j] = exp(s[j] - m);
        denom += s[j];
    }
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < L; ++j)
            acc += s[j] * load_elem(v, dtype, ((seq_start + j) * H + h) * (int64_t)d + c);
        out[c] = acc / denom;
    }
}

/* Full ragged attention: out [T, H, d] doubles for every packed row of every image.
 * scale <= 0 selects 1/sqrt(d).  Returns 0, or -1 on a malformed cu_seqlens. */
int rra_oracle_attend(const void *q, const void *k, const void *v, int dtype,
                      const int32_t *cu, int B, int H, int d, double scale, double *out)
{
    if (scale <= 0.0)
        scale = 1.0 / sqrt((double)d);
    int64_t maxL = 0;
    for (int b = 0; b < B; ++b) {
        if (cu[b + 1] < cu[b])
            return -1;
        if (cu[b + 1] - cu[b] > maxL)
            maxL = cu[b + 1] - cu[b];
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
    if (!s)
        return -1;
    for (int b = 0; b < B; ++b) {
        int64_t L = cu[b + 1] - cu[b];
        for (int64_t i = 0; i < L; ++i) {
            int64_t t = cu[b] + i;
            for (int h = 0; h < H; ++h)
                attend_row(q, k, v, dtype, cu[b], L, t, h, H, d, scale, s, out + (t * H + h) * (int64_t)d);
        }
    }
    free(s);
    return 0;
}

/* Selected rows only: for each r < n_rows, out[r*d .. r*d+d) = attention row of packed token
 * row_t[r], head row_h[r].  Used to check full-size launches on a sample.  Returns 0 or -1. */
int rra_oracle_attend_rows(const void *q, const void *k, const void *v, int dtype,
                           const int32_t *cu, int B, int H, int d, double scale,
                           int64_t n_rows, const int64_t *row_t, const int32_t *row_h, double *out)
{
    if (scale <= 0.0)
        scale = 1.0 / sqrt((double)d);
    int64_t maxL = 0;
    for (int b = 0; b < B; ++b)
        if (cu[b + 1] - cu[b] > maxL)
            maxL = cu[b + 1] - cu[b];
    double *s = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
    if (!s)
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t t = row_t[r];
        int b = -1;
        for (int bb = 0; bb < B; ++bb)
            if (cu[bb] <= t && t < cu[bb + 1]) {
                b = bb;
                break;
            }
        if (b < 0) {
            free(s);
            return -1;
        }
        attend_row(q, k, v, dtype, cu[b], cu[b + 1] - cu[b], t, row_h[r], H, d, scale, s, out + r * d);
    }
    free(s);
    return 0;
}

/* Unpack (sota2.com card, Abstract: the pipeline ends by returning to the padded layout):
 * dst[b, n] = packed[cu[b] + rank(b, n)] for kept (b, n); pruned rows are set to zero bytes
 * (fill_mode 0) or left untouched (fill_mode 1).  Packed rows at or beyond `capacity` are never
 * read; their padded rows are left untouched.  Returns 0. */
int rra_oracle_unpack(const uint8_t *packed, const int32_t *cu, const uint8_t *mask,
                      int B, int N, int64_t row_bytes, int fill_mode, int64_t capacity, uint8_t *dst)
{
    for (int b = 0; b < B; ++b) {
        int64_t r = 0;
        for (int n = 0; n < N; ++n) {
            uint8_t *out = dst + ((int64_t)b * N + n) * row_bytes;
            if (mask[(int64_t)b * N + n] != 0) {
                int64_t src_row = (int64_t)cu[b] + r;
                r += 1;
                if (src_row < capacity)
                    memcpy(out, packed + src_row * row_bytes, (size_t)row_bytes);
            } else if (fill_mode == 0) {
                memset(out, 0, (size_t)row_bytes);
            }
        }
    }
    return 0;
}

/*
 * Threshold-l2 token selection, the step in front of the pipeline (aissential.tech summary,
 * Summary: the DeiT models are pruned with Threshold-l2, EViT and other methods -- the pages
 * name the method and nothing more).  Readings taken where they are silent:
 *   - a token's score is the l2 norm of its embedding row x[b, n, 0..C-1]; the squared norm,
 *     which orders tokens the same way, is what is compared;
 *   - the squared norm is the EXACT sum of the squares, with no rounding anywhere: every
 *     16-bit (or single-precision) input is an odd integer M times a power of two 2^e, its
 *     square M^2 * 2^(2e) is added into a fixed-point integer whose last bit is 2^-298 (the
 *     square of the smallest single-precision subnormal), so the comparison between two
 *     tokens is the comparison between the two exact rational numbers, whatever the order of
 *     the terms; a score with a NaN term is NaN and ranks below every other score, one with an
 *     infinite term (and no NaN) is +infinity;
 *   - the CLS token (n = 0) is always kept;
 *   - the candidates are the tokens n >= 1 kept by the previous stage (`prev`, or every token
 *     n >= 1 when there is none), which makes multi-stage masks nested (EViT-like schedules);
 *   - with `k_keep`, image b keeps its k_b best candidates: highest score first, the lower
 *     index first among equal scores (k_b clamped to [0, #candidates]); without it, every
 *     candidate whose squared norm is >= threshold_sq (compared exactly; a NaN score never
 *     passes).
 */
enum { SCORE_NAN = 0, SCORE_FINITE = 1, SCORE_INF = 2 };
#define SCORE_WORDS 20    /* 640 bits: squares of single-precision values stay below 2^256,
                             i.e. bit 554 above 2^-298, plus 31 bits of carries for C < 2^31 */
#define SCORE_EMIN (-298) /* weight of bit 0 */

typedef struct {
    int cls;                      /* SCORE_NAN, SCORE_FINITE or SCORE_INF */
    uint32_t w[SCORE_WORDS];      /* finite value = sum_i w[i] 2^(32 i) * 2^SCORE_EMIN */
} Score;

static void score_zero(Score *s)
{
    s->cls = SCORE_FINITE;
    memset(s->w, 0, sizeof s->w);
}

/* Add the integer m * 2^shift (m < 2^48, shift >= 0) into the fixed-point words.  Returns 0 when
 * the sum does not fit in SCORE_WORDS words. */
static int words_add(uint32_t *w, uint64_t m, int shift)
{
    /* m * 2^(shift % 32) < 2^80: three 32-bit words, starting at word shift / 32 */
    const int i0 = shift / 32, r = shift % 32;
    uint32_t part[3];
    part[0] = (uint32_t)(m << r);
    part[1] = (uint32_t)(r ? (m >> (32 - r)) : (m >> 32));
    part[2] = (uint32_t)(r ? (m >> (64 - r)) : 0);
    uint64_t carry = 0;
    int j = i0;
    for (; j < SCORE_WORDS; ++j) {
        const uint64_t add = (j - i0 < 3 ? (uint64_t)part[j - i0] : 0) + carry;
        if (j - i0 >= 3 && add == 0)
            return 1;
        const uint64_t t = (uint64_t)w[j] + add;
        w[j] = (uint32_t)t;
        carry = t >> 32;
    }
    if (carry != 0)
        return 0;
    for (; j < i0 + 3; ++j)
        if (part[j - i0] != 0)
            return 0;
    return 1;
}

/* s += x^2 exactly.  x is a value of one of the input types (at most 24 significant bits and a
 * binary exponent of at least -149), widened exactly to double. */
static void score_add_square(Score *s, double x)
{
    if (isnan(x)) {
        s->cls = SCORE_NAN;
        return;
    }
    if (isinf(x)) {
        if (s->cls != SCORE_NAN)
            s->cls = SCORE_INF;
        return;
    }
    if (x == 0.0)
        return;
    int k;
    double f = frexp(fabs(x), &k);       /* |x| = f * 2^k, 0.5 <= f < 1 */
    uint64_t m = (uint64_t)ldexp(f, 53); /* exact: f has at most 53 significant bits */
    int e = k - 53;
    while ((m & 1u) == 0) {              /* |x| = m * 2^e with m odd */
        m >>= 1;
        e += 1;
    }
    /* m < 2^24, so m^2 < 2^48; x^2 = m^2 * 2^(2e) and 2e >= SCORE_EMIN for the input types */
    words_add(s->w, m * m, 2 * e - SCORE_EMIN);
}

/* -1, 0, +1 as a < b, a == b, a > b, with NaN below every number. */
static int score_cmp(const Score *a, const Score *b)
{
    if (a->cls != b->cls)
        return a->cls < b->cls ? -1 : 1;
    if (a->cls != SCORE_FINITE)
        return 0;
    for (int i = SCORE_WORDS - 1; i >= 0; --i)
        if (a->w[i] != b->w[i])
            return a->w[i] < b->w[i] ? -1 : 1;
    return 0;
}

/* The smallest score value >= t, for comparing a score with a threshold t (not NaN):
 * score >= t  <=>  score >= score_ceil(t).  A t beyond every finite score maps to +infinity. */
static void score_ceil(Score *s, double t)
{
    score_zero(s);
    if (t <= 0.0)
        return;
    if (isinf(t)) {
        s->cls = SCORE_INF;
        return;
    }
    int k;
    double f = frexp(t, &k);
    uint64_t m = (uint64_t)ldexp(f, 53);
    int e = k - 53; /* t = m * 2^e */
    int shift = e - SCORE_EMIN;
    if (shift < 0) {
        /* t / 2^SCORE_EMIN = m / 2^-shift: round up to the next integer */
        uint64_t q = (-shift >= 64) ? 0 : (m >> -shift);
        int exact = (-shift < 64) && ((q << -shift) == m);
        m = q + (exact ? 0 : 1);
        shift = 0;
    }
    if (shift + 64 > SCORE_WORDS * 32 || !words_add(s->w, m >> 16, shift + 16) || !words_add(s->w, m & 0xFFFF, shift))
        s->cls = SCORE_INF; /* beyond every finite score */
}

static void l2_score(const void *x, int dtype, int64_t row, int C, Score *s)
{
    score_zero(s);
    for (int c = 0; c < C; ++c)
        score_add_square(s, load_elem(x, dtype, row * C + c));
}

/* The exact squared norm of row `row` of x [., C]: returns its class (0 NaN, 1 finite,
 * 2 +infinity) and, for a finite one, writes the SCORE_WORDS 32-bit words of the integer
 * value / 2^-298 (least significant first) to `words`. */
int rra_oracle_l2_score(const void *x, int dtype, int64_t row, int C, uint32_t *words)
{
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16 && dtype != ORACLE_F32)
        return -1;
    Score s;
    l2_score(x, dtype, row, C, &s);
    memcpy(words, s.w, sizeof s.w);
    return s.cls;
}

int rra_oracle_l2_score_words(void) { return SCORE_WORDS; }

int rra_oracle_l2_mask(const void *x, int dtype, int B, int N, int C, const int32_t *k_keep, double threshold_sq,
                       const uint8_t *prev, uint8_t *mask)
{
    if (B < 0 || N < 1 || C < 1 || isnan(threshold_sq))
        return -1;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16 && dtype != ORACLE_F32)
        return -1;
    Score *score = (Score *)malloc(sizeof(Score) * (size_t)N);
    char *cand = (char *)malloc((size_t)N);
    if (score == NULL || cand == NULL) {
        free(score);
        free(cand);
        return -1;
    }
    Score thr;
    score_ceil(&thr, threshold_sq);
    for (int b = 0; b < B; ++b) {
        int ncand = 0;
        for (int n = 0; n < N; ++n) {
            l2_score(x, dtype, (int64_t)b * N + n, C, &score[n]);
            cand[n] = (char)(n >= 1 && (prev == NULL || prev[(int64_t)b * N + n] != 0));
            ncand += cand[n];
            mask[(int64_t)b * N + n] = 0;
        }
        mask[(int64_t)b * N] = 1;
        if (k_keep != NULL) {
            int k = k_keep[b] < 0 ? 0 : (k_keep[b] > ncand ? ncand : k_keep[b]);
            /* pick the best remaining candidate k times; a strict '>' over ascending n keeps
             * the lowest index among equal scores */
            for (int t = 0; t < k; ++t) {
                int best = -1;
                for (int n = 1; n < N; ++n)
                    if (cand[n] && (best < 0 || score_cmp(&score[n], &score[best]) > 0))
                        best = n;
                mask[(int64_t)b * N + best] = 1;
                cand[best] = 0;
            }
        } else {
            for (int n = 1; n < N; ++n)
                if (cand[n] && score[n].cls != SCORE_NAN && score_cmp(&score[n], &thr) >= 0)
                    mask[(int64_t)b * N + n] = 1;
        }
    }
    free(score);
    free(cand);
    return 0;
}
