/*
 * sdpa_oracle.c -- plain float64 CPU oracle for scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  The product library never links, loads or calls
 * this file.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA path: it has its own dtype decoding, its own indexing and its own
 * loops, written to be read against the definition, not to be fast.
 *
 * What it computes, per batch b, query head h and query row i:
 *
 *   MLX issue #3585 ("mx.fast.scaled_dot_product_attention produces incorrect
 *   attention scores (MLX 0.31.2)"), section "Reproduction": the fixed
 *   composite forms scores = q . k^T * scale, takes softmax along the key
 *   axis (axis=-1) and multiplies the weights by v.  Its minimal reproduction
 *   sets scale = D^-0.5.
 *
 *   MLX issue #3885 ("Metal SDPA: no fused path for head_dim=512 ..."),
 *   section "Measured impact": the composite path shapes scores as
 *   [B, n_kv, n_rep, qL, kL], so the n_rep query heads of one group share KV
 *   head g = h / n_rep (contiguous groups).  Same issue, "Current routing":
 *   the (192, 128) combination means Dqk and Dv may differ.
 *
 *   MLX PR #4330 ("Support head dimension 72 in Metal full attention"),
 *   "Proposed changes": masks are none, additive, boolean or causal.
 *
 *   MLX issue #3885, "Current routing": Gemma 4's hybrid layout has sliding
 *   (local) attention layers next to its global ones.  The pages name the
 *   layers but not their rule; the reading taken here is causal attention
 *   limited to a window of the `window` most recent keys.
 *
 * Readings taken where the pages are silent (each is also a test):
 *   - additive mask: added after scaling: s_j = scale * (q . k_j) + mask_ij;
 *     entries may be -inf;
 *   - boolean mask: nonzero = attend, zero = the key is removed (-inf);
 *   - causal with Lq != Lk: bottom-right alignment, key j is visible to
 *     query i iff j <= i + (Lk - Lq); with Lq == Lk this is plain causal;
 *   - sliding window of W keys: with the same alignment, key j is visible to
 *     query i iff i + (Lk - Lq) - W < j <= i + (Lk - Lq): the W most recent
 *     keys up to the query's own position (W >= Lk is plain causal);
 *   - a row whose every key is removed outputs zeros (no NaN).
 *
 * Every element is widened exactly to double (fp32, fp16 and bf16 values are
 * all exactly representable), every sum is a sequential double loop, and the
 * result is returned in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };
enum { ORACLE_MASK_NONE = 0, ORACLE_MASK_ADDITIVE = 1, ORACLE_MASK_BOOL = 2, ORACLE_MASK_CAUSAL = 3,
       ORACLE_MASK_SLIDING = 4 };

/* IEEE binary16 -> double, from the format's definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits). */
static double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 31;
    int frac = h & 1023;
    double mag;
    if (expo == 0) {
        mag = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    } else if (expo == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(frac + 1024), expo - 25);  /* (1 + frac/1024) * 2^(expo-15) */
    }
    return sign ? -mag : mag;
}

/* bfloat16 -> double: a bfloat16 is the upper half of an IEEE binary32. */
static double oracle_bf16_to_double(uint16_t b) {
    uint32_t bits = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double oracle_load(const void* base, int64_t idx, int dtype) {
    if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
    if (dtype == ORACLE_F16) return oracle_half_to_double(((const uint16_t*)base)[idx]);
    return oracle_bf16_to_double(((const uint16_t*)base)[idx]);
}

/*
 * Attention for an explicit list of query rows.
 *
 * q, k, v    : base pointers of the stored tensors (storage dtype `dtype`).
 * strides    : 12 element strides, (b, h, l, d) for q, then k, then v.
 * mask       : for ADDITIVE, storage dtype `dtype`; for BOOL, uint8.
 * mask_st    : 4 element strides (b, h, lq, lk) of the mask; 0 broadcasts.
 * window     : for SLIDING, the number of most recent keys a query sees (>= 1).
 * rows       : nrows triples (b, h, i) naming the query rows to compute.
 * out        : nrows * Dv doubles, row-major.
 * probs      : optional (may be NULL): nrows * Lk doubles, the normalised
 *              softmax weights of each row (0 where a key is removed).
 * Returns 0, or -1 on an argument error or allocation failure.
 */
int oracle_sdpa_rows(const void* q, const void* k, const void* v,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                     int64_t Dqk, int64_t Dv, const int64_t* strides, double scale,
                     int mask_kind, const void* mask, const int64_t* mask_st, int64_t window, int dtype,
                     const int64_t* rows, int64_t nrows, double* out, double* probs) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Lq < 0 || Lk < 0 || Dqk <= 0 || Dv <= 0) return -1;
    if (mask_kind == ORACLE_MASK_SLIDING && window < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    if (dtype < ORACLE_F32 || dtype > ORACLE_BF16) return -1;
    const int64_t n_rep = Hq / Hkv;
    const int64_t *sq = strides, *sk = strides + 4, *sv = strides + 8;

    double* s = (double*)malloc((size_t)(Lk > 0 ? Lk : 1) * sizeof(double));
    if (!s) return -1;

    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= Lq) { free(s); return -1; }
        const int64_t g = h / n_rep;                 /* KV head of this query head */
        double* o = out + r * Dv;

        /* scores s_j = scale * sum_d q[b,h,i,d] * k[b,g,j,d], then the mask */
        for (int64_t j = 0; j < Lk; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < Dqk; ++d) {
                double qv = oracle_load(q, b * sq[0] + h * sq[1] + i * sq[2] + d * sq[3], dtype);
                double kv = oracle_load(k, b * sk[0] + g * sk[1] + j * sk[2] + d * sk[3], dtype);
                dot += qv * kv;
            }
            double sj = scale * dot;
            const int64_t midx = b * (mask_st ? mask_st[0] : 0) + h * (mask_st ? mask_st[1] : 0) +
                                 i * (mask_st ? mask_st[2] : 0) + j * (mask_st ? mask_st[3] : 0);
            if (mask_kind == ORACLE_MASK_ADDITIVE) {
                sj += oracle_load(mask, midx, dtype);
            } else if (mask_kind == ORACLE_MASK_BOOL) {
                if (((const uint8_t*)mask)[midx] == 0) sj = -INFINITY;
            } else if (mask_kind == ORACLE_MASK_CAUSAL) {
                if (j > i + (Lk - Lq)) sj = -INFINITY;
            } else if (mask_kind == ORACLE_MASK_SLIDING) {
                const int64_t own = i + (Lk - Lq);        /* the query's own key position */
                if (j > own || j <= own - window) sj = -INFINITY;
            }
            s[j] = sj;
        }

        /* softmax along the keys: m = max s_j, p_j = exp(s_j - m), l = sum p_j */
        double m = -INFINITY;
        for (int64_t j = 0; j < Lk; ++j)
            if (s[j] > m) m = s[j];
        double l = 0.0;
        for (int64_t j = 0; j < Lk; ++j) {
            double p = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
            s[j] = p;
            l += p;
        }

        /* out = sum_j p_j v[b,g,j,:] / l ; a row with no visible key is 0 */
        for (int64_t e = 0; e < Dv; ++e) o[e] = 0.0;
        if (l > 0.0) {
            for (int64_t j = 0; j < Lk; ++j) {
                for (int64_t e = 0; e < Dv; ++e)
                    o[e] += s[j] * oracle_load(v, b * sv[0] + g * sv[1] + j * sv[2] + e * sv[3], dtype);
            }
            for (int64_t e = 0; e < Dv; ++e) o[e] /= l;
        }
        if (probs) {
            for (int64_t j = 0; j < Lk; ++j) probs[r * Lk + j] = (l > 0.0) ? s[j] / l : 0.0;
        }
    }
    free(s);
    return 0;
}

/* Version tag so the Python side can check it loaded this file's build. */
int oracle_version(void) { return 2; }
