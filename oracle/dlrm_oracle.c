/*
 * Oracle for the DLRMv1 sparse/interaction stage: a plain, slow, obviously
 * correct CPU restatement of what the stage computes.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline do. It shares no header, helper, table or constant with the CUDA
 * library: every definition below is written out here on its own.
 *
 * Sources (the pages are git compare views of the luminal fork,
 * "luminal compare main...vanilla-pytorch"):
 *   - embedding_bag.rs, module doc comment: the pooled sum
 *         out[b, d] = sum over the bag's l of table[indices[b, l], d]
 *     with table (n_emb, d) f32 row-major, int32 indices, f32 output.
 *   - embedding_bag.rs, multi-table section doc comment: K independent
 *     (weight_k, idx_k) pairs fold into one (batch, num_tables, d) output;
 *     per-table row counts may differ, d and the bag length are shared.
 *   - movement.rs, translate_embedding_bag_forward_only: mode must be sum,
 *     no per-sample weights, bag length L = len(indices) / len(offsets).
 *   - dlrm_interact.rs, module doc comment: out[b, p] = sum_d v_i[b,d]*v_j[b,d]
 *     for every ordered pair with i > j, strict lower triangle, row-major over
 *     i then j (the torch.tril_indices(F, F, -1) convention).
 *   - dlrm_interact.rs, stacked-kernel doc comment: feature 0 is the dense
 *     vector, features 1..N are the N pooled embeddings, F = N + 1.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - offsets follow torch.nn.EmbeddingBag with include_last_offset=False,
 *     per table, relative to that table's own segment of B*L indices: bag b
 *     of table k is [offsets[k*B+b], next) where next is offsets[k*B+b+1],
 *     or B*L for the last bag. Offsets must satisfy 0 <= start <= end <= B*L.
 *   - an empty bag pools to the zero vector (torch sum mode).
 *   - an index outside [0, rows_k) is an error (the oracle rejects it).
 *   - the pooled sum is f32, accumulated from 0.0f in bag order, because the
 *     pages' kernels sum that way; dots are accumulated in fp64 over d in
 *     ascending order and rounded once to f32 at the end.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off (no -ffast-math),
 * so every f32 addition is one IEEE single-precision round-to-nearest add.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

/* Return codes of the oracle (its own; not shared with the library). */
#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_OFFSETS 2
#define ORACLE_INDEX_OOB 3

/* Largest table count accepted, as stated for the library's boundary. */
#define ORACLE_MAX_TABLES 256

static int check_shapes(int B, int F, int L, int D) {
    if (B < 1 || F < 1 || F > ORACLE_MAX_TABLES || L < 0 || D < 1) return ORACLE_BAD_ARG;
    if ((int64_t)B * (int64_t)L > (int64_t)INT32_MAX) return ORACLE_BAD_ARG;
    return ORACLE_OK;
}

/*
 * Bag bounds of (table k, sample b), the torch include_last_offset=False rule:
 * the bag starts at offsets[k][b] and ends where the next bag starts, or at the
 * end of the table's B*L index segment for the last bag.
 */
static int bag_bounds(const int32_t* offsets, int B, int L, int k, int b,
                      int64_t* start, int64_t* end) {
    const int64_t seg = (int64_t)B * (int64_t)L;
    int64_t s = offsets[(int64_t)k * B + b];
    int64_t e = (b + 1 < B) ? (int64_t)offsets[(int64_t)k * B + b + 1] : seg;
    if (s < 0 || s > e || e > seg) return ORACLE_BAD_OFFSETS;
    *start = s;
    *end = e;
    return ORACLE_OK;
}

/*
 * Multi-table EmbeddingBag, mode=sum.
 *   weights[k] : table k, rows[k] x D f32, row-major
 *   indices    : (F, B*L) int32, table-major
 *   offsets    : (F, B) int32
 *   out        : (B, F, D) f32, out[(b*F + k)*D + d]
 *   out_f64    : nullable, same layout, the same sums taken in fp64
 *   out_absum  : nullable, same layout, sum of |w| over the bag (error scale)
 * The whole input is validated first; on error nothing is written.
 */
int oracle_embbag_sum_multi(const float* const* weights, const int64_t* rows,
                            const int32_t* indices, const int32_t* offsets,
                            int B, int F, int L, int D, float* out,
                            double* out_f64, double* out_absum) {
    int rc = check_shapes(B, F, L, D);
    if (rc) return rc;
    if (!weights || !rows || !offsets || !out) return ORACLE_BAD_ARG;
    if (L > 0 && !indices) return ORACLE_BAD_ARG;
    const int64_t seg = (int64_t)B * (int64_t)L;

    for (int k = 0; k < F; ++k) {
        if (!weights[k] || rows[k] < 0) return ORACLE_BAD_ARG;
        for (int b = 0; b < B; ++b) {
            int64_t s, e;
            rc = bag_bounds(offsets, B, L, k, b, &s, &e);
            if (rc) return rc;
        }
        for (int64_t t = 0; t < seg; ++t) {
            int32_t r = indices[(int64_t)k * seg + t];
            if (r < 0 || (int64_t)r >= rows[k]) return ORACLE_INDEX_OOB;
        }
    }

    for (int b = 0; b < B; ++b) {
        for (int k = 0; k < F; ++k) {
            int64_t s, e;
            bag_bounds(offsets, B, L, k, b, &s, &e);
            const float* W = weights[k];
            const int32_t* idx = indices ? indices + (int64_t)k * seg : NULL;
            for (int d = 0; d < D; ++d) {
                float acc = 0.0f;
                double acc64 = 0.0;
                double absum = 0.0;
                for (int64_t t = s; t < e; ++t) {
                    float w = W[(int64_t)idx[t] * D + d];
                    acc = acc + w;
                    acc64 += (double)w;
                    absum += (w < 0.0f) ? -(double)w : (double)w;
                }
                int64_t o = ((int64_t)b * F + k) * D + d;
                out[o] = acc;
                if (out_f64) out_f64[o] = acc64;
                if (out_absum) out_absum[o] = absum;
            }
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * General pooling: ragged bags, include_last_offset, per-sample weights,
 * sum / mean / max, f32 or bf16 tables.
 *
 * The pages support only the fixed-stride, unweighted sum over f32 tables and
 * name the rest as what a later model would need (movement.rs,
 * translate_embedding_bag_forward_only: mean/max and per_sample_weights are
 * rejected with an error that says to extend it when a model needs them).
 * The semantics below are torch.nn.EmbeddingBag's, with these readings:
 *   - weighted sum: each step is one fused multiply-add, acc = fma(w_t, x, acc),
 *     from 0.0f in bag order (one rounding per entry);
 *   - mean: the f32 sum in bag order, then one division by the entry count;
 *     an empty bag gives 0;
 *   - max: the first entry, then acc = (x > acc) ? x : acc in bag order (ties,
 *     including -0 vs +0, keep the earlier value); an empty bag gives 0;
 *   - bf16 tables: a bf16 value is the upper 16 bits of an f32, so it is
 *     widened exactly by shifting its bits up by 16 before any arithmetic.
 * ------------------------------------------------------------------------ */
#define ORACLE_POOL_SUM 0
#define ORACLE_POOL_MEAN 1
#define ORACLE_POOL_MAX 2
#define ORACLE_TABLE_F32 0
#define ORACLE_TABLE_BF16 1

static float bf16_bits_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float table_value(const void* W, int dtype, int64_t row, int D, int d) {
    if (dtype == ORACLE_TABLE_BF16) return bf16_bits_to_f32(((const uint16_t*)W)[row * D + d]);
    return ((const float*)W)[row * D + d];
}

/* Bag b of table k when each table's offsets row holds B (+1) entries. */
static int bag_bounds_general(const int32_t* offsets, int B, int64_t T, int ilo, int k, int b,
                              int64_t* start, int64_t* end) {
    const int64_t row = (int64_t)B + (ilo ? 1 : 0);
    int64_t s = offsets[(int64_t)k * row + b];
    int64_t e = (ilo || b + 1 < B) ? (int64_t)offsets[(int64_t)k * row + b + 1] : T;
    if (s < 0 || s > e || e > T) return ORACLE_BAD_OFFSETS;
    *start = s;
    *end = e;
    return ORACLE_OK;
}

/*
 * weights[k] : rows[k] x D table, f32 or bf16 (raw 16-bit patterns)
 * indices    : (F, T) int32, table-major; psw : (F, T) f32 or NULL (sum only)
 * offsets    : (F, B) int32, or (F, B+1) with include_last_offset
 * out        : (B, F, D) f32
 * Only entries covered by some bag are read and must lie in [0, rows[k]).
 */
int oracle_embbag_pool_multi(const void* const* weights, int dtype, const int64_t* rows,
                             const int32_t* indices, const int32_t* offsets, const float* psw,
                             int64_t T, int include_last_offset, int mode, int B, int F, int D,
                             float* out) {
    if (B < 1 || F < 1 || F > ORACLE_MAX_TABLES || D < 1 || T < 0 || T > INT32_MAX)
        return ORACLE_BAD_ARG;
    if (mode != ORACLE_POOL_SUM && mode != ORACLE_POOL_MEAN && mode != ORACLE_POOL_MAX)
        return ORACLE_BAD_ARG;
    if (dtype != ORACLE_TABLE_F32 && dtype != ORACLE_TABLE_BF16) return ORACLE_BAD_ARG;
    if (psw && mode != ORACLE_POOL_SUM) return ORACLE_BAD_ARG;
    if (!weights || !rows || !offsets || !out) return ORACLE_BAD_ARG;
    if (T > 0 && !indices) return ORACLE_BAD_ARG;

    for (int k = 0; k < F; ++k) {
        if (!weights[k] || rows[k] < 0) return ORACLE_BAD_ARG;
        for (int b = 0; b < B; ++b) {
            int64_t s, e;
            int rc = bag_bounds_general(offsets, B, T, include_last_offset, k, b, &s, &e);
            if (rc) return rc;
            for (int64_t t = s; t < e; ++t) {
                int32_t r = indices[(int64_t)k * T + t];
                if (r < 0 || (int64_t)r >= rows[k]) return ORACLE_INDEX_OOB;
            }
        }
    }

    for (int b = 0; b < B; ++b) {
        for (int k = 0; k < F; ++k) {
            int64_t s, e;
            bag_bounds_general(offsets, B, T, include_last_offset, k, b, &s, &e);
            const int32_t* idx = indices ? indices + (int64_t)k * T : NULL;
            const float* wk = psw ? psw + (int64_t)k * T : NULL;
            for (int d = 0; d < D; ++d) {
                float acc = 0.0f;
                for (int64_t t = s; t < e; ++t) {
                    float x = table_value(weights[k], dtype, idx[t], D, d);
                    if (mode == ORACLE_POOL_MAX) {
                        acc = (t == s) ? x : ((x > acc) ? x : acc);
                    } else if (wk) {
                        acc = fmaf(wk[t], x, acc);
                    } else {
                        acc = acc + x;
                    }
                }
                if (mode == ORACLE_POOL_MEAN && e > s) acc = acc / (float)(e - s);
                out[((int64_t)b * F + k) * D + d] = acc;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Pair list of the strict lower triangle of an nf x nf matrix, written out by
 * the nested loop: i from 1 to nf-1, j from 0 to i-1, p counting up.
 * pi/pj receive nf*(nf-1)/2 entries each. Returns the count.
 */
int64_t oracle_pair_list(int nf, int32_t* pi, int32_t* pj) {
    int64_t p = 0;
    for (int i = 1; i < nf; ++i) {
        for (int j = 0; j < i; ++j) {
            if (pi) pi[p] = i;
            if (pj) pj[p] = j;
            ++p;
        }
    }
    return p;
}

/*
 * The dot of two length-D f32 vectors, every product taken exactly in fp64
 * (a product of two f32 fits in 48 bits) and summed in fp64 in ascending d.
 */
static double dot64(const float* a, const float* b, int D, double* absum) {
    double s = 0.0, m = 0.0;
    for (int d = 0; d < D; ++d) {
        double t = (double)a[d] * (double)b[d];
        s += t;
        m += (t < 0.0) ? -t : t;
    }
    if (absum) *absum = m;
    return s;
}

/*
 * Strict-lower-triangular pairwise-dot interaction over [dense, emb_0..emb_{F-1}].
 *   dense : (B, D) f32      -> feature 0
 *   emb   : (B, F, D) f32   -> features 1..F
 *   out   : (B, P) f32 with P = (F+1)F/2, or (B, D+P) when concat_dense != 0,
 *           in which case each row is [dense[b], z[b]]
 *   out_f64 : nullable (B, P), the dots before the final rounding to f32
 *   bound   : nullable (B, P), S_ij = sum_d |v_i[d] v_j[d]| (error scale)
 */
int oracle_interact_lower_tri(const float* dense, const float* emb, int B, int F, int D,
                              float* out, int concat_dense, double* out_f64, double* bound) {
    if (B < 1 || F < 1 || F > ORACLE_MAX_TABLES || D < 1) return ORACLE_BAD_ARG;
    if (!dense || !emb || !out) return ORACLE_BAD_ARG;
    const int nf = F + 1;
    const int64_t P = (int64_t)nf * (nf - 1) / 2;
    const int64_t row_len = concat_dense ? (int64_t)D + P : P;

    for (int b = 0; b < B; ++b) {
        float* row = out + (int64_t)b * row_len;
        float* z = row;
        if (concat_dense) {
            for (int d = 0; d < D; ++d) row[d] = dense[(int64_t)b * D + d];
            z = row + D;
        }
        int64_t p = 0;
        for (int i = 1; i < nf; ++i) {
            const float* vi = emb + ((int64_t)b * F + (i - 1)) * D;
            for (int j = 0; j < i; ++j) {
                const float* vj = (j == 0) ? dense + (int64_t)b * D
                                           : emb + ((int64_t)b * F + (j - 1)) * D;
                double m = 0.0;
                double s = dot64(vi, vj, D, &m);
                z[p] = (float)s;
                if (out_f64) out_f64[(int64_t)b * P + p] = s;
                if (bound) bound[(int64_t)b * P + p] = m;
                ++p;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * The whole stage: pooled = EmbeddingBag-sum over all F tables, then the
 * interaction over [dense, pooled]. pooled_out may be NULL (then a caller
 * buffer pooled_tmp of B*F*D floats must be given to hold it).
 */
int oracle_sparse_interact(const float* const* weights, const int64_t* rows,
                           const int32_t* indices, const int32_t* offsets,
                           const float* dense, int B, int F, int L, int D,
                           float* pooled_tmp, float* inter_out, int concat_dense,
                           double* bound) {
    if (!pooled_tmp) return ORACLE_BAD_ARG;
    int rc = oracle_embbag_sum_multi(weights, rows, indices, offsets, B, F, L, D,
                                     pooled_tmp, NULL, NULL);
    if (rc) return rc;
    return oracle_interact_lower_tri(dense, pooled_tmp, B, F, D, inter_out, concat_dense,
                                     NULL, bound);
}

/*
 * The end of a linear layer for one output: add the bias to the exact sum s
 * (and |bias| to the magnitude mag), apply the activation to acc + bias
 * (0 none, 1 ReLU max(x, 0), 2 sigmoid 1 / (1 + exp(-x))) and store.
 */
static void linear_finish(double s, double mag, const float* bias, int64_t n, int act,
                          int64_t at, double* out, double* pre, double* bound) {
    if (bias) {
        s += (double)bias[n];
        mag += fabs((double)bias[n]);
    }
    double y = s;
    if (act == 1) y = (s > 0.0) ? s : 0.0;
    if (act == 2) y = 1.0 / (1.0 + exp(-s));
    out[at] = y;
    if (pre) pre[at] = s;
    if (bound) bound[at] = mag;
}

/*
 * One DLRMv1 MLP layer, y = act(A W^T + bias), the linear-with-bias layer the
 * pages' matmul2d.rs page describes (linear_bias, linear_bias_relu,
 * linear_bias_sigmoid): A is (M, K), W is (N, K) (the nn.Linear weight
 * layout, "transpose_b"), bias is (N,), the activation is applied to
 * acc + bias. The split form of the same page (linear_bias_split_a and its
 * ReLU/Sigmoid variants) reads columns 0..k_lo-1 of A from a_lo and columns
 * k_lo..K-1 from a_hi, without building the concatenation.
 *
 * Operands are bf16 bit patterns (the tensor-core path takes bf16 operands;
 * see the design notes): a value is the f32 whose upper 16 bits are the
 * pattern. Every product of two such values is exact in fp64 and the sum is
 * taken in fp64 in ascending k, so out holds the exact layer up to fp64
 * rounding.
 *   a_lo  : (M, lda_lo) rows, columns [0, k_lo) used
 *   a_hi  : (M, lda_hi) rows, columns [0, k_hi) used; NULL when k_hi == 0
 *   w     : (N, ldw) rows, columns [0, k_lo + k_hi) used
 *   bias  : (N,) f32, or NULL for no bias
 *   act   : 0 none, 1 ReLU max(x, 0), 2 sigmoid 1 / (1 + exp(-x))
 *   out   : (M, N) fp64, the activation of the exact pre-activation
 *   pre   : nullable (M, N) fp64, the exact pre-activation acc + bias
 *   bound : nullable (M, N) fp64, sum_k |a_k w_k| + |bias| (error scale)
 */
int oracle_linear_bf16(const uint16_t* a_lo, int64_t lda_lo, int64_t k_lo,
                       const uint16_t* a_hi, int64_t lda_hi, int64_t k_hi,
                       const uint16_t* w, int64_t ldw, const float* bias,
                       int64_t M, int64_t N, int act, double* out, double* pre,
                       double* bound) {
    if (M < 1 || N < 1 || k_lo < 1 || k_hi < 0 || act < 0 || act > 2) return ORACLE_BAD_ARG;
    if (!a_lo || !w || !out || (k_hi > 0 && !a_hi)) return ORACLE_BAD_ARG;
    if (lda_lo < k_lo || (k_hi > 0 && lda_hi < k_hi) || ldw < k_lo + k_hi) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            const uint16_t* wn = w + n * ldw;
            double s = 0.0, mag = 0.0;
            for (int64_t k = 0; k < k_lo; ++k) {
                const double t = (double)bf16_bits_to_f32(a_lo[m * lda_lo + k]) *
                                 (double)bf16_bits_to_f32(wn[k]);
                s += t;
                mag += (t < 0.0) ? -t : t;
            }
            for (int64_t k = 0; k < k_hi; ++k) {
                const double t = (double)bf16_bits_to_f32(a_hi[m * lda_hi + k]) *
                                 (double)bf16_bits_to_f32(wn[k_lo + k]);
                s += t;
                mag += (t < 0.0) ? -t : t;
            }
            linear_finish(s, mag, bias, n, act, m * N + n, out, pre, bound);
        }
    }
    return ORACLE_OK;
}

/*
 * One DLRMv1 MLP layer with f32 activations: the mixed-precision linear the
 * pages' matmul2d.rs page describes (A is F32 (M, K), the weights are BF16
 * or F32 (N, K) by the kernel's weight_dtype, the result F32 (M, N)), with the
 * bias and activation of oracle_linear_bf16 and the same split form
 * (columns 0..k_lo-1 of A from a_lo, k_lo..K-1 from a_hi).
 *   a_lo, a_hi : f32 rows (row pitches lda_lo, lda_hi); a_hi NULL when k_hi == 0
 *   w          : (N, ldw) rows of f32 values (w_bf16 == 0) or of bf16 bit
 *                patterns (w_bf16 != 0)
 *   bias, act, out, pre, bound : as for oracle_linear_bf16
 * A product of two f32 values has at most 48 significant bits, so it is exact
 * in fp64; the sum is taken in fp64 in ascending k.
 */
static double weight_at(const void* w, int w_bf16, int64_t i) {
    if (w_bf16) return (double)bf16_bits_to_f32(((const uint16_t*)w)[i]);
    return (double)((const float*)w)[i];
}

int oracle_linear_f32a(const float* a_lo, int64_t lda_lo, int64_t k_lo,
                       const float* a_hi, int64_t lda_hi, int64_t k_hi,
                       const void* w, int w_bf16, int64_t ldw, const float* bias,
                       int64_t M, int64_t N, int act, double* out, double* pre,
                       double* bound) {
    if (M < 1 || N < 1 || k_lo < 1 || k_hi < 0 || act < 0 || act > 2) return ORACLE_BAD_ARG;
    if (!a_lo || !w || !out || (k_hi > 0 && !a_hi)) return ORACLE_BAD_ARG;
    if (lda_lo < k_lo || (k_hi > 0 && lda_hi < k_hi) || ldw < k_lo + k_hi) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0, mag = 0.0;
            for (int64_t k = 0; k < k_lo; ++k) {
                const double t = (double)a_lo[m * lda_lo + k] * weight_at(w, w_bf16, n * ldw + k);
                s += t;
                mag += (t < 0.0) ? -t : t;
            }
            for (int64_t k = 0; k < k_hi; ++k) {
                const double t =
                    (double)a_hi[m * lda_hi + k] * weight_at(w, w_bf16, n * ldw + k_lo + k);
                s += t;
                mag += (t < 0.0) ? -t : t;
            }
            linear_finish(s, mag, bias, n, act, m * N + n, out, pre, bound);
        }
    }
    return ORACLE_OK;
}
