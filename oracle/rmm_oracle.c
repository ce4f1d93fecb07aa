/*
 * rmm_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU statement of Reduced Matrix
 * Multiplication (RMM) in fp64.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this code; the product path never does.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Source: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
 * Reduction for LLM Inference" (arXiv 2608.13426), called "the RMM paper" below.
 *
 * Every array is row-major with an explicit leading dimension (elements).
 * All arithmetic is IEEE fp64; inputs that were bf16 or fp32 on the GPU side
 * are widened exactly to fp64 by the caller before they reach this file.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/*
 * Retained count k = ceil(rho * d)  [RMM paper, §3.2, definition of RMM_rho].
 *
 * Reading of the rounding: the product rho*d is formed in fp64; when it lies
 * within 1e-9*d of an integer it is taken to be that integer (so that, e.g.,
 * rho = 0.07, d = 100 gives 7 and not 8 through fp64 representation error);
 * otherwise the ceiling is taken.  The result is clamped to [1, d].
 * Returns -1 when rho is outside (0, 1] or d < 1.
 */
int64_t rmm_oracle_retained_count(double rho, int64_t d)
{
    if (d < 1 || !(rho > 0.0) || rho > 1.0)
        return -1;
    double x = rho * (double)d;
    double r = nearbyint(x);
    int64_t k;
    if (fabs(x - r) <= 1e-9 * (double)d)
        k = (int64_t)r;
    else
        k = (int64_t)ceil(x);
    if (k < 1) k = 1;
    if (k > d) k = d;
    return k;
}

/*
 * Squared column scores s2[j] = sum_i A[i,j]^2, i.e. ||A[:,j]||_2^2
 * [RMM paper, §3.2 "Activation-aware dimension selection"; §3.3 uses the same
 * score on Q (attention features), on P (token positions) and on X (MLP)].
 * Ordering by s2 equals ordering by s = sqrt(s2), so the square root is not
 * taken.  Rows are summed in increasing order.
 */
void rmm_oracle_column_scores_sq(const double *A, int64_t n, int64_t d,
                                 int64_t lda, double *s2)
{
    for (int64_t j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            double a = A[i * lda + j];
            acc += a * a;
        }
        s2[j] = acc;
    }
}

/* Sort key for the full sort in rmm_oracle_topk_indices. */
typedef struct {
    double key;
    int64_t index;
} scored_index;

/* Larger score first; equal scores: lower index first (the tie reading). */
static int by_score_desc_then_index(const void *pa, const void *pb)
{
    const scored_index *a = (const scored_index *)pa;
    const scored_index *b = (const scored_index *)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    if (a->index < b->index) return -1;
    if (a->index > b->index) return 1;
    return 0;
}

static int by_int32_asc(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * I = TopK({s_j}, k)  [RMM paper, §3.2]: the k indices with the largest
 * scores.  The paper calls the rule "fully deterministic" but states no
 * tie-break; the reading here is that among equal scores the lower index is
 * kept.  The paper states no order for I; the reading here is ascending.
 * Implementation: one full sort of all d indices by (score descending,
 * index ascending), keep the first k, then sort those k ascending.
 * Returns 0, or -1 on a bad argument or allocation failure.
 */
int rmm_oracle_topk_indices(const double *s2, int64_t d, int64_t k, int32_t *I)
{
    if (d < 1 || k < 1 || k > d)
        return -1;
    scored_index *all = (scored_index *)malloc((size_t)d * sizeof(scored_index));
    if (!all)
        return -1;
    for (int64_t j = 0; j < d; ++j) {
        all[j].key = s2[j];
        all[j].index = j;
    }
    qsort(all, (size_t)d, sizeof(scored_index), by_score_desc_then_index);
    for (int64_t t = 0; t < k; ++t)
        I[t] = (int32_t)all[t].index;
    free(all);
    qsort(I, (size_t)k, sizeof(int32_t), by_int32_asc);
    return 0;
}

/*
 * Y = A[:, I] * B[I, :]  [RMM paper, §3.2, definition of RMM_rho; §3.4 and
 * Appendix D.1, Eq. (3)-(4) for the cost O(n k m)].
 * Y[i,c] = sum over t = 0..k-1 (I ascending) of A[i, I[t]] * B[I[t], c].
 * A is n x (any width >= max(I)+1) with leading dimension lda; B has rows
 * indexed by I and m columns with leading dimension ldb; Y is n x m.
 * Output rows are independent, so they may run on several threads; the
 * order of the sum inside each element does not change.
 */
void rmm_oracle_reduced_product(const double *A, int64_t lda,
                                const double *B, int64_t ldb,
                                int64_t n, int64_t m,
                                const int32_t *I, int64_t k,
                                double *Y, int64_t ldy)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double *y = Y + i * ldy;
        for (int64_t c = 0; c < m; ++c)
            y[c] = 0.0;
        for (int64_t t = 0; t < k; ++t) {
            int64_t j = I[t];
            double a = A[i * lda + j];
            const double *b = B + j * ldb;
            for (int64_t c = 0; c < m; ++c)
                y[c] += a * b[c];
        }
    }
}

/*
 * Reduced attention scores for one head [RMM paper, §3.3 "Attention"]:
 *   S[i, c] = alpha * sum over t (I ascending) of Q[i, I[t]] * K[c, I[t]]
 * where the paper's alpha is 1/sqrt(d_h) with the full head dimension d_h.
 * The contraction runs over the feature axis of both Q (nq x d_h) and
 * K (nk x d_h).  When causal != 0 the paper's optional mask M is the
 * aligned causal mask: entries with key index c > query index are -inf.
 * Row i of Q is query number row0 + i (row0 lets a caller pass a slice).
 */
void rmm_oracle_reduced_scores(const double *Q, int64_t ldq,
                               const double *K, int64_t ldk,
                               int64_t nq, int64_t nk, int64_t row0,
                               const int32_t *I, int64_t k,
                               double alpha, int causal,
                               double *S, int64_t lds)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nq; ++i) {
        for (int64_t c = 0; c < nk; ++c) {
            if (causal && c > row0 + i) {
                S[i * lds + c] = -INFINITY;
                continue;
            }
            double acc = 0.0;
            for (int64_t t = 0; t < k; ++t) {
                int64_t j = I[t];
                acc += Q[i * ldq + j] * K[c * ldk + j];
            }
            S[i * lds + c] = alpha * acc;
        }
    }
}

/*
 * Attention weights of one head, P = softmax(S + M)  [RMM paper, §3.3
 * "Attention": P = softmax(S~ + M), M the optional causal or attention mask;
 * the softmax normalises each query row over the key axis].  The mask is
 * already in S as -inf entries (the causal form written by
 * rmm_oracle_reduced_scores), and such entries get weight exactly 0.
 * Row i, with mu_i = max_c S[i,c]:
 *   P[i,c] = exp(S[i,c] - mu_i) / sum over c' of exp(S[i,c'] - mu_i).
 * Subtracting mu_i changes nothing in exact arithmetic and keeps every exp
 * finite.  Returns 0, or -1 when some row has no finite entry (out of
 * contract: the mask leaves every query at least its own key).
 */
int rmm_oracle_softmax_rows(const double *S, int64_t lds, int64_t n, int64_t t,
                            double *P, int64_t ldp)
{
    int bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        const double *s = S + i * lds;
        double *p = P + i * ldp;
        double mu = -INFINITY;
        for (int64_t c = 0; c < t; ++c)
            if (s[c] > mu) mu = s[c];
        if (!(mu > -INFINITY)) {
            bad = 1;
            continue;
        }
        double sum = 0.0;
        for (int64_t c = 0; c < t; ++c) {
            double e = (s[c] == -INFINITY) ? 0.0 : exp(s[c] - mu);
            p[c] = e;
            sum += e;
        }
        for (int64_t c = 0; c < t; ++c)
            p[c] = p[c] / sum;
    }
    return bad ? -1 : 0;
}

/*
 * Exact value of 8-bit floating-point codes in the E4M3 format of the OCP
 * 8-bit floating point specification (the "e4m3fn" variant: no infinities,
 * the all-ones exponent and mantissa is NaN, largest magnitude 448).  The
 * RMM paper runs RMM alongside 8-bit weight quantization (App. B.6) and names
 * dedicated low-bit kernels as future work (App. B.7); the low-bit form here
 * stores A and B in this format with per-tensor scales folded into the
 * output scale alpha, and the method's arithmetic (scores, TopK, product)
 * runs on the exact decoded values.
 * Bit layout: sign s (bit 7), exponent e (bits 6..3, bias 7), mantissa f
 * (bits 2..0).  e = 0: (-1)^s * f * 2^-9 (subnormal); otherwise
 * (-1)^s * 2^(e-7) * (1 + f/8).  Returns 0, or -1 if a code is NaN.
 */
int rmm_oracle_decode_e4m3(const uint8_t *codes, int64_t count, double *out)
{
    int bad = 0;
    for (int64_t i = 0; i < count; ++i) {
        unsigned b = codes[i];
        unsigned s = b >> 7, e = (b >> 3) & 15u, f = b & 7u;
        double v;
        if (e == 15u && f == 7u) {
            v = NAN;
            bad = 1;
        } else if (e == 0u) {
            v = ldexp((double)f, -9);
        } else {
            v = ldexp(1.0 + (double)f / 8.0, (int)e - 7);
        }
        out[i] = s ? -v : v;
    }
    return bad ? -1 : 0;
}
