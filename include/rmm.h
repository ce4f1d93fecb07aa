/*
 * rmm.h -- C ABI of librmm, Reduced Matrix Multiplication (RMM) on NVIDIA B200
 * (sm_100a).
 *
 * Method: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
 * Reduction for LLM Inference" (arXiv 2608.13426), "the RMM paper" below.
 * For Y = A B with A in R^{n x d} (activations) and B in R^{d x m}, RMM
 *   1. scores every contraction index j by s_j = ||A[:, j]||_2        (§3.2)
 *   2. keeps I = TopK({s_j}, k), k = ceil(rho d), rho in (0, 1]         (§3.2)
 *   3. returns A[:, I] B[I, :]                                         (§3.2)
 * and has per-head forms for attention (§3.3): QK^T with features chosen
 * per query head from Q's column norms (grouped-query attention gathers the
 * same features of the shared K head), scaled by alpha (the paper uses
 * 1/sqrt(d_h)) and optionally causally masked; and PV with token positions
 * chosen per head from the column norms of P.
 *
 * Readings where the paper is silent (fixed by this library):
 *   - ties between equal scores keep the lower index;
 *   - I is returned in ascending order, int32;
 *   - k = ceil(rho d), except that a product rho*d within 1e-9 d of an
 *     integer counts as that integer; k is clamped to [1, d];
 *   - the causal mask writes -inf where key index > query index (QK); for
 *     PV the same flag states that P is zero above its diagonal;
 *   - scores are accumulated in fp32 from the stored values; the product
 *     accumulates in fp32 (bf16 inputs) or tf32 (fp32 inputs) and is stored
 *     in the input dtype.
 *
 * Memory: every pointer passed to a compute call is DEVICE memory on the
 * current CUDA device, owned by the caller, and must be 16-byte aligned (the
 * workspace 256-byte aligned).  The library never allocates device memory.
 * A plan is host memory owned by the caller through create/destroy.
 *
 * Execution: compute calls only enqueue kernels on `stream` (a cudaStream_t
 * passed as void*; NULL = the legacy default stream) and return without
 * synchronising, so they can be captured in a CUDA graph.  Kernels are
 * launched with programmatic stream serialisation: one may be scheduled while
 * the work before it on the stream drains, and waits for that work to finish
 * before it touches global memory.  Argument errors are detected on the host before anything
 * is enqueued; outputs are then untouched.  A kernel that gives up on an
 * internal wait (bounded at about two seconds) records it in the workspace;
 * rmm_workspace_status() reports it.  One plan and one workspace may be used
 * by one stream at a time.  Nothing is thrown across this ABI.
 */
#ifndef RMM_H_
#define RMM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RMM_API __attribute__((visibility("default")))
#else
#define RMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rmm_status {
    RMM_OK = 0,
    RMM_ERR_INVALID_ARG = 1,  /* a NULL, misaligned, out-of-range or inconsistent argument */
    RMM_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement (e.g. d too large) */
    RMM_ERR_WORKSPACE = 3,    /* workspace missing, too small or misaligned */
    RMM_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (launch, attribute, encode) */
    RMM_ERR_TIMEOUT = 5       /* a kernel gave up on an internal wait (see rmm_workspace_status) */
} rmm_status;

typedef enum rmm_dtype {
    RMM_BF16 = 0, /* bfloat16 storage, fp32 accumulation (tcgen05 kind::f16) */
    RMM_F32 = 1,  /* fp32 storage, tf32 products with fp32 accumulation (tcgen05 kind::tf32) */
    /* Low-bit form (the RMM paper runs RMM next to 8-bit weight quantization,
       App. B.6, and names dedicated low-bit kernels as future work, App. B.7):
       A and B hold 8-bit E4M3 codes (OCP 8-bit floating point, e4m3fn: no
       infinities, largest magnitude 448), Y is bfloat16.  Per-tensor scales go
       into alpha: Y = alpha * A[:, I] B[I, :] over the decoded codes, so a
       caller with A = sa * Aq and B = sb * Bq passes alpha = sa * sb.  Scores
       are sums of squares of the decoded codes (a positive per-tensor scale
       does not change I); products on tcgen05 kind::f8f6f4 with fp32
       accumulation.  LINEAR with one head only, n = 0 or n > 128
       (RMM_ERR_UNSUPPORTED otherwise); d, m, lda and ldb multiples of 16;
       ldy a multiple of 8 (bf16 elements). */
    RMM_FP8_E4M3 = 2
} rmm_dtype;

typedef enum rmm_mode {
    /* Y[h] = RMM(A[h], B[g]): A n x d (lda), B d x m (ldb, row j = contraction
       index j), Y n x m (ldy).  The RMM paper §3.2, §3.3 "MLP and linear
       projections". */
    RMM_LINEAR = 0,
    /* S[h] = alpha * Q[h][:, I_h] K[g][:, I_h]^T (+ causal mask): A = Q[h] is
       n x d with d = d_h (lda), B = K[g] is m x d (ldb; m = number of keys,
       the contraction axis is contiguous), Y = S[h] is n x m.  I_h is chosen
       from Q[h]'s column norms.  The RMM paper §3.3 "Attention". */
    RMM_QK = 1,
    /* O[h] = P[h][:, T_h] V[g][T_h, :]: A = P[h] is n x d with d = number of
       key tokens (lda), B = V[g] is d x m (ldb; m = d_v), Y = O[h] is n x m.
       T_h is chosen from P[h]'s column norms.  The RMM paper §3.3, last
       sentence of "Attention"; Appendix D.1 Eq. (2). */
    RMM_PV = 2
} rmm_mode;

/* Causal structure.  QK: the output is masked, S[i][c] = -inf for c > i.
   PV (n = d, query i is token i): the caller guarantees P[h][i][t] = 0 for
   t > i, as a causal softmax leaves it; the op then skips the blocks of P that
   lie entirely above the diagonal when it forms the token scores and the
   product, which gives the same result as reading them.  Other modes:
   RMM_ERR_INVALID_ARG. */
#define RMM_FLAG_CAUSAL 1u
/* rmm_matmul*: take I from the caller (I_inout, [heads][k], ascending,
   distinct, each in [0, d)) instead of computing it; no scores are formed. */
#define RMM_FLAG_USE_GIVEN_INDICES 2u
/* Producer-fused scoring (the RMM paper §3.3 "Attention" scores tokens by the
   column norms of P, and Appendix D.1 "Practical implications" asks for the
   norms to be computed efficiently).  rmm_matmul_ex only:
   RMM_FLAG_GIVEN_SCORES -- take the column scores of A from the caller
   (s2_in[h][j] = fp32 sum_i A[h][i][j]^2, as written by the op that produced
   A: RMM_FLAG_EMIT_SCORES of an earlier product, or rmm_softmax_scores)
   instead of reading A for them; I = TopK of s2_in, exactly as if the op had
   computed those scores.  Not with RMM_FLAG_USE_GIVEN_INDICES.
   RMM_FLAG_EMIT_SCORES -- also write the column scores of this op's output,
   s2_out[h][c] = fp32 sum_i Y[h][i][c]^2 over the stored (rounded) values,
   summed in a fixed order (the same bits on every call), so that an op
   taking Y as its A can skip its score pass.  LINEAR and PV only. */
#define RMM_FLAG_GIVEN_SCORES 4u
#define RMM_FLAG_EMIT_SCORES 8u

/* One problem shape.  All sizes and strides count ELEMENTS.  Heads: query
   head h (0 <= h < heads) reads A, I and Y at offset h * stride_{a,y} and B at
   offset g * stride_b with g = h / (heads / kv_heads) (grouped-query sharing;
   kv_heads = heads means one B per head, kv_heads = 1 one shared B). */
typedef struct rmm_problem {
    int32_t mode;      /* rmm_mode */
    int32_t dtype;     /* rmm_dtype of A, B and Y (E4M3: A and B; Y is bf16) */
    int64_t n;         /* rows of A and Y (tokens / queries), >= 0 */
    int64_t d;         /* contraction size, >= 1, multiple of 8 (bf16) or 4 (fp32) */
    int64_t m;         /* columns of Y, >= 0, multiple of 8 (bf16) or 4 (fp32) */
    int64_t lda, ldb, ldy; /* row strides; multiples of 16 bytes; lda >= d, ldy >= m,
                              ldb >= m (LINEAR, PV) or >= d (QK) */
    int64_t heads;     /* >= 1 */
    int64_t kv_heads;  /* >= 1, divides heads */
    int64_t stride_a, stride_b, stride_y; /* per-head strides (multiples of 16 bytes);
                                             ignored when the count of that operand is 1 */
    double rho;        /* retention ratio in (0, 1]; used when k == 0 */
    int64_t k;         /* 0: k = ceil(rho d) (see readings above); else 1 <= k <= d */
    float alpha;       /* output scale applied in fp32 before rounding; QK: 1/sqrt(d_h) */
    uint32_t flags;    /* RMM_FLAG_* */
} rmm_problem;

typedef struct rmm_plan rmm_plan;

/* Fill *p with defaults for a single-head LINEAR problem (alpha 1, rho 1,
   dense row-major strides lda = d, ldb = m, ldy = m). */
RMM_API void rmm_problem_init(rmm_problem* p, int32_t mode, int32_t dtype, int64_t n, int64_t d,
                      int64_t m);

/* Validate *p, fix k and the kernel choices, and report the workspace the
   compute calls need (bytes, may be 0 only for n == 0 or m == 0 problems).
   Reads the current CUDA device's SM count.  On error *plan is set to NULL. */
RMM_API rmm_status rmm_plan_create(rmm_plan** plan, const rmm_problem* p, size_t* workspace_bytes);

/* Release a plan (NULL is allowed). */
RMM_API rmm_status rmm_plan_destroy(rmm_plan* plan);

/* The number of retained indices k of a plan (-1 for NULL). */
RMM_API int64_t rmm_plan_k(const rmm_plan* plan);

/* Workspace size of a plan in bytes (0 for NULL). */
RMM_API size_t rmm_plan_workspace_size(const rmm_plan* plan);

/* Selection only (§3.2 scores + TopK): for every head write I[h][0..k) in
   ascending order and, when s2 != NULL, s2[h][0..d) = fp32 sum_i A[h][i][j]^2.
   A: as in the plan.  I: device int32 [heads][k].  s2: device fp32 [heads][d]
   or NULL. */
RMM_API rmm_status rmm_select(const rmm_plan* plan, const void* A, int32_t* I, float* s2,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Selection without any device allocation.  The RMM paper has no counterpart:
   this is a deployment convenience.  Same result as rmm_select (I ascending,
   optional fp32 s2), for callers that cannot allocate device memory when they
   need an index set (a frozen or captured memory pool, a plugin inside
   another runtime's allocator, a process with a fixed memory budget).  Plans
   whose selection runs in one kernel per head (few rows, one row, or a small
   head; the same kernel rmm_select takes) use no scratch at all.  Otherwise
   the scratch of the score pass (partials, completion counters, final
   scores) lives in one 8 MiB file-scope device array inside this library,
   held by every GPU that loads it until the process exits; the caller passes
   only A, I and s2.  Limits: heads * d * 4 * (nsplit + 1) bytes plus the
   counters must fit in 8 MiB (nsplit <= 16, chosen by the plan; e.g.
   d = 28672 with one head fits), else RMM_ERR_UNSUPPORTED and nothing is
   launched.  The array's device address is looked up (cudaGetSymbolAddress)
   with the calling thread's current device and context on the first such call
   in that context, and again whenever the context changes (e.g. after
   cudaDeviceReset); make that first call before any stream capture.  `stream`
   must belong to the current device (RMM_ERR_INVALID_ARG otherwise: the
   address is that device's).  Every call reuses the same array and it keeps
   the last call's contents (the counters are cleared on the stream at the
   start of each call): calls that overlap on the GPU -- two streams, or two
   host threads -- race and corrupt each other's results; serialise them.
   Calls no cudaMalloc, cudaFree or other allocating routine. */
RMM_API rmm_status rmm_select_no_alloc(const rmm_plan* plan, const void* A, int32_t* I, float* s2,
                                       void* stream);

/* Full op for a plan with heads == 1: Y = A[:, I] B[I, :] (LINEAR, PV) or
   alpha * A[:, I] B[:, I]^T with the optional causal mask (QK).
   I_inout: NULL, or device int32 [k] that receives I (or supplies it with
   RMM_FLAG_USE_GIVEN_INDICES).  Y must not overlap A, B or the workspace. */
RMM_API rmm_status rmm_matmul(const rmm_plan* plan, const void* A, const void* B, void* Y,
                      int32_t* I_inout, void* workspace, size_t workspace_bytes, void* stream);

/* Same as rmm_matmul for any number of heads; I_inout is [heads][k].
   rmm_matmul and rmm_matmul_batched return RMM_ERR_INVALID_ARG for a plan
   with RMM_FLAG_GIVEN_SCORES or RMM_FLAG_EMIT_SCORES (use rmm_matmul_ex). */
RMM_API rmm_status rmm_matmul_batched(const rmm_plan* plan, const void* A, const void* B, void* Y,
                              int32_t* I_inout, void* workspace, size_t workspace_bytes,
                              void* stream);

/* rmm_matmul_batched with producer-fused scoring.  s2_in: device fp32
   [heads][d], the column scores of A; required with RMM_FLAG_GIVEN_SCORES,
   else ignored.  s2_out: device fp32 [heads][m], receives the column scores
   of Y; required with RMM_FLAG_EMIT_SCORES, else ignored.  On the CTA-pair
   product (more than 128 rows) the scores come from the product's epilogue:
   each warp squares its 32 x 32 block of stored outputs, sums the 32 rows of
   each column, and the last block of a column adds the row blocks' sums in
   row order; other shapes add one score pass over Y after the product.
   Errors: a required pointer NULL or not 4-byte aligned, RMM_ERR_INVALID_ARG. */
RMM_API rmm_status rmm_matmul_ex(const rmm_plan* plan, const void* A, const void* B, void* Y,
                                 int32_t* I_inout, const float* s2_in, float* s2_out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Attention weights with producer-fused token scores: the op that produces
   P for an RMM PV call (the RMM paper §3.3 "Attention": P = softmax(S~ + M);
   the PV product then keeps the tokens with the largest a_t = ||P[:, t]||).
   For each head h and row i of S[h] (n x t bf16, row stride lds, head
   stride stride_s, -inf entries are masked keys) it writes
     P[h][i][c] = exp(S[h][i][c] - max_c' S[h][i][c']) / sum_c' exp(...)
   rounded to bf16 (row stride ldp, head stride stride_p), and
     s2[h][c] = fp32 sum over i of P[h][i][c]^2 of the stored values,
   each thread's rows summed in row order and the row blocks in block order
   (the same bits on every call); pass s2 as s2_in of an RMM_PV plan with
   RMM_FLAG_GIVEN_SCORES.  flags: RMM_FLAG_CAUSAL states S[h][i][c] = -inf
   for c > i (those entries are not read; P is written as 0 there).  Every
   row needs a finite entry.  Sizes: t a multiple of 8, t <= 8192; strides
   multiples of 8 elements, lds and ldp >= t.  workspace: device memory of
   rmm_softmax_workspace_size(heads, n, t) bytes, 256-byte aligned, its
   first word (an error word) zeroed once (cudaMemsetAsync) before its first
   use: if the kernel gives up waiting for a row of S to arrive in shared
   memory (about two seconds) it writes a nonzero code there.  Two launches:
   the weights with per-row-block column sums, then their sum in block order.
   Errors: RMM_ERR_INVALID_ARG / RMM_ERR_UNSUPPORTED / RMM_ERR_WORKSPACE
   before any launch, RMM_ERR_CUDA if a launch fails. */
RMM_API size_t rmm_softmax_workspace_size(int64_t heads, int64_t n, int64_t t);
RMM_API rmm_status rmm_softmax_scores(const void* S, void* P, float* s2, int64_t heads, int64_t n, int64_t t,
                                      int64_t lds, int64_t stride_s, int64_t ldp, int64_t stride_p, uint32_t flags,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* Zero the workspace's header (its error word, the score pass's completion
   counters and the product's split-tail counters, which the kernels return to
   zero) on `stream`.  Call once after allocating a workspace, before the
   first compute call. */
RMM_API rmm_status rmm_workspace_init(const rmm_plan* plan, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Synchronise `stream` and read the workspace's error word: RMM_OK, or
   RMM_ERR_TIMEOUT if a kernel gave up on a wait since the last check (the
   word is then cleared), or RMM_ERR_CUDA if the stream reports an error. */
RMM_API rmm_status rmm_workspace_status(const rmm_plan* plan, void* workspace, void* stream);

/* Self-test of the failure path (the pages have no counterpart): launches
   one CTA on `stream` that waits, with the library's bounded wait, on a
   barrier nothing ever completes.  After the wait limit (2 s) the CTA records
   a timeout in the workspace's error word and exits, exactly as a kernel of
   the op does when a peer stage never arrives; the context stays usable and
   the next rmm_workspace_status reports RMM_ERR_TIMEOUT.  Errors: NULL plan or
   workspace, or a workspace smaller than the plan's, RMM_ERR_WORKSPACE /
   RMM_ERR_INVALID_ARG before any launch. */
RMM_API rmm_status rmm_selftest_wait_timeout(const rmm_plan* plan, void* workspace, size_t workspace_bytes,
                                             void* stream);

/* Tracing hook.  When both are non-NULL, every later rmm_matmul* call with
   this plan records `start` immediately before and `stop` immediately after
   the launch of its reduced-product kernel, on the call's stream, so that
   cudaEventElapsedTime isolates that kernel (the RMM paper §6.3 times the
   whole operation, norms + TopK + product; this separates the last step).
   The events are cudaEvent_t passed as void*, created by the caller; NULL
   clears the hook.  Not thread-safe with concurrent calls on the plan. */
RMM_API rmm_status rmm_plan_set_product_events(rmm_plan* plan, void* start, void* stop);

/* Number of kernels one rmm_matmul* call of this plan launches (-1 for NULL). */
RMM_API int32_t rmm_plan_kernel_launches(const rmm_plan* plan);

/* Fused RMM attention (self-attention, one call for all heads): the RMM
   paper's three steps of §3.3 "Attention" without writing the score matrix
   or the weights.  Per query head h (grouped-query K/V head g = h / (heads /
   kv_heads)): I_h = TopK of Q[h]'s column norms, k_d = ceil(rho_d d_h);
   S = alpha Q[h][:, I_h] K[g][:, I_h]^T (-inf above the diagonal with
   RMM_FLAG_CAUSAL); P = softmax(S) over each row; T_h = TopK of P's column
   norms, k_t = ceil(rho_t n); O[h] = P[:, T_h] V[g][T_h, :].  The scores are
   recomputed in three passes (row statistics; token scores, which need every
   row's final normalisation; the output over the key blocks that hold a kept
   token), on the tensor cores; the token scores are fp32 sums of P^2 of the
   fp32 weights, and the product rounds P to bf16.  Ties keep the lower index;
   I and T are ascending.  The pages' own attention kernels were not fully
   fused (App. B.7); this form has no counterpart there beyond the method. */
typedef struct rmm_attn_problem {
    int64_t heads, kv_heads;  /* query heads; K/V heads, dividing heads */
    int64_t n;                /* queries = keys per head, a multiple of 8, <= 49152 */
    int64_t d_h, d_v;         /* both 128 (RMM_ERR_UNSUPPORTED otherwise) */
    int64_t ldq, ldk, ldv, ldo;                      /* row strides, multiples of 8 elements */
    int64_t stride_q, stride_k, stride_v, stride_o;  /* head strides (elements) */
    double rho_d, rho_t;      /* feature and token retention ratios in (0, 1] */
    float alpha;              /* score scale; the paper's 1/sqrt(d_h) */
    uint32_t flags;           /* RMM_FLAG_CAUSAL or 0 */
} rmm_attn_problem;

/* Workspace bytes rmm_attention needs for *p (0 for an invalid problem).
   Reads the current device's SM count. */
RMM_API size_t rmm_attention_workspace_size(const rmm_attn_problem* p);

/* Q [heads][n][d_h], K [kv_heads][n][d_h], V [kv_heads][n][d_v], O
   [heads][n][d_v]: bf16 device memory, 16-byte aligned.  I_out ([heads][k_d])
   and T_out ([heads][k_t]) receive the index sets when not NULL.  workspace:
   device memory of rmm_attention_workspace_size(p) bytes, 256-byte aligned,
   its first word (an error word) zeroed once (cudaMemsetAsync) before its
   first use: a kernel that gives up on a wait (about two seconds) writes a
   nonzero code there.  Asynchronous on `stream`.
   Errors: RMM_ERR_INVALID_ARG / RMM_ERR_UNSUPPORTED / RMM_ERR_WORKSPACE before
   any launch, RMM_ERR_CUDA if a launch fails. */
RMM_API rmm_status rmm_attention(const rmm_attn_problem* p, const void* Q, const void* K, const void* V, void* O,
                                 int32_t* I_out, int32_t* T_out, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* Static string naming a status code. */
RMM_API const char* rmm_status_string(rmm_status s);

/* Library version, "major.minor.patch". */
RMM_API const char* rmm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RMM_H_ */
