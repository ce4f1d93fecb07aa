// rmm_internal.h -- launchers shared between the C-ABI layer (rmm_api.cu) and
// the kernels.  Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm.h"

namespace rmm {

// ---------------------------------------------------------------- launches
// Every kernel of the library is launched with programmatic stream
// serialisation: it may be scheduled while the previous kernel on the stream
// is still running, and it calls pdl_wait() before its first global memory
// access (reads of what earlier work wrote, and writes that earlier work may
// still read); pdl_wait() returns once every earlier kernel has completed and
// its writes are visible.  pdl_trigger() lets the next kernel be scheduled.
// Work before pdl_wait() touches only shared memory, tensor memory and the
// kernel's parameters.
#if defined(__CUDACC__)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// TopK of 32 J keys held by one warp (lane l holds the keys of columns
// l + 32 j; keys are the bit patterns of non-negative fp32 scores, which order
// as the scores do): bit j of the result is set when column lane + 32 j is
// among the k largest, ties going to the lower column.  The k-th largest key
// T is found bit by bit (the largest T with at least k keys >= T); the keys
// equal to T are then kept in column order until k are kept.  Columns past
// the end must hold key 0 and `valid` false.
template <int J>
__device__ __forceinline__ uint32_t warp_topk_bits(const uint32_t (&key)[J], const bool (&valid)[J], uint32_t k,
                                                   int lane) {
    uint32_t T = 0u;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        uint32_t c = 0u;
#pragma unroll
        for (int j = 0; j < J; ++j) c += (valid[j] && key[j] >= cand) ? 1u : 0u;
        if (__reduce_add_sync(0xffffffffu, c) >= k) T = cand;
    }
    uint32_t gt = 0u;
#pragma unroll
    for (int j = 0; j < J; ++j) gt += (valid[j] && key[j] > T) ? 1u : 0u;
    const uint32_t r = k - __reduce_add_sync(0xffffffffu, gt);  // keys equal to T that are kept
    uint32_t kept = 0u, eq_before = 0u;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const bool eq = valid[j] && key[j] == T;
        const unsigned b = __ballot_sync(0xffffffffu, eq);
        const uint32_t rank = eq_before + __popc(b & ((1u << lane) - 1u));
        if ((valid[j] && key[j] > T) || (eq && rank < r)) kept |= 1u << j;
        eq_before += __popc(b);
    }
    return kept;
}
#endif

template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// ---------------------------------------------------------------- selection
struct SelectArgs {
    const void* A;       // [heads][n][lda]
    int dtype;           // RMM_BF16 / RMM_F32
    int64_t n, d, lda, stride_a;
    int heads;
    int64_t k;
    int32_t* I;          // [heads][k] out, ascending
    float* s2;           // [heads][d] out or nullptr
    // two-stage path only
    float* partials;     // [heads][nsplit][d]
    unsigned* counters;  // [heads][column blocks], zero between calls
    float* scores;       // [heads][d] final fp32 scores (may alias s2)
    int nsplit;          // 1 .. kMaxSplitRows
    int64_t rows_per_split;
    int causal_rows;     // A[i][j] = 0 for j > i: a column block skips the rows above it
    uint32_t* mask;      // [heads][mask_words] membership bits of I (bit j of word j / 32), or nullptr
    int64_t mask_words;  // ceil(d / 32) when mask is set
};
constexpr int kMaxSplitRows = 64;

// Column sums of squares in fp32: one partial per row split, then the last
// CTA of each column block adds the partials in split order into `scores`.
cudaError_t launch_colnorm(const SelectArgs& a, cudaStream_t s);
// Radix-select the k largest final scores per head, emit I ascending.
cudaError_t launch_topk(const SelectArgs& a, cudaStream_t s);
// Scores and selection in one CTA per head (small inputs).
cudaError_t launch_normselect(const SelectArgs& a, cudaStream_t s);
// d <= 256 columns, n <= 8 rows: one warp per head ranks the columns.
bool select_small_fits(int64_t n, int64_t d);
cudaError_t launch_select_small(const SelectArgs& a, cudaStream_t s);
// n = 1 bf16 rows (d <= 65535, a multiple of 8): a two-digit radix select over
// the 15 magnitude bits on a cluster of CTAs per head, the same I as the fp32
// score path.
cudaError_t launch_select16(const SelectArgs& a, cudaStream_t s);
// I[h][j] = j for j < k (k == d: every index kept).
cudaError_t launch_identity(int32_t* I, int64_t k, int heads, cudaStream_t s);

constexpr int64_t kMaxSelectD = 49152;  // keys staged in shared memory (192 KiB)
size_t topk_smem_bytes(int64_t d);
size_t normselect_smem_bytes(int64_t d, int dtype);

// ---------------------------------------------------------------- pack
// dst[h][r][t] = src[h / group][r][I[h][t]] for t < k, 0 for k <= t < ld_dst.
struct PackArgs {
    const void* src;
    int dtype;
    int64_t rows, d, ld_src, stride_src;
    int group;
    const int32_t* I;
    int64_t I_stride, k;
    void* dst;
    int64_t ld_dst, stride_dst;
    int heads;
};
cudaError_t launch_pack(const PackArgs& a, cudaStream_t s);
// dst[h][r][j] = src[h][r][j] if j is in I[h][0..k) else 0 (dst has the
// source's shape; used for attention scores, where the product is bound by
// its output and a zero-masked operand gives the same sum over I).
cudaError_t launch_mask_columns(const PackArgs& a, cudaStream_t s);

// QK feature selection and the masked copy of Q in one launch (bf16,
// d <= 256 and a multiple of 8): a cluster of `cluster` CTAs per query head
// sums the squares of Q's features over its rows, the cluster's first CTA
// adds the CTAs' sums in rank order through distributed shared memory, takes
// the TopK (ties to the lower feature), writes I and hands the kept-feature
// words to the cluster; every CTA then writes its rows of Q with the unkept
// features zeroed.
// The whole op in one launch for tiny fp32 problems (LINEAR, one head,
// n <= kTinyMaxRows, d <= 256, a selected or given index set): scores, TopK
// and an fp32 FMA product.
constexpr int kTinyMaxRows = 64;
struct TinyArgs {
    const float* A;
    const float* B;
    float* Y;
    int32_t* I_out;          // [k] out, or nullptr
    const int32_t* I_given;  // [k] in (RMM_FLAG_USE_GIVEN_INDICES), or nullptr
    int n, d, m, k;
    int64_t lda, ldb, ldy;
    float alpha;
};
bool tiny_fits(const rmm_problem& p, int64_t k);  // k: the plan's index count
cudaError_t launch_tiny(const TinyArgs& a, cudaStream_t s);

struct QkMaskArgs {
    const void* Q;          // [heads][n][ldq] bf16
    int64_t n, d, ldq, stride_q;
    int heads;
    int64_t k;
    int32_t* I;             // [heads][k] out, ascending
    void* Qm;               // [heads][n][ldm] bf16 out
    int64_t ldm, stride_m;
    int cluster;            // CTAs per head: 1, 2, 4 or 8
};
bool qk_select_mask_fits(int dtype, int64_t d);
int qk_select_cluster(int64_t heads, int64_t n, int sms);
cudaError_t launch_qk_select_mask(const QkMaskArgs& a, cudaStream_t s);
// dst[h][c][t] = src[h / group][I[h][t]][c]: gathered rows written K-major
// (rows = number of source columns c; I == nullptr means I[t] = t).
cudaError_t launch_pack_rows_transposed(const PackArgs& a, cudaStream_t s);
// dst[h][t][:] = src[h / group][I[h][t]][:] for t < k: the retained rows of a
// row-major B, contiguous (a.rows = number of columns of B).
cudaError_t launch_pack_rows(const PackArgs& a, cudaStream_t s);
// launch_pack(a) and launch_pack_rows(b) as one launch: the A pack's CTAs, then
// the row copy's (bf16, packed A rows wider than the narrow variant's;
// pack_ab_one_launch says whether an A pack qualifies).
bool pack_ab_one_launch(int dtype, int64_t ld_a);
cudaError_t launch_pack_ab(const PackArgs& a, const PackArgs& b, cudaStream_t s);
// dst[h][t][:] = src[h / group][t][:] if t is in I[h][0..k) (ascending, unique)
// else 0, for t < rows_out (rows t >= a.d are zero); a.rows = columns of B.
// Used for attention PV, where the product is bound by reading P and a
// zero-masked V gives the same sum over I without a copy of P's columns.
// block_any (or nullptr): [heads][ceil(rows_out / 64)] bytes, 1 where the
// 64-row block holds a kept row.
cudaError_t launch_mask_rows(const PackArgs& a, int64_t rows_out, cudaStream_t s, uint8_t* block_any = nullptr);

// ---------------------------------------------------------------- GEMM
// How the B operand reaches shared memory (see rmm_gemm.cu).
constexpr int kBKMajor = 0;  // TMA tiles of an m x K row-major matrix (K-major)
constexpr int kBRows = 1;    // TMA tiles of consecutive rows of a d x m matrix (MN-major)
constexpr int kBGather = 2;  // tile::gather4 of indexed rows of a d x m matrix (MN-major)

// A operand: TMA tile loads from a 3-D map {K extent, rows, heads}, K-major.
struct __align__(64) GemmParams {
    CUtensorMap map_a;
    CUtensorMap map_b;          // kBKMajor: 3-D {K, m, heads}; kBRows/kBGather: 2-D {m, rows}
    CUtensorMap map_y;          // CTA-pair kernel: 3-D {m, n, heads} store map, box {32, 32, 1}
    const int32_t* I;           // kBGather: [heads][I_stride] row indices
    int64_t I_stride;
    void* Y;
    int64_t ldy, stride_y;
    int32_t n, m, k, d;
    int32_t heads, group;       // MN-major B head = h / group
    int32_t b_head_rows;        // MN-major B: row offset between consecutive B heads
    int32_t b_rows_total;       // MN-major B: rows of the 2-D map (an out-of-range row reads zeros)
    int32_t b_head_div;         // kBKMajor: B head coordinate = h / b_head_div
    int32_t m_tiles, n_tiles;
    int32_t group_m;            // CTA-pair kernel: 256-row tiles per rasterisation group
    float alpha;
    int32_t causal;             // QK: -inf above the diagonal of the output
    int32_t causal_k;           // A[i][j] = 0 for j > i (K axis = rows' positions): a row tile's
                                // K loop ends at its last row (CTA-pair kernel)
    int* err;
    // CTA-pair kernel, split tail: the last split_tiles tiles of the tile order
    // are computed as split_f K-parts each (0 = none).  Part j of split tile i
    // writes its fp32 accumulator to split_partials[(i * split_f + j)][256][BN];
    // split_counters[i][2][8] counts the parts each epilogue warp has finished
    // (zero between launches: the last part resets them).
    int32_t split_tiles, split_f;
    float* split_partials;
    unsigned* split_counters;
    // CTA-pair kernel, producer-fused scoring (no split tail): when emit_s2 is
    // set, every epilogue warp squares its 32 x 32 block of stored outputs and
    // sums each column over its 32 rows into emit_partials[h][row group][m]
    // (row group = 32-row slice of the output); emit_counters[h][column chunk]
    // counts the row groups done, and the warp that completes a chunk adds the
    // row groups in order into emit_s2[h][m] and resets the counter.
    float* emit_s2;
    float* emit_partials;
    unsigned* emit_counters;
    // CTA-pair kernel, K axis on a masked operand (attention PV with V's
    // unkept rows zeroed): kb_keep[h * kb_keep_stride + kb] == 0 says that
    // k-block kb of head h holds no kept index, so its products are zero and
    // the K loop skips it (the first k-block of a unit always runs, so that
    // every accumulator is written).
    const uint8_t* kb_keep;
    int32_t kb_keep_stride;
};

struct GemmLaunch {
    int dtype;
    int b_mode;       // kBKMajor / kBRows / kBGather
    int bn;           // 128 or 256 (the N of one tile)
    bool pair;        // CTA pairs (cta_group::2): 256-row tiles, m_tiles counts 256-row tiles,
                      // and a kBKMajor map_b box is bn/2 rows
    int num_sms;
};
cudaError_t launch_gemm(const GemmParams& p, const GemmLaunch& l, cudaStream_t s);
size_t gemm_smem_bytes(int dtype, int bn, bool pair);
// Split tail of the CTA-pair kernel for `tiles` 256-row tiles of `num_kb`
// k-blocks on `clusters` pairs: sets *split_tiles and *split_f (0 and 1 when
// the last wave is full or too short to split).
void pair_split_tail(int64_t tiles, int64_t num_kb, int clusters, int* split_tiles, int* split_f);
constexpr int kSplitCounterWarps = 8;  // counters per CTA per split tile (epilogue warps)


// ---------------------------------------------------------------- decode step
// Attention with group * n <= 8 query vectors per KV head (rmm_decode.cu).
struct DecodeArgs {
    const __nv_bfloat16* A;  // qk: Q [heads][n][d]; pv: P [heads][n][t]
    int64_t lda, stride_a;
    const __nv_bfloat16* B;  // qk: K [kv_heads][t][d]; pv: V [kv_heads][t][d_v]
    int64_t ldb, stride_b;
    const int32_t* I;        // qk: [heads][k] kept features, nullptr = all (or selected in the kernel)
    int32_t* I_out;          // qk with fused_select: where the selected I goes, or nullptr
    const uint32_t* mask;    // pv: [heads][mask_words] kept tokens (bit t of word t / 32), nullptr = all
    int64_t mask_words;
    __nv_bfloat16* Y;        // qk: S [heads][n][t]; pv: O [heads][n][d_v]
    int64_t ldy, stride_y;
    float* partials;         // pv: [kv_heads][token ranges][8][d_v] fp32
    unsigned* counters;      // pv: [kv_heads], zero between launches
    int64_t k;               // qk: entries of I per head
    int64_t d;               // qk: features d_h; pv: tokens t
    int64_t m;               // qk: keys t; pv: d_v
    int32_t n, group, kv_heads;
    int32_t tokens;          // pv: tokens per CTA (128, 256 or 512)
    int32_t sms;             // qk: SMs of the device (persistent grid)
    int32_t fused_select;    // qk: select each head's k features in the kernel (I unused)
    float alpha;             // qk: scale of the scores
};
bool decode_qk_supported(int64_t d);
bool decode_pv_supported(int64_t dv);
// tokens per CTA for t tokens on kv_heads heads: 512, halved while that
// leaves fewer than two CTAs per SM (down to 128)
int decode_pv_tokens(int64_t t, int64_t kv_heads, int num_sms);
cudaError_t launch_decode_qk(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_pv(const DecodeArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- few rows
// Product for n <= 64 with swapped operands (rmm_skinny.cu).
struct __align__(64) SkinnyParams {
    CUtensorMap map_a;      // A[:, I] (packed, or A itself when every index is kept):
                            // 3-D {K extent, n, 1}, box {64, np, 1}
    const void* B;          // row-major d x m bf16
    int64_t ldb;
    const int32_t* I;       // [k] retained rows of B, nullptr = every row in order
    void* Y;                // n x m bf16
    int64_t ldy;
    float* partials;        // [splits][np][m] fp32 when splits > 1
    float alpha;
    int32_t n, m, k, d, np, m_tiles, splits;
    int* err;
};
int skinny_pad(int64_t n);
int skinny_splits(int64_t m, int64_t k, int num_sms, int np);
cudaError_t launch_skinny(const SkinnyParams& p, cudaStream_t s);

}  // namespace rmm

// The plan behind the opaque rmm_plan handle of include/rmm.h.
#include "rmm.h"
struct rmm_plan {
    rmm_problem p;
    int64_t k;
    int64_t ldp;        // row stride of the packed operands (k rounded up to 8)
    int es;             // element size of A and B
    int es_out;         // element size of Y (2 for E4M3 operands: a bf16 output)
    int group;          // heads / kv_heads
    bool need_select;   // scores + TopK on each call
    bool fused_select;  // one-kernel selection
    bool select16;      // n = 1 bf16: the radix select over magnitude bits (a cluster per head)
    bool select_small;  // d <= 256, n <= 8: one warp per head ranks the columns
    int nsplit;
    int64_t rows_per_split;
    int bn;
    bool pack_b;        // bf16 LINEAR/PV with k < d: stage B[I, :] contiguously
    bool pack_ab;       // the A pack and the B row copy run as one launch
    int num_sms;
    size_t off_err, off_counters, off_partials, off_scores, off_I, off_apack, off_bpack, ws_bytes;
    size_t header_bytes;  // zeroed by rmm_workspace_init: error word + colnorm counters
    cudaEvent_t product_start, product_stop;  // tracing hook, may be null
    bool skinny;        // n <= 64 bf16 LINEAR: swapped-operand split-K product
    bool tiny;          // tiny fp32 LINEAR: the whole op in one launch (tiny_fits)
    int sk_np, sk_splits;
    bool pv_mask;       // bf16 PV with a selected T: V's unkept rows zeroed per query head, P read as stored
    int split_tiles, split_f;           // split tail of the CTA-pair product (0, 1: none)
    size_t off_split_cnt, off_split;    // its counters (in the header) and fp32 partials
    bool decode;        // bf16 attention with group * n <= 8 query vectors per KV head (rmm_decode.cu)
    bool decode_select; // decode QK: the features are selected inside the product kernel
    int qk_cluster;     // QK, bf16, d <= 256: selection and masked Q in one cluster launch (CTAs per head), else 0
    int dec_tokens, dec_parts;          // pv: tokens per CTA, token ranges per KV head
    size_t off_dec_cnt, off_dec_mask, off_dec_part;  // pv: counters (header), membership words, partials
    size_t off_kb_keep;                               // masked PV: per-head 64-token blocks holding a kept token
    bool given_scores;  // RMM_FLAG_GIVEN_SCORES: I = TopK of the caller's scores (no score pass)
    bool emit_scores;   // RMM_FLAG_EMIT_SCORES: column scores of Y (epilogue, or a score pass over Y)
    size_t off_emit_cnt, off_emit_part;               // epilogue form: counters (header), row-group sums
    int emit_nsplit;                                  // score-pass form over Y: its row splits,
    int64_t emit_rows_per_split;
    size_t off_emit_ycnt, off_emit_ypart;             // its counters (header) and partials
};
