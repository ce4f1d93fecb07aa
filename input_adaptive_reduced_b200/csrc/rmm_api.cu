// rmm_api.cu -- the C ABI of librmm (declared in include/rmm.h): problem
// validation, plans, workspace layout, tensor-map encoding and the launch
// sequence of Reduced Matrix Multiplication ("Reduced Matrix Multiplication:
// Input-Adaptive Matrix-Product Reduction for LLM Inference", §3.2-§3.3).
//
// Launch sequence of one call (all on the caller's stream, no host sync):
//   select : normselect (small inputs)  |  colnorm -> topk      -> I
//            identity fill when k == d (TopK of every index is all of them)
//   stage  : pack A[:, I] (and K[:, I] in QK mode) when k < d or I is given
//   product: gather_gemm (tcgen05, TMEM accumulators)
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_internal.h"



namespace {

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
constexpr size_t kFusedSelectBytes = size_t(128) << 10;  // per head: one CTA reads it all

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// k = ceil(rho d) with near-integer products snapped (see include/rmm.h).
int64_t retained_count(double rho, int64_t d) {
    const double x = rho * static_cast<double>(d);
    const double r = std::nearbyint(x);
    int64_t k = (std::fabs(x - r) <= 1e-9 * static_cast<double>(d)) ? static_cast<int64_t>(r)
                                                                      : static_cast<int64_t>(std::ceil(x));
    if (k < 1) k = 1;
    if (k > d) k = d;
    return k;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3-D K-major map {K extent, rows, heads} with a {box_k, box_rows, 1} box,
// 128-byte swizzle and zero fill outside the extents.
bool encode_kmajor_map(CUtensorMap* map, int es, const void* base, int64_t kext, int64_t rows,
                       int64_t heads, int64_t ld, int64_t stride_h, uint32_t box_k, uint32_t box_rows,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const uint64_t row_bytes = static_cast<uint64_t>(ld) * es;
    uint64_t head_bytes = static_cast<uint64_t>(stride_h) * es;
    if (heads <= 1 || head_bytes == 0) head_bytes = row_bytes * static_cast<uint64_t>(rows > 0 ? rows : 1);
    head_bytes = (head_bytes + 15) & ~uint64_t(15);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kext), static_cast<cuuint64_t>(rows > 0 ? rows : 1),
                          static_cast<cuuint64_t>(heads)};
    cuuint64_t strides[2] = {row_bytes, head_bytes};
    cuuint32_t box[3] = {box_k, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = es == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                             : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUresult r = enc(map, dt, 3,
                           const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D row-major map {m columns, rows} of an MN-major B operand with a
// {128 bytes of columns, box_rows} box, 128-byte swizzle, zero fill; es is the
// element size (2: bf16, 1: E4M3 codes).
bool encode_rows_map(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int64_t ld,
                     uint32_t box_rows, int es = 2) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * es};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / es), box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                           const_cast<void*>(base), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

rmm_status validate_problem(const rmm_problem* p) {
    if (!p) return RMM_ERR_INVALID_ARG;
    if (p->mode < RMM_LINEAR || p->mode > RMM_PV) return RMM_ERR_INVALID_ARG;
    if (p->dtype != RMM_BF16 && p->dtype != RMM_F32 && p->dtype != RMM_FP8_E4M3) return RMM_ERR_INVALID_ARG;
    const int es = p->dtype == RMM_F32 ? 4 : p->dtype == RMM_FP8_E4M3 ? 1 : 2;
    const int vec = 16 / es;                               // input elements per 16 bytes
    const int vec_y = p->dtype == RMM_FP8_E4M3 ? 8 : vec;  // output elements per 16 bytes (E4M3 -> bf16)
    if (p->n < 0 || p->m < 0 || p->d < 1) return RMM_ERR_INVALID_ARG;
    if (p->n > kMaxDim || p->m > kMaxDim || p->d > kMaxDim) return RMM_ERR_UNSUPPORTED;
    if (p->d % vec != 0 || p->m % vec != 0) return RMM_ERR_INVALID_ARG;
    if (p->heads < 1 || p->kv_heads < 1 || p->heads % p->kv_heads != 0) return RMM_ERR_INVALID_ARG;
    if (p->heads > 65535) return RMM_ERR_UNSUPPORTED;
    if (p->lda < p->d || p->lda % vec != 0) return RMM_ERR_INVALID_ARG;
    if (p->ldy < p->m || p->ldy % vec_y != 0) return RMM_ERR_INVALID_ARG;
    const int64_t b_cols = p->mode == RMM_QK ? p->d : p->m;
    if (p->ldb < b_cols || p->ldb % vec != 0) return RMM_ERR_INVALID_ARG;
    if (p->heads > 1) {
        if (p->stride_a < 0 || p->stride_a % vec != 0) return RMM_ERR_INVALID_ARG;
        if (p->stride_y % vec_y != 0 || (p->n > 0 && p->stride_y < p->n * p->ldy)) return RMM_ERR_INVALID_ARG;
    }
    if (p->kv_heads > 1 && (p->stride_b < 0 || p->stride_b % vec != 0)) return RMM_ERR_INVALID_ARG;
    // bf16 row gathers address every B head through one 2-D map: heads must sit
    // a whole number of rows apart.
    if (p->kv_heads > 1 && p->mode != RMM_QK && p->dtype == RMM_BF16 && p->stride_b % p->ldb != 0)
        return RMM_ERR_INVALID_ARG;
    if (p->kv_heads > 1 && p->mode != RMM_QK && p->dtype == RMM_BF16 &&
        ((p->kv_heads - 1) * (p->stride_b / p->ldb) + p->d) > kMaxDim - 1)
        return RMM_ERR_UNSUPPORTED;
    if (p->k == 0) {
        if (!(p->rho > 0.0) || p->rho > 1.0) return RMM_ERR_INVALID_ARG;
    } else if (p->k < 0 || p->k > p->d) {
        return RMM_ERR_INVALID_ARG;
    }
    if (p->flags & ~(RMM_FLAG_CAUSAL | RMM_FLAG_USE_GIVEN_INDICES | RMM_FLAG_GIVEN_SCORES | RMM_FLAG_EMIT_SCORES))
        return RMM_ERR_INVALID_ARG;
    if ((p->flags & RMM_FLAG_GIVEN_SCORES) && (p->flags & RMM_FLAG_USE_GIVEN_INDICES)) return RMM_ERR_INVALID_ARG;
    if ((p->flags & RMM_FLAG_EMIT_SCORES) && p->mode == RMM_QK) return RMM_ERR_INVALID_ARG;
    if ((p->flags & RMM_FLAG_CAUSAL) && !(p->mode == RMM_QK || (p->mode == RMM_PV && p->n == p->d)))
        return RMM_ERR_INVALID_ARG;
    if (!std::isfinite(p->alpha)) return RMM_ERR_INVALID_ARG;
    // The low-bit form runs on the CTA-pair product only: linear ops of more than 128 rows.
    if (p->dtype == RMM_FP8_E4M3 && (p->mode != RMM_LINEAR || p->heads != 1 || (p->n > 0 && p->n <= 128)))
        return RMM_ERR_UNSUPPORTED;
    return RMM_OK;
}

rmm_status check_workspace(const rmm_plan* plan, void* ws, size_t ws_bytes) {
    if (ws_bytes < plan->ws_bytes) return RMM_ERR_WORKSPACE;
    if (plan->ws_bytes > 0 && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)) return RMM_ERR_WORKSPACE;
    return RMM_OK;
}

template <typename T>
T* ws_at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

rmm_status run_select(const rmm_plan* plan, const void* A, int32_t* I, float* s2, void* ws,
                      cudaStream_t stream, const float* given = nullptr) {
    const rmm_problem& p = plan->p;
    rmm::SelectArgs a{};
    a.A = A;
    a.dtype = p.dtype;
    a.n = p.n;
    a.d = p.d;
    a.lda = p.lda;
    a.stride_a = p.stride_a;
    a.heads = static_cast<int>(p.heads);
    a.k = plan->k;
    a.I = I;
    a.s2 = s2;
    if (plan->decode && p.mode == RMM_PV) {  // the decode product reads membership words, not I
        a.mask = ws_at<uint32_t>(ws, plan->off_dec_mask);
        a.mask_words = (p.d + 31) / 32;
    }
    cudaError_t e;
    if (given) {
        // producer-fused scoring: the scores come from the op that produced A
        a.scores = const_cast<float*>(given);
        e = rmm::launch_topk(a, stream);
    } else if (plan->select_small) {
        e = rmm::launch_select_small(a, stream);
    } else if (plan->select16) {
        e = rmm::launch_select16(a, stream);
    } else if (plan->fused_select) {
        e = rmm::launch_normselect(a, stream);
    } else {
        a.partials = ws_at<float>(ws, plan->off_partials);
        a.counters = ws_at<unsigned>(ws, plan->off_counters);
        a.scores = s2 ? s2 : ws_at<float>(ws, plan->off_scores);
        a.nsplit = plan->nsplit;
        a.rows_per_split = plan->rows_per_split;
        // PV over a causal P: rows above a column block are zero there
        a.causal_rows = p.mode == RMM_PV && (p.flags & RMM_FLAG_CAUSAL) ? 1 : 0;
        e = rmm::launch_colnorm(a, stream);
        if (e == cudaSuccess) e = rmm::launch_topk(a, stream);
    }
    return e == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
}

rmm_status run_product(const rmm_plan* plan, const void* A, const void* B, void* Y, int32_t* I_inout,
                       float* s2_out, bool* scores_done, void* ws, size_t ws_bytes, void* stream_v,
                       const float* s2_in);

// Column scores of the output by a score pass over Y (shapes whose product has
// no epilogue form of the emission).
rmm_status emit_scores_pass(const rmm_plan* plan, const void* Y, float* s2_out, void* ws, cudaStream_t stream) {
    const rmm_problem& p = plan->p;
    rmm::SelectArgs a{};
    a.A = Y;
    a.dtype = p.dtype == RMM_FP8_E4M3 ? RMM_BF16 : p.dtype;  // the stored output's type
    a.n = p.n;
    a.d = p.m;
    a.lda = p.ldy;
    a.stride_a = p.stride_y;
    a.heads = static_cast<int>(p.heads);
    a.partials = ws_at<float>(ws, plan->off_emit_ypart);
    a.counters = ws_at<unsigned>(ws, plan->off_emit_ycnt);
    a.scores = s2_out;
    a.nsplit = plan->emit_nsplit;
    a.rows_per_split = plan->emit_rows_per_split;
    return rmm::launch_colnorm(a, stream) == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
}

rmm_status run_matmul(const rmm_plan* plan, const void* A, const void* B, void* Y, int32_t* I_inout,
                      const float* s2_in, float* s2_out, void* ws, size_t ws_bytes, void* stream_v) {
    if (!plan) return RMM_ERR_INVALID_ARG;
    const rmm_problem& p = plan->p;
    if (plan->given_scores && (!s2_in || (reinterpret_cast<uintptr_t>(s2_in) & 3u))) return RMM_ERR_INVALID_ARG;
    if (plan->emit_scores && (!s2_out || (reinterpret_cast<uintptr_t>(s2_out) & 3u))) return RMM_ERR_INVALID_ARG;
    bool scores_done = false;
    const rmm_status st = run_product(plan, A, B, Y, I_inout, plan->emit_scores ? s2_out : nullptr, &scores_done, ws,
                                      ws_bytes, stream_v, plan->given_scores ? s2_in : nullptr);
    if (st != RMM_OK || !plan->emit_scores || scores_done || p.m == 0) return st;
    if (p.n == 0) return cudaMemsetAsync(s2_out, 0, static_cast<size_t>(p.heads) * p.m * sizeof(float),
                                         static_cast<cudaStream_t>(stream_v)) == cudaSuccess
                             ? RMM_OK
                             : RMM_ERR_CUDA;
    return emit_scores_pass(plan, Y, s2_out, ws, static_cast<cudaStream_t>(stream_v));
}

rmm_status run_product(const rmm_plan* plan, const void* A, const void* B, void* Y, int32_t* I_inout,
                       float* s2_out, bool* scores_done, void* ws, size_t ws_bytes, void* stream_v,
                       const float* s2_in) {
    const rmm_problem& p = plan->p;
    const bool given = (p.flags & RMM_FLAG_USE_GIVEN_INDICES) != 0;
    const bool empty = p.n == 0 || p.m == 0;  // nothing to read or write but I
    if (!empty && (!A || !B || !Y)) return RMM_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(Y)) return RMM_ERR_INVALID_ARG;
    if (I_inout && (reinterpret_cast<uintptr_t>(I_inout) & 3u)) return RMM_ERR_INVALID_ARG;
    if (given && !I_inout) return RMM_ERR_INVALID_ARG;
    rmm_status st = check_workspace(plan, ws, ws_bytes);
    if (st != RMM_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    const int es = plan->es;
    const int64_t k = plan->k;

    if (plan->tiny) {  // scores, TopK and product in one launch
        rmm::TinyArgs ta{};
        ta.A = static_cast<const float*>(A);
        ta.B = static_cast<const float*>(B);
        ta.Y = static_cast<float*>(Y);
        ta.I_out = given ? nullptr : I_inout;
        ta.I_given = given ? I_inout : nullptr;
        ta.n = static_cast<int>(p.n);
        ta.d = static_cast<int>(p.d);
        ta.m = static_cast<int>(p.m);
        ta.k = static_cast<int>(k);
        ta.lda = p.lda;
        ta.ldb = p.ldb;
        ta.ldy = p.ldy;
        ta.alpha = p.alpha;
        const bool traced = plan->product_start && plan->product_stop;
        if (traced && cudaEventRecord(plan->product_start, stream) != cudaSuccess) return RMM_ERR_CUDA;
        if (rmm::launch_tiny(ta, stream) != cudaSuccess) return RMM_ERR_CUDA;
        if (traced && cudaEventRecord(plan->product_stop, stream) != cudaSuccess) return RMM_ERR_CUDA;
        return RMM_OK;
    }

    // ---- index set
    int32_t* I = I_inout ? I_inout : ws_at<int32_t>(ws, plan->off_I);
    const bool identity = !given && k == p.d;
    if (!given && !plan->decode_select) {
        if (identity) {
            if (I_inout && rmm::launch_identity(I_inout, k, static_cast<int>(p.heads), stream) != cudaSuccess)
                return RMM_ERR_CUDA;
        } else {
            // the decode PV product reads the membership words only: without
            // I_inout the one-row select writes no index list
            const bool words_only =
                plan->decode && p.mode == RMM_PV && plan->select16 && !plan->select_small && !I_inout && !s2_in;
            if (!plan->qk_cluster) {  // (else selected together with the masked copy of Q, below)
                st = run_select(plan, A, words_only ? nullptr : I, nullptr, ws, stream, s2_in);
                if (st != RMM_OK) return st;
            }
        }
    }
    if (p.n == 0 || p.m == 0) return RMM_OK;

    if (plan->decode) {
        rmm::DecodeArgs da{};
        da.A = static_cast<const __nv_bfloat16*>(A);
        da.lda = p.lda;
        da.stride_a = p.stride_a;
        da.B = static_cast<const __nv_bfloat16*>(B);
        da.ldb = p.ldb;
        da.stride_b = p.stride_b;
        da.Y = static_cast<__nv_bfloat16*>(Y);
        da.ldy = p.ldy;
        da.stride_y = p.stride_y;
        da.k = k;
        da.d = p.d;
        da.m = p.m;
        da.n = static_cast<int32_t>(p.n);
        da.group = plan->group;
        da.kv_heads = static_cast<int32_t>(p.kv_heads);
        da.sms = plan->num_sms;
        da.alpha = p.alpha;
        const bool traced = plan->product_start && plan->product_stop;
        if (traced && cudaEventRecord(plan->product_start, stream) != cudaSuccess) return RMM_ERR_CUDA;
        cudaError_t e;
        if (p.mode == RMM_QK) {
            da.I = identity || plan->decode_select ? nullptr : I;
            da.fused_select = plan->decode_select ? 1 : 0;
            da.I_out = plan->decode_select ? I_inout : nullptr;
            e = rmm::launch_decode_qk(da, stream);
        } else {
            da.mask = identity ? nullptr : ws_at<uint32_t>(ws, plan->off_dec_mask);
            da.mask_words = (p.d + 31) / 32;
            da.partials = ws_at<float>(ws, plan->off_dec_part);
            da.counters = ws_at<unsigned>(ws, plan->off_dec_cnt);
            da.tokens = plan->dec_tokens;
            e = rmm::launch_decode_pv(da, stream);
        }
        if (e != cudaSuccess) return RMM_ERR_CUDA;
        if (traced && cudaEventRecord(plan->product_stop, stream) != cudaSuccess) return RMM_ERR_CUDA;
        return RMM_OK;
    }

    if (plan->skinny) {
        rmm::SkinnyParams sp;
        std::memset(&sp, 0, sizeof(sp));
        const uint32_t box_np = static_cast<uint32_t>(plan->sk_np);
        if (!identity) {
            rmm::PackArgs pa{};
            pa.src = A;
            pa.dtype = p.dtype;
            pa.rows = p.n;
            pa.d = p.d;
            pa.ld_src = p.lda;
            pa.stride_src = p.stride_a;
            pa.group = 1;
            pa.I = I;
            pa.I_stride = k;
            pa.k = k;
            pa.dst = ws_at<void>(ws, plan->off_apack);
            pa.ld_dst = plan->ldp;
            pa.stride_dst = p.n * plan->ldp;
            pa.heads = 1;
            if (rmm::launch_pack(pa, stream) != cudaSuccess) return RMM_ERR_CUDA;
            if (!encode_kmajor_map(&sp.map_a, 2, pa.dst, k, p.n, 1, plan->ldp, p.n * plan->ldp, 64, box_np))
                return RMM_ERR_CUDA;
        } else if (!encode_kmajor_map(&sp.map_a, 2, A, p.d, p.n, 1, p.lda, p.n * p.lda, 64, box_np)) {
            return RMM_ERR_CUDA;
        }
        sp.B = B;
        sp.ldb = p.ldb;
        sp.I = identity ? nullptr : I;
        sp.Y = Y;
        sp.ldy = p.ldy;
        sp.partials = ws_at<float>(ws, plan->off_bpack);
        sp.alpha = p.alpha;
        sp.n = static_cast<int32_t>(p.n);
        sp.m = static_cast<int32_t>(p.m);
        sp.k = static_cast<int32_t>(k);
        sp.d = static_cast<int32_t>(p.d);
        sp.np = plan->sk_np;
        sp.m_tiles = static_cast<int32_t>((p.m + 127) / 128);
        sp.splits = plan->sk_splits;
        sp.err = ws_at<int>(ws, plan->off_err);
        const bool traced = plan->product_start && plan->product_stop;
        if (traced && cudaEventRecord(plan->product_start, stream) != cudaSuccess) return RMM_ERR_CUDA;
        if (rmm::launch_skinny(sp, stream) != cudaSuccess) return RMM_ERR_CUDA;
        if (traced && cudaEventRecord(plan->product_stop, stream) != cudaSuccess) return RMM_ERR_CUDA;
        return RMM_OK;
    }

    // ---- stage the gathered A columns (and K columns in QK mode)
    rmm::GemmParams gp;
    std::memset(&gp, 0, sizeof(gp));
    const uint32_t box_k = static_cast<uint32_t>(128 / es);
    const bool qk_masked_path = p.mode == RMM_QK && !identity && p.d <= 1024;
    rmm::PackArgs pa_deferred{};
    if (qk_masked_path) {
        // staged below together with B
    } else if (!identity && !plan->pv_mask) {
        rmm::PackArgs pa{};
        pa.src = A;
        pa.dtype = p.dtype;
        pa.rows = p.n;
        pa.d = p.d;
        pa.ld_src = p.lda;
        pa.stride_src = p.stride_a;
        pa.group = 1;
        pa.I = I;
        pa.I_stride = k;
        pa.k = k;
        pa.dst = ws_at<void>(ws, plan->off_apack);
        pa.ld_dst = plan->ldp;
        pa.stride_dst = p.n * plan->ldp;
        pa.heads = static_cast<int>(p.heads);
        if (plan->pack_ab)
            pa_deferred = pa;  // launched together with the B row copy below
        else if (rmm::launch_pack(pa, stream) != cudaSuccess)
            return RMM_ERR_CUDA;
        if (!encode_kmajor_map(&gp.map_a, es, pa.dst, k, p.n, p.heads, plan->ldp, p.n * plan->ldp, box_k, 128))
            return RMM_ERR_CUDA;
    } else {
        if (!encode_kmajor_map(&gp.map_a, es, A, p.d, p.n, p.heads, p.lda, p.stride_a, box_k, 128))
            return RMM_ERR_CUDA;
    }

    rmm::GemmLaunch gl;
    // CTA pairs (256-row tiles) whenever there is more than one 128-row tile of
    // work; indexed gather4 feeding stays single-CTA.
    const bool pair_ok = p.n > 128;
    const uint32_t kmajor_box_rows = static_cast<uint32_t>(pair_ok ? plan->bn / 2 : plan->bn);
    gl.dtype = p.dtype;
    gl.bn = plan->bn;
    gl.num_sms = plan->num_sms;
    gp.Y = Y;
    gp.ldy = p.ldy;
    gp.stride_y = p.stride_y;
    gp.n = static_cast<int32_t>(p.n);
    gp.m = static_cast<int32_t>(p.m);
    gp.k = static_cast<int32_t>(k);
    gp.d = static_cast<int32_t>(p.d);
    gp.heads = static_cast<int32_t>(p.heads);
    gp.group = plan->group;

    gp.n_tiles = static_cast<int32_t>((p.m + plan->bn - 1) / plan->bn);
    gp.alpha = p.alpha;
    gp.causal = p.mode == RMM_QK && (p.flags & RMM_FLAG_CAUSAL) ? 1 : 0;
    // PV over a causal P with the product's K axis on the tokens (every token
    // kept, or V's unkept rows zeroed): a row tile stops at its last row
    gp.causal_k = p.mode == RMM_PV && (p.flags & RMM_FLAG_CAUSAL) && (identity || plan->pv_mask) ? 1 : 0;
    gp.err = ws_at<int>(ws, plan->off_err);
    gp.b_head_div = 1;

    const bool qk_mask = p.mode == RMM_QK && !identity && p.d <= 1024;
    if (qk_mask) {
        // Attention scores are bound by writing S, not by the contraction: zero
        // Q's features outside I_h and contract over all d_h with the shared K
        // as it is (the zeroed terms add exact zeros, so the sum is the one
        // over I_h) instead of packing Q and, per query head, K.
        rmm::PackArgs pm{};
        pm.src = A;
        pm.dtype = p.dtype;
        pm.rows = p.n;
        pm.d = p.d;
        pm.ld_src = p.lda;
        pm.stride_src = p.stride_a;
        pm.group = 1;
        pm.I = I;
        pm.I_stride = k;
        pm.k = k;
        pm.dst = ws_at<void>(ws, plan->off_apack);
        pm.ld_dst = p.d;
        pm.stride_dst = p.n * p.d;
        pm.heads = static_cast<int>(p.heads);
        if (plan->qk_cluster) {
            rmm::QkMaskArgs qa{};
            qa.Q = A;
            qa.n = p.n;
            qa.d = p.d;
            qa.ldq = p.lda;
            qa.stride_q = p.stride_a;
            qa.heads = static_cast<int>(p.heads);
            qa.k = k;
            qa.I = I;
            qa.Qm = pm.dst;
            qa.ldm = pm.ld_dst;
            qa.stride_m = pm.stride_dst;
            qa.cluster = plan->qk_cluster;
            if (rmm::launch_qk_select_mask(qa, stream) != cudaSuccess) return RMM_ERR_CUDA;
        } else if (rmm::launch_mask_columns(pm, stream) != cudaSuccess) {
            return RMM_ERR_CUDA;
        }
        if (!encode_kmajor_map(&gp.map_a, es, pm.dst, p.d, p.n, p.heads, p.d, p.n * p.d, box_k, 128))
            return RMM_ERR_CUDA;
        gp.k = static_cast<int32_t>(p.d);
        gl.b_mode = rmm::kBKMajor;
        if (!encode_kmajor_map(&gp.map_b, es, B, p.d, p.m, p.kv_heads, p.ldb, p.stride_b, box_k, kmajor_box_rows))
            return RMM_ERR_CUDA;
        gp.b_head_div = plan->group;
    } else if (p.mode == RMM_QK) {
        gl.b_mode = rmm::kBKMajor;
        if (!identity) {
            rmm::PackArgs pb{};
            pb.src = B;
            pb.dtype = p.dtype;
            pb.rows = p.m;
            pb.d = p.d;
            pb.ld_src = p.ldb;
            pb.stride_src = p.stride_b;
            pb.group = plan->group;
            pb.I = I;
            pb.I_stride = k;
            pb.k = k;
            pb.dst = ws_at<void>(ws, plan->off_bpack);
            pb.ld_dst = plan->ldp;
            pb.stride_dst = p.m * plan->ldp;
            pb.heads = static_cast<int>(p.heads);
            if (rmm::launch_pack(pb, stream) != cudaSuccess) return RMM_ERR_CUDA;
            if (!encode_kmajor_map(&gp.map_b, es, pb.dst, k, p.m, p.heads, plan->ldp, p.m * plan->ldp, box_k,
                                   kmajor_box_rows))
                return RMM_ERR_CUDA;
        } else {
            if (!encode_kmajor_map(&gp.map_b, es, B, p.d, p.m, p.kv_heads, p.ldb, p.stride_b, box_k,
                                   kmajor_box_rows))
                return RMM_ERR_CUDA;
            gp.b_head_div = plan->group;
        }
    } else if (p.dtype == RMM_F32) {
        // tf32 operands are staged K-major: B[I, :] is written transposed (m x k).
        gl.b_mode = rmm::kBKMajor;
        rmm::PackArgs pb{};
        pb.src = B;
        pb.dtype = p.dtype;
        pb.rows = p.m;
        pb.d = p.d;
        pb.ld_src = p.ldb;
        pb.stride_src = p.stride_b;
        pb.group = plan->group;
        pb.I = identity ? nullptr : I;
        pb.I_stride = k;
        pb.k = k;
        pb.dst = ws_at<void>(ws, plan->off_bpack);
        pb.ld_dst = plan->ldp;
        pb.stride_dst = p.m * plan->ldp;
        pb.heads = static_cast<int>(p.heads);
        if (rmm::launch_pack_rows_transposed(pb, stream) != cudaSuccess) return RMM_ERR_CUDA;
        if (!encode_kmajor_map(&gp.map_b, es, pb.dst, k, p.m, p.heads, plan->ldp, p.m * plan->ldp, box_k,
                               kmajor_box_rows))
            return RMM_ERR_CUDA;
    } else if (plan->pv_mask) {
        // V's rows outside each query head's T are zeroed in a per-head copy
        // padded to whole K blocks; the product contracts over every token of P.
        const int64_t d_pad = (p.d + 63) / 64 * 64;
        rmm::PackArgs pb{};
        pb.src = B;
        pb.dtype = p.dtype;
        pb.rows = p.m;
        pb.d = p.d;
        pb.ld_src = p.ldb;
        pb.stride_src = p.stride_b;
        pb.group = plan->group;
        pb.I = I;
        pb.I_stride = k;
        pb.k = k;
        pb.dst = ws_at<void>(ws, plan->off_bpack);
        pb.ld_dst = p.m;
        pb.stride_dst = d_pad * p.m;
        pb.heads = static_cast<int>(p.heads);
        uint8_t* kb_keep = ws_at<uint8_t>(ws, plan->off_kb_keep);
        if (rmm::launch_mask_rows(pb, d_pad, stream, kb_keep) != cudaSuccess) return RMM_ERR_CUDA;
        // 64-token blocks without a kept token contribute zeros: the product skips them
        gp.kb_keep = kb_keep;
        gp.kb_keep_stride = static_cast<int32_t>(d_pad / 64);
        gl.b_mode = rmm::kBRows;
        gp.k = static_cast<int32_t>(p.d);
        gp.group = 1;
        gp.b_head_rows = static_cast<int32_t>(d_pad);
        gp.b_rows_total = static_cast<int32_t>(d_pad * p.heads);
        if (!encode_rows_map(&gp.map_b, pb.dst, p.m, d_pad * p.heads, p.m, 64u)) return RMM_ERR_CUDA;
    } else if (!identity && plan->pack_b) {
        // The retained rows B[I, :] are copied into a contiguous k x m buffer per
        // head (a streaming copy at HBM rate), which the product then reads with
        // plain TMA row tiles.
        rmm::PackArgs pb{};
        pb.src = B;
        pb.dtype = p.dtype;
        pb.rows = p.m;
        pb.d = p.d;
        pb.ld_src = p.ldb;
        pb.stride_src = p.stride_b;
        pb.group = plan->group;
        pb.I = I;
        pb.I_stride = k;
        pb.k = k;
        pb.dst = ws_at<void>(ws, plan->off_bpack);
        pb.ld_dst = p.m;
        pb.stride_dst = k * p.m;
        pb.heads = static_cast<int>(p.heads);
        const cudaError_t e = plan->pack_ab ? rmm::launch_pack_ab(pa_deferred, pb, stream)
                                            : rmm::launch_pack_rows(pb, stream);
        if (e != cudaSuccess) return RMM_ERR_CUDA;
        gl.b_mode = rmm::kBRows;
        gp.group = 1;
        gp.b_head_rows = static_cast<int32_t>(k);
        gp.b_rows_total = static_cast<int32_t>(k * p.heads);
        if (!encode_rows_map(&gp.map_b, pb.dst, p.m, k * p.heads, p.m, static_cast<uint32_t>(box_k), es))
            return RMM_ERR_CUDA;
    } else {
        // Plain row tiles only where rows past d are out of the map (one B head)
        // or never reached (d a whole number of K blocks); otherwise rows are
        // fetched four at a time through the index set with tile::gather4.
        const bool row_tiles = identity && (p.kv_heads == 1 || p.d % box_k == 0);
        gl.b_mode = row_tiles ? rmm::kBRows : rmm::kBGather;
        const int64_t head_rows = p.kv_heads > 1 ? p.stride_b / p.ldb : p.d;
        const int64_t rows_total = (p.kv_heads - 1) * head_rows + p.d;
        gp.b_head_rows = static_cast<int32_t>(head_rows);
        gp.b_rows_total = static_cast<int32_t>(rows_total);
        gp.I = identity ? nullptr : I;
        gp.I_stride = k;
        if (!encode_rows_map(&gp.map_b, B, p.m, rows_total, p.ldb, row_tiles ? static_cast<uint32_t>(box_k) : 1u, es))
            return RMM_ERR_CUDA;
    }
    gl.pair = pair_ok && gl.b_mode != rmm::kBGather;
    if (gl.pair && s2_out) {
        gp.emit_s2 = s2_out;
        gp.emit_partials = ws_at<float>(ws, plan->off_emit_part);
        gp.emit_counters = ws_at<unsigned>(ws, plan->off_emit_cnt);
        *scores_done = true;
    }
    gp.split_tiles = gl.pair ? plan->split_tiles : 0;
    gp.split_f = gl.pair ? plan->split_f : 1;
    gp.split_partials = ws_at<float>(ws, plan->off_split);
    gp.split_counters = ws_at<unsigned>(ws, plan->off_split_cnt);
    gp.m_tiles = static_cast<int32_t>(gl.pair ? (p.n + 255) / 256 : (p.n + 127) / 128);
    // rasterisation groups of 8 row tiles (measured best on the workloads' shapes)
    gp.group_m = gp.m_tiles < 8 ? gp.m_tiles : 8;
    // the pair kernel stores 32 x 32 output boxes by TMA (64- or 128-byte rows)
    if (gl.pair && !encode_kmajor_map(&gp.map_y, plan->es_out, Y, p.m, p.n, p.heads, p.ldy, p.stride_y, 32, 32,
                                      plan->es_out == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B))
        return RMM_ERR_CUDA;
    const bool traced = plan->product_start && plan->product_stop;
    if (traced && cudaEventRecord(plan->product_start, stream) != cudaSuccess) return RMM_ERR_CUDA;
    if (rmm::launch_gemm(gp, gl, stream) != cudaSuccess) return RMM_ERR_CUDA;
    if (traced && cudaEventRecord(plan->product_stop, stream) != cudaSuccess) return RMM_ERR_CUDA;
    return RMM_OK;
}

// Whether the product runs on the CTA-pair kernel (run_product's choice),
// where emitted column scores come from the epilogue.
bool product_on_pairs(const rmm_plan* plan) {
    const rmm_problem& p = plan->p;
    if (plan->decode || plan->skinny || p.n <= 128) return false;
    const bool given = (p.flags & RMM_FLAG_USE_GIVEN_INDICES) != 0;
    const bool identity = !given && plan->k == p.d;
    const bool gather = p.mode != RMM_QK && p.dtype == RMM_BF16 && identity && p.kv_heads > 1 && p.d % 64 != 0;
    return !gather;
}

int32_t launches_per_call(const rmm_plan* plan) {
    const rmm_problem& p = plan->p;
    const bool given = (p.flags & RMM_FLAG_USE_GIVEN_INDICES) != 0;
    const bool identity = !given && plan->k == p.d;
    int32_t n = 0;
    if (plan->tiny) return 1;  // scores, TopK and product in one launch
    if (!given && !identity && !plan->decode_select && !plan->qk_cluster)  // (QK: with the masked Q below)
        n += (plan->given_scores || plan->fused_select || plan->select16 || plan->select_small) ? 1 : 2;
    if (plan->emit_scores && p.m > 0 && p.n > 0 && !product_on_pairs(plan)) n += 1;  // score pass over Y
    if (p.n == 0 || p.m == 0) return n;
    if (plan->decode) return n + 1;
    if (plan->skinny) return n + (identity ? 0 : 1) + 1 + (plan->sk_splits > 1 ? 1 : 0);
    if (!identity) n += 1;                                   // pack A[:, I] (PV: mask V's rows instead)
    if (p.mode == RMM_QK && !identity && p.d > 1024) n += 1; // pack K[:, I] (else Q is masked in place of the A pack)
    if (p.mode != RMM_QK && p.dtype == RMM_F32) n += 1;      // B[I, :] transposed for tf32
    if (!identity && plan->pack_b && !plan->pack_ab) n += 1; // B[I, :] rows, contiguous (else in the A pack's launch)
    return n + 1;                                            // the product
}

}  // namespace

extern "C" {

void rmm_problem_init(rmm_problem* p, int32_t mode, int32_t dtype, int64_t n, int64_t d, int64_t m) {
    if (!p) return;
    std::memset(p, 0, sizeof(*p));
    p->mode = mode;
    p->dtype = dtype;
    p->n = n;
    p->d = d;
    p->m = m;
    p->lda = d;
    p->ldb = mode == RMM_QK ? d : m;
    p->ldy = m;
    p->heads = 1;
    p->kv_heads = 1;
    p->rho = 1.0;
    p->alpha = 1.0f;
}

rmm_status rmm_plan_create(rmm_plan** out, const rmm_problem* p, size_t* workspace_bytes) {
    if (!out) return RMM_ERR_INVALID_ARG;
    *out = nullptr;
    rmm_status st = validate_problem(p);
    if (st != RMM_OK) return st;
    rmm_plan* plan = new (std::nothrow) rmm_plan;
    if (!plan) return RMM_ERR_UNSUPPORTED;
    std::memset(plan, 0, sizeof(*plan));
    plan->p = *p;
    plan->es = p->dtype == RMM_F32 ? 4 : p->dtype == RMM_FP8_E4M3 ? 1 : 2;
    plan->es_out = p->dtype == RMM_FP8_E4M3 ? 2 : plan->es;
    plan->k = p->k > 0 ? p->k : retained_count(p->rho, p->d);
    // packed rows: whole groups of 8 elements (the packs write 8 at a time) and whole 16-byte granules
    const int64_t pack_group = plan->es == 1 ? 16 : 8;
    plan->ldp = (plan->k + pack_group - 1) / pack_group * pack_group;
    plan->group = static_cast<int>(p->heads / p->kv_heads);
    const bool given = (p->flags & RMM_FLAG_USE_GIVEN_INDICES) != 0;
    plan->need_select = !given && plan->k < p->d;
    plan->bn = p->m <= 128 ? 128 : 256;
    plan->pack_b = p->mode != RMM_QK && (p->dtype == RMM_BF16 || p->dtype == RMM_FP8_E4M3) && (plan->k < p->d || given);
    // PV over short value heads is bound by reading P: instead of copying P's
    // retained columns, zero V's unkept rows (per query head) and read P as is.
    plan->pv_mask = p->mode == RMM_PV && p->dtype == RMM_BF16 && !given && plan->k < p->d && p->m <= 256;
    if (plan->pv_mask) plan->pack_b = false;
    // Few rows: the op is a stream of B[I, :]; gather it inside a split-K
    // product with swapped operands instead of staging it.
    plan->skinny = p->mode == RMM_LINEAR && p->dtype == RMM_BF16 && p->heads == 1 && p->n >= 1 && p->n <= 64 &&
                   p->m >= 1;
    plan->tiny = rmm::tiny_fits(*p, plan->k);
    if (plan->tiny) plan->pack_b = false;
    if (plan->skinny) {
        plan->pack_b = false;
        plan->sk_np = rmm::skinny_pad(p->n);
        plan->sk_splits = rmm::skinny_splits(p->m, plan->k, 0, plan->sk_np);  // fixed below once the SM count is known
    }
    // Decode step: a few query rows per head against cached keys / values;
    // the group's query vectors are taken together (each cache row is read
    // once per KV head).  PV needs the selection's membership words, so a
    // given token set takes the general path.
    const bool causal = (p->flags & RMM_FLAG_CAUSAL) != 0;
    plan->decode = p->dtype == RMM_BF16 && !causal && p->n >= 1 && p->n * plan->group <= 8 &&
                   ((p->mode == RMM_QK && rmm::decode_qk_supported(p->d)) ||
                    (p->mode == RMM_PV && !given && rmm::decode_pv_supported(p->m)));
    if (plan->decode) {
        plan->pack_b = false;
        plan->pv_mask = false;
    }
    plan->given_scores = (p->flags & RMM_FLAG_GIVEN_SCORES) != 0;
    plan->emit_scores = (p->flags & RMM_FLAG_EMIT_SCORES) != 0;
    plan->decode_select = plan->decode && p->mode == RMM_QK && plan->need_select && !plan->given_scores;
    plan->pack_ab = plan->pack_b && rmm::pack_ab_one_launch(p->dtype, plan->ldp);

    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        cudaGetLastError();
        delete plan;
        return RMM_ERR_CUDA;
    }
    plan->num_sms = sms;
    if (plan->skinny) plan->sk_splits = rmm::skinny_splits(p->m, plan->k, sms, plan->sk_np);
    const bool dec_pv = plan->decode && p->mode == RMM_PV;
    if (dec_pv) {
        plan->dec_tokens = rmm::decode_pv_tokens(p->d, p->kv_heads, sms);
        plan->dec_parts = static_cast<int>((p->d + plan->dec_tokens - 1) / plan->dec_tokens);
    }

    // Selection kernels need every score of a head in shared memory.
    const bool select_possible = p->d <= rmm::kMaxSelectD;
    if (plan->need_select && !select_possible) {
        delete plan;
        return RMM_ERR_UNSUPPORTED;
    }
    const size_t head_bytes = static_cast<size_t>(p->n) * p->d * plan->es;
    plan->fused_select = p->dtype != RMM_FP8_E4M3 && head_bytes <= kFusedSelectBytes &&
                         rmm::normselect_smem_bytes(p->d, p->dtype) <= 180 * 1024;
    // one bf16 row per head: a radix select over the magnitude bits
    plan->select16 = p->n == 1 && p->dtype == RMM_BF16 && p->d % 8 == 0 && p->d <= 65535;
    plan->select_small = rmm::select_small_fits(p->n, p->d);
    // QK with a selected I: the scores, the TopK and the masked copy of Q in one launch
    plan->qk_cluster = p->mode == RMM_QK && plan->need_select && !plan->given_scores && !plan->decode &&
                               p->n >= 1 && p->m >= 1 && rmm::qk_select_mask_fits(p->dtype, p->d)
                           ? rmm::qk_select_cluster(p->heads, p->n, sms)
                           : 0;
    // Row splits for the score pass: as many CTAs as fit on the SMs at once
    // (two per SM; one CTA more than that would run as a second wave of its
    // own), at most 16 partials per column, at least 64 rows each.
    const int vec = 16 / plan->es;
    const int64_t colblocks = (p->d + 32 * vec - 1) / (32 * vec);
    const int64_t target = 2LL * sms;
    int64_t nsplit = target / (colblocks * p->heads);
    if (nsplit < 1) nsplit = 1;
    const int64_t max_split = (p->n + 63) / 64;
    if (nsplit > max_split) nsplit = max_split;
    // a causal P: splits of 512 rows, those above a column block end at once
    if (p->mode == RMM_PV && (p->flags & RMM_FLAG_CAUSAL) && max_split > 1) {
        const int64_t causal_split = (p->n + 511) / 512;
        if (causal_split > nsplit) nsplit = causal_split;
    }
    if (nsplit > 16) nsplit = 16;
    if (nsplit < 1) nsplit = 1;
    int64_t rps = (p->n + nsplit - 1) / nsplit;
    rps = (rps + 7) / 8 * 8;
    if (rps < 8) rps = 8;
    nsplit = p->n > 0 ? (p->n + rps - 1) / rps : 1;
    plan->nsplit = static_cast<int>(nsplit);
    plan->rows_per_split = rps;

    size_t off = 0;
    plan->off_err = off;
    off += 256;
    plan->off_counters = off;
    off += align256(static_cast<size_t>(p->heads) * colblocks * sizeof(unsigned));
    // Split tail of the CTA-pair product (256-row tiles, more than one 128-row
    // tile of work, no causal mask): its counters live in the header.
    plan->split_tiles = 0;
    plan->split_f = 1;
    if (!plan->skinny && p->n > 128 && p->m > 0 && !(p->flags & RMM_FLAG_CAUSAL) && !plan->emit_scores) {
        const int64_t k_eff = ((p->mode == RMM_QK && p->d <= 1024) || plan->pv_mask) ? p->d : plan->k;
        const int64_t bk = 128 / plan->es;
        const int64_t tiles = p->heads * ((p->n + 255) / 256) * ((p->m + plan->bn - 1) / plan->bn);
        rmm::pair_split_tail(tiles, (k_eff + bk - 1) / bk, sms / 2, &plan->split_tiles, &plan->split_f);
    }
    plan->off_split_cnt = off;
    off += align256(static_cast<size_t>(plan->split_tiles) * 2 * rmm::kSplitCounterWarps * sizeof(unsigned));
    plan->off_dec_cnt = off;
    if (dec_pv) off += align256(static_cast<size_t>(p->kv_heads) * sizeof(unsigned));
    // Producer-fused scoring of the output: counters of the epilogue form
    // (per 32-column chunk) and of the score pass over Y (per column block).
    const int vec_y = 16 / plan->es_out;
    const int64_t y_colblocks = (p->m + 32 * vec_y - 1) / (32 * vec_y);
    plan->off_emit_cnt = off;
    plan->off_emit_ycnt = off;
    if (plan->emit_scores) {
        off += align256(static_cast<size_t>(p->heads) * ((p->m + 255) / 256) * 8 * sizeof(unsigned));
        plan->off_emit_ycnt = off;
        off += align256(static_cast<size_t>(p->heads) * y_colblocks * sizeof(unsigned));
    }
    plan->header_bytes = off;
    plan->off_partials = off;
    plan->off_scores = off;
    if (select_possible && !plan->fused_select && !plan->select16 && !plan->select_small) {
        off += align256(static_cast<size_t>(p->heads) * nsplit * p->d * sizeof(float));
        plan->off_scores = off;
        off += align256(static_cast<size_t>(p->heads) * p->d * sizeof(float));
    }
    plan->off_I = off;
    off += align256(static_cast<size_t>(p->heads) * plan->k * sizeof(int32_t));
    plan->off_apack = off;
    const bool qk_mask = p->mode == RMM_QK && p->d <= 1024;  // Q masked at full width, K used as is
    if (!plan->pv_mask && !plan->decode)
        off += align256(static_cast<size_t>(p->heads) * p->n * (qk_mask ? p->d : plan->ldp) * plan->es);
    plan->off_bpack = off;
    if (qk_mask) {
        // no staged B
    } else if (plan->skinny)
        off += align256(static_cast<size_t>(plan->sk_splits) * p->m * plan->sk_np * sizeof(float));
    else if (p->mode == RMM_QK || p->dtype == RMM_F32)
        off += align256(static_cast<size_t>(p->heads) * p->m * plan->ldp * plan->es);
    else if (plan->pv_mask)
        off += align256(static_cast<size_t>(p->heads) * ((p->d + 63) / 64 * 64) * p->m * plan->es);
    else if (plan->pack_b || given)
        off += align256(static_cast<size_t>(p->heads) * plan->k * p->m * plan->es);
    plan->off_split = off;
    off += align256(static_cast<size_t>(plan->split_tiles) * plan->split_f * 256 * plan->bn * sizeof(float));
    plan->off_kb_keep = off;
    if (plan->pv_mask) off += align256(static_cast<size_t>(p->heads) * ((p->d + 63) / 64));
    plan->off_dec_mask = off;
    plan->off_dec_part = off;
    if (dec_pv) {
        off += align256(static_cast<size_t>(p->heads) * ((p->d + 31) / 32) * sizeof(uint32_t));
        plan->off_dec_part = off;
        off += align256(static_cast<size_t>(p->kv_heads) * plan->dec_parts * 8 * p->m * sizeof(float));
    }
    plan->off_emit_part = off;
    plan->off_emit_ypart = off;
    if (plan->emit_scores) {
        // epilogue form: row groups of 32 rows x m per head
        off += align256(static_cast<size_t>(p->heads) * 8 * ((p->n + 255) / 256) * p->m * sizeof(float));
        // score-pass form: row splits as for a score pass over A (one wave)
        int64_t ens = (2LL * sms) / (y_colblocks * p->heads);
        const int64_t emax = (p->n + 63) / 64;
        if (ens > emax) ens = emax;
        if (ens > 16) ens = 16;
        if (ens < 1) ens = 1;
        int64_t erps = (p->n + ens - 1) / ens;
        erps = (erps + 7) / 8 * 8;
        if (erps < 8) erps = 8;
        ens = p->n > 0 ? (p->n + erps - 1) / erps : 1;
        plan->emit_nsplit = static_cast<int>(ens);
        plan->emit_rows_per_split = erps;
        plan->off_emit_ypart = off;
        off += align256(static_cast<size_t>(p->heads) * ens * p->m * sizeof(float));
    }
    plan->ws_bytes = off;
    if (workspace_bytes) *workspace_bytes = plan->ws_bytes;
    *out = plan;
    return RMM_OK;
}

rmm_status rmm_plan_destroy(rmm_plan* plan) {
    delete plan;
    return RMM_OK;
}

int64_t rmm_plan_k(const rmm_plan* plan) { return plan ? plan->k : -1; }

size_t rmm_plan_workspace_size(const rmm_plan* plan) { return plan ? plan->ws_bytes : 0; }

rmm_status rmm_select(const rmm_plan* plan, const void* A, int32_t* I, float* s2, void* ws, size_t ws_bytes,
                      void* stream) {
    if (!plan || !A || !I) return RMM_ERR_INVALID_ARG;
    if (!aligned16(A) || (reinterpret_cast<uintptr_t>(I) & 3u) || (s2 && (reinterpret_cast<uintptr_t>(s2) & 3u)))
        return RMM_ERR_INVALID_ARG;
    if (plan->p.d > rmm::kMaxSelectD) return RMM_ERR_UNSUPPORTED;
    rmm_status st = check_workspace(plan, ws, ws_bytes);
    if (st != RMM_OK) return st;
    return run_select(plan, A, I, s2, ws, static_cast<cudaStream_t>(stream));
}

rmm_status rmm_matmul(const rmm_plan* plan, const void* A, const void* B, void* Y, int32_t* I_inout, void* ws,
                      size_t ws_bytes, void* stream) {
    if (!plan) return RMM_ERR_INVALID_ARG;
    if (plan->p.heads != 1 || plan->given_scores || plan->emit_scores) return RMM_ERR_INVALID_ARG;
    return run_matmul(plan, A, B, Y, I_inout, nullptr, nullptr, ws, ws_bytes, stream);
}

rmm_status rmm_matmul_batched(const rmm_plan* plan, const void* A, const void* B, void* Y, int32_t* I_inout,
                              void* ws, size_t ws_bytes, void* stream) {
    if (!plan) return RMM_ERR_INVALID_ARG;
    if (plan->given_scores || plan->emit_scores) return RMM_ERR_INVALID_ARG;
    return run_matmul(plan, A, B, Y, I_inout, nullptr, nullptr, ws, ws_bytes, stream);
}

rmm_status rmm_matmul_ex(const rmm_plan* plan, const void* A, const void* B, void* Y, int32_t* I_inout,
                         const float* s2_in, float* s2_out, void* ws, size_t ws_bytes, void* stream) {
    return run_matmul(plan, A, B, Y, I_inout, s2_in, s2_out, ws, ws_bytes, stream);
}

rmm_status rmm_workspace_init(const rmm_plan* plan, void* ws, size_t ws_bytes, void* stream) {
    if (!plan) return RMM_ERR_INVALID_ARG;
    rmm_status st = check_workspace(plan, ws, ws_bytes);
    if (st != RMM_OK) return st;
    if (cudaMemsetAsync(ws, 0, plan->header_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return RMM_ERR_CUDA;
    return RMM_OK;
}

rmm_status rmm_workspace_status(const rmm_plan* plan, void* ws, void* stream) {
    if (!plan || !ws) return RMM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return RMM_ERR_CUDA;
    int word = 0;
    int* dev_word = ws_at<int>(ws, plan->off_err);
    if (cudaMemcpy(&word, dev_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return RMM_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpy(dev_word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return RMM_ERR_CUDA;
        return RMM_ERR_TIMEOUT;
    }
    return RMM_OK;
}

rmm_status rmm_plan_set_product_events(rmm_plan* plan, void* start, void* stop) {
    if (!plan) return RMM_ERR_INVALID_ARG;
    if ((start == nullptr) != (stop == nullptr)) return RMM_ERR_INVALID_ARG;
    plan->product_start = static_cast<cudaEvent_t>(start);
    plan->product_stop = static_cast<cudaEvent_t>(stop);
    return RMM_OK;
}

int32_t rmm_plan_kernel_launches(const rmm_plan* plan) { return plan ? launches_per_call(plan) : -1; }

const char* rmm_status_string(rmm_status s) {
    switch (s) {
        case RMM_OK: return "RMM_OK";
        case RMM_ERR_INVALID_ARG: return "RMM_ERR_INVALID_ARG";
        case RMM_ERR_UNSUPPORTED: return "RMM_ERR_UNSUPPORTED";
        case RMM_ERR_WORKSPACE: return "RMM_ERR_WORKSPACE";
        case RMM_ERR_CUDA: return "RMM_ERR_CUDA";
        case RMM_ERR_TIMEOUT: return "RMM_ERR_TIMEOUT";
    }
    return "RMM_ERR_UNKNOWN";
}

const char* rmm_version(void) { return "0.1.0"; }

}  // extern "C"
