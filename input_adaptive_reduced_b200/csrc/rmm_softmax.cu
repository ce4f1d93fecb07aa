// rmm_softmax.cu -- attention weights with producer-fused token scores.
//
// "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
// LLM Inference" (§3.3 "Attention") forms P = softmax(S~ + M) and, for the
// value product, keeps the tokens t with the largest a_t = ||P[:, t]||_2.
// Scoring the tokens is a full extra read of P when the PV op does it (the
// op is bound by reading P).  This kernel is the op that produces P: while it
// writes each row of P it also adds the squares of the stored bf16 weights of
// its rows into per-column sums, so the PV op can take them as given scores
// (RMM_FLAG_GIVEN_SCORES) and skip its score pass.
//
// Grid (row blocks of rows_per_cta rows, heads), 256 threads, three CTAs per
// SM.  The
// op is bound by moving S in and P out, so the rows of S stream into shared
// memory by bulk copies (cp.async.bulk, kStages stages of R rows; under the
// causal mask only the first ceil8(i + 1) entries of row i) while the CTA
// works on earlier rows.  Thread x owns the 16-byte column groups x, x + 256,
// ... of every row.  Per batch of R rows: the row maxima (warp shuffles, then
// the 8 warps' maxima in warp order), the exponentials and the row sums (the
// same two steps), then P and the squares of the stored weights, which the
// thread keeps in registers (its columns, its rows in row order).  The CTA's
// column sums go to the workspace, and a second kernel (one thread per
// column) adds the row blocks' sums in block order: the same bits on every
// call.
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRows = 128;        // rows per CTA, fewer when the grid would be small
constexpr int kMinCtas = 512;        // about three CTAs per SM of a 148-SM part
constexpr int kStages = 4;           // row batches in flight
constexpr int kStageElems = 8192;    // bf16 entries per stage (16 KB)
constexpr size_t kSmem = (size_t)kStages * kStageElems * 2;
constexpr size_t kHeader = 256;      // workspace: error word, then the column partials

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Rows per CTA: 128, halved (down to 16) while the grid has fewer than
// kMinCtas CTAs.  A function of the sizes alone, so that the workspace size
// and the launch agree.
int64_t rows_per_cta(int64_t heads, int64_t n) {
    int64_t r = kMaxRows;
    while (r > 16 && heads * ((n + r - 1) / r) < kMinCtas) r /= 2;
    return r;
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// E columns per thread per row (t <= kThreads * E); R rows per stage.
template <int E>
__global__ void __launch_bounds__(kThreads, 3) softmax_scores_kernel(
    const __nv_bfloat16* __restrict__ S, __nv_bfloat16* __restrict__ P,
    float* __restrict__ partials, int* err, int n, int t, int64_t lds,
    int64_t stride_s, int64_t ldp, int64_t stride_p, int causal, int row_blocks, int rows) {
    constexpr int V = E / 8;                       // 16-byte groups per thread per row
    constexpr int W = kThreads * E;                // entries per staged row
    constexpr int R = kStageElems / W;             // rows per stage
    static_assert(R >= 1, "a stage holds at least one row");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint16_t* stage = reinterpret_cast<uint16_t*>(smem_raw);
    __shared__ uint64_t full[kStages];
    __shared__ float red_m[2][R][kWarps], red_l[2][R][kWarps];
    __shared__ int abort_flag;
    const int h = blockIdx.y, rb = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint16_t* Sh = reinterpret_cast<const uint16_t*>(S) + (int64_t)h * stride_s;
    uint16_t* Ph = reinterpret_cast<uint16_t*>(P) + (int64_t)h * stride_p;
    constexpr float kLog2e = 1.4426950408889634f;  // e^x = 2^(x log2 e)
    const int r0 = rb * rows, r1 = min(n, r0 + rows);
    const int batches = (r1 - r0 + R - 1) / R;
    // entries of row i that are read: all t, or under the causal mask the
    // 16-byte groups up to the diagonal
    auto row_len = [&](int row) { return causal ? min(t, (row + 8) & ~7) : t; };
    auto issue = [&](int j) {
        const int st = j % kStages;
        uint32_t bytes = 0;
        for (int b = 0; b < R; ++b) {
            const int row = r0 + j * R + b;
            if (row < r1) bytes += 2u * (uint32_t)row_len(row);
        }
        mbar_arrive_expect_tx(&full[st], bytes);
        for (int b = 0; b < R; ++b) {
            const int row = r0 + j * R + b;
            if (row < r1)
                bulk_load(stage + ((size_t)st * R + b) * W, Sh + (int64_t)row * lds, 2u * row_len(row), &full[st]);
        }
    };
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&full[i], 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    if (tid == 0)
        for (int j = 0; j < min(kStages, batches); ++j) issue(j);
    float acc[E];
#pragma unroll
    for (int i = 0; i < E; ++i) acc[i] = 0.f;
#pragma unroll 1
    for (int j = 0; j < batches; ++j) {
        const int st = j % kStages, par = j & 1;
        const bool got = mbar_wait(&full[st], (uint32_t)(j / kStages) & 1u, &abort_flag, err, kErrTimeoutEpilogue);
        // this thread's scores (-inf where masked) and their maximum per row
        float x[R][E];
        int len[R];
#pragma unroll
        for (int b = 0; b < R; ++b) {
            const int row = r0 + j * R + b;
            len[b] = row < r1 ? row_len(row) : 0;
            const uint16_t* src = stage + ((size_t)st * R + b) * W;
            float mx = -INFINITY;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int c0 = 8 * (tid + kThreads * v);
                if (c0 < len[b]) {
                    const uint4 q = *reinterpret_cast<const uint4*>(src + c0);
                    const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        x[b][8 * v + i] = __uint_as_float((i & 1) ? (wd[i >> 1] & 0xffff0000u) : (wd[i >> 1] << 16));
                    if (causal && c0 + 7 > row) {  // the group on the diagonal
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            if (c0 + i > row) x[b][8 * v + i] = -INFINITY;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[b][8 * v + i] = -INFINITY;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) mx = fmaxf(mx, x[b][8 * v + i]);
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) red_m[par][b][warp] = mx;
        }
        // every thread has read the stage: it may be refilled
        if (!__syncthreads_and(got)) break;
        if (tid == 0 && j + kStages < batches) {
            fence_proxy_async_smem();
            issue(j + kStages);
        }
        // exponentials relative to the row maximum, and the row sums
#pragma unroll
        for (int b = 0; b < R; ++b) {
            float mx = red_m[par][b][0];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) mx = fmaxf(mx, red_m[par][b][w]);
            // a row without a finite entry gets base +inf: all its weights are 0
            const float base = mx == -INFINITY ? INFINITY : mx * kLog2e;
            float sm[2] = {0.f, 0.f};
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int c0 = 8 * (tid + kThreads * v);
                if (c0 < len[b]) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float e = fast_exp2(fmaf(x[b][8 * v + i], kLog2e, -base));  // 2^-inf = 0 where masked
                        x[b][8 * v + i] = e;
                        sm[i & 1] += e;
                    }
                }
            }
            float sum = sm[0] + sm[1];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) red_l[par][b][warp] = sum;
        }
        __syncthreads();
        // P = the exponentials over the row sum, rounded to bf16; the squares of
        // the stored weights
#pragma unroll
        for (int b = 0; b < R; ++b) {
            const int row = r0 + j * R + b;
            if (row >= r1) break;
            float sum = red_l[par][b][0];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) sum += red_l[par][b][w];
            const float inv = sum > 0.f ? 1.0f / sum : 0.f;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int c0 = 8 * (tid + kThreads * v);
                if (c0 >= t) continue;
                uint4 out = make_uint4(0u, 0u, 0u, 0u);  // past the causal range: 0
                if (c0 < len[b]) {
                    uint32_t wv[4];
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        const __nv_bfloat162 p2 = __floats2bfloat162_rn(x[b][8 * v + i] * inv, x[b][8 * v + i + 1] * inv);
                        wv[i >> 1] = *reinterpret_cast<const uint32_t*>(&p2);
                        const float lo = __uint_as_float(wv[i >> 1] << 16), hi = __uint_as_float(wv[i >> 1] & 0xffff0000u);
                        acc[8 * v + i] = fmaf(lo, lo, acc[8 * v + i]);
                        acc[8 * v + i + 1] = fmaf(hi, hi, acc[8 * v + i + 1]);
                    }
                    out = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                }
                *reinterpret_cast<uint4*>(Ph + (int64_t)row * ldp + c0) = out;
            }
        }
    }
    // this CTA's column sums
    float* part = partials + ((int64_t)h * row_blocks + rb) * t;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int c0 = 8 * (tid + kThreads * v);
        if (c0 >= t) continue;
        float4* dst = reinterpret_cast<float4*>(part + c0);
        __stcg(dst, make_float4(acc[8 * v], acc[8 * v + 1], acc[8 * v + 2], acc[8 * v + 3]));
        __stcg(dst + 1, make_float4(acc[8 * v + 4], acc[8 * v + 5], acc[8 * v + 6], acc[8 * v + 7]));
    }
}

// s2[h][c] = the row blocks' column sums added in block order (16 loads in
// flight per thread).
__global__ void __launch_bounds__(256) softmax_scores_reduce_kernel(const float* __restrict__ partials,
                                                                    float* __restrict__ s2, int t, int row_blocks) {
    pdl_wait();
    pdl_trigger();
    const int h = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= t) return;
    const float* pc = partials + (int64_t)h * row_blocks * t + c;
    float z = 0.f;
    for (int b = 0; b < row_blocks; b += 16) {
        float v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] = b + u < row_blocks ? __ldcg(pc + (int64_t)(b + u) * t) : 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) z += v[u];  // the terms past the last block are +0
    }
    s2[(int64_t)h * t + c] = z;
}

template <int E>
cudaError_t launch_softmax(const void* S, void* P, float* s2, float* partials, int* err, int64_t heads, int64_t n,
                           int64_t t, int64_t lds, int64_t stride_s, int64_t ldp, int64_t stride_p, int causal,
                           int row_blocks, int rows, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(softmax_scores_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(softmax_scores_kernel<E>, dim3((unsigned)row_blocks, (unsigned)heads), dim3(kThreads), kSmem, s,
                   static_cast<const __nv_bfloat16*>(S), static_cast<__nv_bfloat16*>(P), partials, err, (int)n,
                   (int)t, lds, stride_s, ldp, stride_p, causal, row_blocks, rows);
    if (e != cudaSuccess) return e;
    return launch_pdl(softmax_scores_reduce_kernel, dim3((unsigned)((t + 255) / 256), (unsigned)heads), dim3(256), 0,
                      s, (const float*)partials, s2, (int)t, row_blocks);
}

}  // namespace
}  // namespace rmm

extern "C" {

size_t rmm_softmax_workspace_size(int64_t heads, int64_t n, int64_t t) {
    if (heads < 1 || n < 1 || t < 1) return 0;
    const int64_t rows = rmm::rows_per_cta(heads, n);
    const int64_t row_blocks = (n + rows - 1) / rows;
    return rmm::kHeader + rmm::align256(static_cast<size_t>(heads) * row_blocks * t * sizeof(float));
}

rmm_status rmm_softmax_scores(const void* S, void* P, float* s2, int64_t heads, int64_t n, int64_t t, int64_t lds,
                              int64_t stride_s, int64_t ldp, int64_t stride_p, uint32_t flags, void* ws,
                              size_t ws_bytes, void* stream) {
    if (heads < 1 || n < 0 || t < 1) return RMM_ERR_INVALID_ARG;
    if (n == 0) return RMM_OK;
    if (!S || !P || !s2) return RMM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(S) & 15u) || (reinterpret_cast<uintptr_t>(P) & 15u) ||
        (reinterpret_cast<uintptr_t>(s2) & 3u))
        return RMM_ERR_INVALID_ARG;
    if (flags & ~RMM_FLAG_CAUSAL) return RMM_ERR_INVALID_ARG;
    if (t % 8 != 0 || lds < t || ldp < t || lds % 8 != 0 || ldp % 8 != 0) return RMM_ERR_INVALID_ARG;
    if (heads > 1 && (stride_s % 8 != 0 || stride_p % 8 != 0 || stride_s < n * lds || stride_p < n * ldp))
        return RMM_ERR_INVALID_ARG;
    if (t > 8192 || heads > 65535 || n > (int64_t(1) << 30)) return RMM_ERR_UNSUPPORTED;
    const size_t need = rmm_softmax_workspace_size(heads, n, t);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return RMM_ERR_WORKSPACE;
    const int rows = static_cast<int>(rmm::rows_per_cta(heads, n));
    const int row_blocks = static_cast<int>((n + rows - 1) / rows);
    int* err = static_cast<int*>(ws);
    float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + rmm::kHeader);
    const int causal = (flags & RMM_FLAG_CAUSAL) ? 1 : 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (t <= 2048)
        e = rmm::launch_softmax<8>(S, P, s2, partials, err, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                   row_blocks, rows, s);
    else if (t <= 4096)
        e = rmm::launch_softmax<16>(S, P, s2, partials, err, heads, n, t, lds, stride_s, ldp, stride_p,
                                    causal, row_blocks, rows, s);
    else
        e = rmm::launch_softmax<32>(S, P, s2, partials, err, heads, n, t, lds, stride_s, ldp, stride_p,
                                    causal, row_blocks, rows, s);
    return e == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
}

}  // extern "C"
