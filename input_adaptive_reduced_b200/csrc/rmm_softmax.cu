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
// Grid (row blocks of rows_per_cta rows, heads), 8 warps that own columns and
// one that copies rows.  The op is bound by moving S in and P out, so the rows
// of S stream into shared memory by bulk copies (cp.async.bulk, kStages stages
// of 8 / G rows; under the causal mask only the first ceil8(i + 1) entries of
// row i) while the warps work on earlier rows.  A row is owned by a group of
// G = ceil(t / 1024) warps (lane l of the group's warp w holds the 16-byte
// column groups 32 w + l + 32 G v, v < 4: 32 entries), so its maximum and sum
// are warp shuffles plus, for G > 1, one exchange among the group's warps;
// the CTA's 8 / G groups take 8 / G rows at a time.  Each lane keeps the
// squares of its columns' stored weights in registers (its group's rows in
// row order), every group writes its column sums to the workspace, and a
// second kernel (one thread per column) adds them in row-block and group
// order: the same bits on every call.
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kWarps = 8;                   // warps that own columns
constexpr int kThreads = 32 * kWarps;
constexpr int kBlock = kThreads + 32;       // + one warp that issues the row copies
constexpr int kLaneGroups = 4;              // 16-byte column groups per lane (32 entries)
constexpr int kMaxRows = 128;               // rows per CTA, fewer when the grid would be small
constexpr int kMinCtas = 512;               // about three CTAs per SM of a 148-SM part
constexpr int kStages = 4;                  // row rounds in flight
constexpr int kStageElems = 8192;           // bf16 entries per stage (16 KB): 8 / G rows of 1024 G
constexpr size_t kSmem = (size_t)kStages * kStageElems * 2;
constexpr size_t kHeader = 256;             // workspace: error word, then the column partials
constexpr uint32_t kNegInfPair = 0xff80ff80u;  // two bf16 -inf

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Rows per CTA: 128, halved (down to 16) while the grid has fewer than
// kMinCtas CTAs.  A function of the sizes alone, so that the workspace size
// and the launch agree.
int64_t rows_per_cta(int64_t heads, int64_t n) {
    int64_t r = kMaxRows;
    while (r > 16 && heads * ((n + r - 1) / r) < kMinCtas) r /= 2;
    return r;
}

// Warps per row: one per 1024 entries.
int warps_per_row(int64_t t) { return t <= 1024 ? 1 : t <= 2048 ? 2 : t <= 4096 ? 4 : 8; }

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Barrier `id` of `count` threads that returns the AND of v over them.
__device__ __forceinline__ bool group_barrier_and(int id, int count, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void group_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int G>
__global__ void __launch_bounds__(kBlock, 2) softmax_scores_kernel(
    const __nv_bfloat16* __restrict__ S, __nv_bfloat16* __restrict__ P, float* __restrict__ partials, int* err,
    int n, int t, int64_t lds, int64_t stride_s, int64_t ldp, int64_t stride_p, int causal, int row_blocks,
    int rows) {
    constexpr int NG = kWarps / G;      // row groups per CTA = rows per round
    constexpr int W = 1024 * G;         // entries per staged row
    constexpr int E = 8 * kLaneGroups;  // entries per lane and row
    static_assert(NG * W == kStageElems, "a stage holds one round of rows");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint16_t* stage = reinterpret_cast<uint16_t*>(smem_raw);
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ float red_m[2][kWarps], red_l[2][kWarps];  // per warp (G > 1): its part of the row
    __shared__ int abort_flag, copy_abort;  // give-up flags of the column-owning warps and of the copy warp
    const int h = blockIdx.y, rb = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint16_t* Sh = reinterpret_cast<const uint16_t*>(S) + (int64_t)h * stride_s;
    uint16_t* Ph = reinterpret_cast<uint16_t*>(P) + (int64_t)h * stride_p;
    constexpr float kLog2e = 1.4426950408889634f;  // e^x = 2^(x log2 e)
    const int r0 = rb * rows, r1 = min(n, r0 + rows);
    const int rounds = (r1 - r0 + NG - 1) / NG;
    // entries of row i that are read: all t, or under the causal mask the
    // 16-byte groups up to the diagonal
    auto row_len = [&](int row) { return causal ? min(t, (row + 8) & ~7) : t; };
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kWarps);  // one arrival per column-owning warp
        }
        abort_flag = 0;
        copy_abort = 0;
        mbar_fence_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    if (warp == kWarps) {
        // copy warp: refill each stage as soon as the 8 warps have read it
        if (lane == 0) {
            for (int j = 0; j < rounds; ++j) {
                const int st = j % kStages;
                if (j >= kStages && !mbar_wait(&empty[st], (uint32_t)(j / kStages - 1) & 1u, &copy_abort, err,
                                               kErrTimeoutProducer))
                    break;
                uint32_t bytes = 0;
                for (int g = 0; g < NG; ++g) {
                    const int row = r0 + j * NG + g;
                    if (row < r1) bytes += 2u * (uint32_t)row_len(row);
                }
                mbar_arrive_expect_tx(&full[st], bytes);
                for (int g = 0; g < NG; ++g) {
                    const int row = r0 + j * NG + g;
                    if (row < r1)
                        bulk_load(stage + ((size_t)st * NG + g) * W, Sh + (int64_t)row * lds, 2u * row_len(row),
                                  &full[st]);
                }
            }
        }
        return;
    }
    const int grp = warp / G, wg = warp % G;  // row group, warp within the group
    const int bar_id = 1 + grp;               // the group's named barrier (G > 1)
    float acc[E];
#pragma unroll
    for (int i = 0; i < E; ++i) acc[i] = 0.f;
#pragma unroll 1
    for (int j = 0; j < rounds; ++j) {
        const int st = j % kStages, par = j & 1;
        const int row = r0 + j * NG + grp;
        const int len = row < r1 ? row_len(row) : 0;
        bool got = mbar_wait(&full[st], (uint32_t)(j / kStages) & 1u, &abort_flag, err, kErrTimeoutEpilogue);
        // this lane's scores as bf16 pairs (-inf where masked); their maximum
        // is taken on the pairs (exact: a maximum of bf16 values)
        const uint16_t* src = stage + ((size_t)st * NG + grp) * W;
        uint32_t q[E / 2];
#pragma unroll
        for (int v = 0; v < kLaneGroups; ++v) {
            const int c0 = 8 * (wg * 32 + lane + 32 * G * v);
            uint4 u = make_uint4(kNegInfPair, kNegInfPair, kNegInfPair, kNegInfPair);
            if (c0 < len) {
                u = *reinterpret_cast<const uint4*>(src + c0);
                if (causal && c0 + 7 > row) {  // the group on the diagonal: -inf past it
                    uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (c0 + i > row)
                            wd[i >> 1] = (i & 1) ? ((wd[i >> 1] & 0xffffu) | 0xff800000u)
                                                 : ((wd[i >> 1] & 0xffff0000u) | 0xff80u);
                    u = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                }
            }
            q[4 * v] = u.x;
            q[4 * v + 1] = u.y;
            q[4 * v + 2] = u.z;
            q[4 * v + 3] = u.w;
        }
        // this warp has read the stage: the copy warp may refill it
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        __nv_bfloat162 m2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) m2[i] = *reinterpret_cast<const __nv_bfloat162*>(&q[i]);
#pragma unroll
        for (int i = 4; i < E / 2; ++i) m2[i & 3] = __hmax2(m2[i & 3], *reinterpret_cast<const __nv_bfloat162*>(&q[i]));
        const __nv_bfloat162 mm = __hmax2(__hmax2(m2[0], m2[1]), __hmax2(m2[2], m2[3]));
        float mx = fmaxf(__low2float(mm), __high2float(mm));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if constexpr (G > 1) {
            if (lane == 0) red_m[par][warp] = mx;
            got = group_barrier_and(bar_id, 32 * G, got);
            mx = red_m[par][grp * G];
#pragma unroll
            for (int w = 1; w < G; ++w) mx = fmaxf(mx, red_m[par][grp * G + w]);
        } else {
            got = __all_sync(0xffffffffu, got);
        }
        if (!got) break;  // the same decision in every warp of the group
        // exponentials relative to the row maximum, and the row sum; a row
        // without a finite entry gets base +inf: all its weights are 0
        const float base = mx == -INFINITY ? INFINITY : mx * kLog2e;
        float x[E];
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int v = 0; v < kLaneGroups; ++v) {
            const int c0 = 8 * (wg * 32 + lane + 32 * G * v);
            if (c0 < len) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t w = q[4 * v + (i >> 1)];
                    const float xi = __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
                    const float e = fast_exp2(fmaf(xi, kLog2e, -base));  // 2^-inf = 0 where masked
                    x[8 * v + i] = e;
                    sm[i & 3] += e;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) x[8 * v + i] = 0.f;
            }
        }
        float sum = (sm[0] + sm[1]) + (sm[2] + sm[3]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if constexpr (G > 1) {
            if (lane == 0) red_l[par][warp] = sum;
            group_barrier(bar_id, 32 * G);
            sum = red_l[par][grp * G];
#pragma unroll
            for (int w = 1; w < G; ++w) sum += red_l[par][grp * G + w];
        }
        if (row >= r1) continue;
        // P = the exponentials over the row sum, rounded to bf16; the squares
        // of the stored weights
        const float inv = sum > 0.f ? 1.0f / sum : 0.f;
#pragma unroll
        for (int v = 0; v < kLaneGroups; ++v) {
            const int c0 = 8 * (wg * 32 + lane + 32 * G * v);
            if (c0 >= t) continue;
            uint4 out = make_uint4(0u, 0u, 0u, 0u);  // past the causal range: 0
            if (c0 < len) {
                uint32_t wv[4];
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const __nv_bfloat162 p2 = __floats2bfloat162_rn(x[8 * v + i] * inv, x[8 * v + i + 1] * inv);
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
    // this group's column sums: partial (row block rb, group grp) of the head
    float* part = partials + (((int64_t)h * row_blocks + rb) * NG + grp) * t;
#pragma unroll
    for (int v = 0; v < kLaneGroups; ++v) {
        const int c0 = 8 * (wg * 32 + lane + 32 * G * v);
        if (c0 >= t) continue;
        float4* dst = reinterpret_cast<float4*>(part + c0);
        __stcg(dst, make_float4(acc[8 * v], acc[8 * v + 1], acc[8 * v + 2], acc[8 * v + 3]));
        __stcg(dst + 1, make_float4(acc[8 * v + 4], acc[8 * v + 5], acc[8 * v + 6], acc[8 * v + 7]));
    }
}

// s2[h][c] = the partial column sums added in order (row block, then group;
// 16 loads in flight per thread).
__global__ void __launch_bounds__(256) softmax_scores_reduce_kernel(const float* __restrict__ partials,
                                                                    float* __restrict__ s2, int t, int parts) {
    pdl_wait();
    pdl_trigger();
    const int h = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= t) return;
    const float* pc = partials + (int64_t)h * parts * t + c;
    float z = 0.f;
    for (int b = 0; b < parts; b += 16) {
        float v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] = b + u < parts ? __ldcg(pc + (int64_t)(b + u) * t) : 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) z += v[u];  // the terms past the last part are +0
    }
    s2[(int64_t)h * t + c] = z;
}

template <int G>
cudaError_t launch_softmax(const void* S, void* P, float* s2, float* partials, int* err, int64_t heads, int64_t n,
                           int64_t t, int64_t lds, int64_t stride_s, int64_t ldp, int64_t stride_p, int causal,
                           int row_blocks, int rows, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(softmax_scores_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(softmax_scores_kernel<G>, dim3((unsigned)row_blocks, (unsigned)heads), dim3(kBlock), kSmem, s,
                   static_cast<const __nv_bfloat16*>(S), static_cast<__nv_bfloat16*>(P), partials, err, (int)n,
                   (int)t, lds, stride_s, ldp, stride_p, causal, row_blocks, rows);
    if (e != cudaSuccess) return e;
    return launch_pdl(softmax_scores_reduce_kernel, dim3((unsigned)((t + 255) / 256), (unsigned)heads), dim3(256), 0,
                      s, (const float*)partials, s2, (int)t, row_blocks * (kWarps / G));
}

}  // namespace
}  // namespace rmm

extern "C" {

size_t rmm_softmax_workspace_size(int64_t heads, int64_t n, int64_t t) {
    if (heads < 1 || n < 1 || t < 1) return 0;
    const int64_t rows = rmm::rows_per_cta(heads, n);
    const int64_t parts = (n + rows - 1) / rows * (rmm::kWarps / rmm::warps_per_row(t));
    return rmm::kHeader + rmm::align256(static_cast<size_t>(heads) * parts * t * sizeof(float));
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
    switch (rmm::warps_per_row(t)) {
        case 1:
            e = rmm::launch_softmax<1>(S, P, s2, partials, err, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                       row_blocks, rows, s);
            break;
        case 2:
            e = rmm::launch_softmax<2>(S, P, s2, partials, err, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                       row_blocks, rows, s);
            break;
        case 4:
            e = rmm::launch_softmax<4>(S, P, s2, partials, err, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                       row_blocks, rows, s);
            break;
        default:
            e = rmm::launch_softmax<8>(S, P, s2, partials, err, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                       row_blocks, rows, s);
            break;
    }
    return e == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
}

}  // extern "C"
