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
// Grid (row blocks of kRows rows, heads), 256 threads.  Thread x owns the
// 16-byte column groups x, x + 256, ... of every row; a CTA walks its rows in
// batches (several rows in flight), finds each row's maximum and exponential
// sum by block reductions, writes P and keeps the squares of the rounded
// weights in registers (its columns, its rows in row order).  The CTA's column
// sums go to the workspace; the last CTA of the head adds the row blocks' sums
// in block order (the same bits on every call) and resets the head's counter.
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 128;  // rows per CTA

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// E columns per thread per row (t <= kThreads * E), B rows per batch.
template <int E, int B>
__global__ void __launch_bounds__(kThreads) softmax_scores_kernel(
    const __nv_bfloat16* __restrict__ S, __nv_bfloat16* __restrict__ P, float* __restrict__ s2,
    float* __restrict__ partials, unsigned* __restrict__ counters, int n, int t, int64_t lds, int64_t stride_s,
    int64_t ldp, int64_t stride_p, int causal, int row_blocks) {
    constexpr int V = E / 8;  // 16-byte groups per thread per row
    __shared__ float red[B][kWarps];
    __shared__ int last_cta;
    pdl_wait();
    pdl_trigger();
    const int h = blockIdx.y, rb = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint16_t* Sh = reinterpret_cast<const uint16_t*>(S) + (int64_t)h * stride_s;
    uint16_t* Ph = reinterpret_cast<uint16_t*>(P) + (int64_t)h * stride_p;
    const float ninf = -__int_as_float(0x7f800000);
    constexpr float kLog2e = 1.4426950408889634f;  // scores are taken in base 2: e^x = 2^(x log2 e)
    float acc[E];
#pragma unroll
    for (int i = 0; i < E; ++i) acc[i] = 0.f;
    const int r0 = rb * kRows, r1 = min(n, r0 + kRows);
#pragma unroll 1
    for (int r = r0; r < r1; r += B) {
        float x[B][E];
        float mx[B];
        bool vin[B][V];  // the 16-byte group holds an entry that is read (not masked)
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int row = r + b;
            mx[b] = ninf;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int c0 = 8 * (tid + kThreads * v);
                const bool in = row < r1 && c0 < t && (!causal || c0 <= row);
                vin[b][v] = in;
                uint4 q = make_uint4(0u, 0u, 0u, 0u);
                if (in) q = __ldcs(reinterpret_cast<const uint4*>(Sh + (int64_t)row * lds + c0));
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
                const bool whole = !causal || c0 + 7 <= row;  // no entry of the group past the diagonal
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const bool live = in && (whole || c0 + j <= row);
                    const float y = live ? bf16_bits_to_float((w[j >> 1] >> (16 * (j & 1))) & 0xffffu) * kLog2e
                                         : ninf;
                    x[b][8 * v + j] = y;
                    mx[b] = fmaxf(mx[b], y);
                }
            }
        }
        // row maxima
#pragma unroll
        for (int b = 0; b < B; ++b) {
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx[b] = fmaxf(mx[b], __shfl_xor_sync(0xffffffffu, mx[b], o));
            if (lane == 0) red[b][warp] = mx[b];
        }
        __syncthreads();
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float m = red[b][0];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[b][w]);
            mx[b] = m;
        }
        __syncthreads();
        // exponentials and row sums
        float sum[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            sum[b] = 0.f;
            const bool finite_row = mx[b] > ninf;  // a row without a finite entry is written as zeros
#pragma unroll
            for (int v = 0; v < V; ++v) {
                if (finite_row && vin[b][v]) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float e = exp2f(x[b][8 * v + j] - mx[b]);  // 2^-inf = 0 where masked
                        x[b][8 * v + j] = e;
                        sum[b] += e;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[b][8 * v + j] = 0.f;
                }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum[b] += __shfl_xor_sync(0xffffffffu, sum[b], o);
            if (lane == 0) red[b][warp] = sum[b];
        }
        __syncthreads();
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float z = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) z += red[b][w];
            sum[b] = z;
        }
        __syncthreads();
        // store P; add the squares of the stored weights
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int row = r + b;
            if (row >= r1) break;
            const float inv = sum[b] > 0.f ? 1.0f / sum[b] : 0.f;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int c0 = 8 * (tid + kThreads * v);
                if (c0 >= t) continue;
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const __nv_bfloat162 p2 = __floats2bfloat162_rn(x[b][8 * v + j] * inv, x[b][8 * v + j + 1] * inv);
                    const float2 f = __bfloat1622float2(p2);
                    acc[8 * v + j] += f.x * f.x;
                    acc[8 * v + j + 1] += f.y * f.y;
                    w[j >> 1] = *reinterpret_cast<const uint32_t*>(&p2);
                }
                *reinterpret_cast<uint4*>(Ph + (int64_t)row * ldp + c0) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    // this CTA's column sums, then the head's last CTA adds them in block order
    float* part = partials + ((int64_t)h * row_blocks + rb) * t;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int c0 = 8 * (tid + kThreads * v);
        if (c0 >= t) continue;
        float4* dst = reinterpret_cast<float4*>(part + c0);
        __stcg(dst, make_float4(acc[8 * v], acc[8 * v + 1], acc[8 * v + 2], acc[8 * v + 3]));
        __stcg(dst + 1, make_float4(acc[8 * v + 4], acc[8 * v + 5], acc[8 * v + 6], acc[8 * v + 7]));
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) last_cta = atomicAdd(counters + h, 1u) == (unsigned)(row_blocks - 1) ? 1 : 0;
    __syncthreads();
    if (!last_cta) return;
    __threadfence();
    const float* ph = partials + (int64_t)h * row_blocks * t;
    for (int c = tid; c < t; c += kThreads) {
        float z = 0.f;
        for (int j = 0; j < row_blocks; ++j) z += __ldcg(ph + (int64_t)j * t + c);
        s2[(int64_t)h * t + c] = z;
    }
    if (tid == 0) counters[h] = 0u;
}

template <int E, int B>
cudaError_t launch_softmax(const void* S, void* P, float* s2, float* partials, unsigned* counters, int64_t heads,
                           int64_t n, int64_t t, int64_t lds, int64_t stride_s, int64_t ldp, int64_t stride_p,
                           int causal, int row_blocks, cudaStream_t s) {
    return launch_pdl(softmax_scores_kernel<E, B>, dim3((unsigned)row_blocks, (unsigned)heads), dim3(kThreads), 0, s,
                      static_cast<const __nv_bfloat16*>(S), static_cast<__nv_bfloat16*>(P), s2, partials, counters,
                      (int)n, (int)t, lds, stride_s, ldp, stride_p, causal, row_blocks);
}

}  // namespace
}  // namespace rmm

extern "C" {

size_t rmm_softmax_workspace_size(int64_t heads, int64_t n, int64_t t) {
    if (heads < 1 || n < 1 || t < 1) return 0;
    const int64_t row_blocks = (n + rmm::kRows - 1) / rmm::kRows;
    return rmm::align256(static_cast<size_t>(heads) * sizeof(unsigned)) +
           rmm::align256(static_cast<size_t>(heads) * row_blocks * t * sizeof(float));
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
    const int row_blocks = static_cast<int>((n + rmm::kRows - 1) / rmm::kRows);
    unsigned* counters = static_cast<unsigned*>(ws);
    float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                               rmm::align256(static_cast<size_t>(heads) * sizeof(unsigned)));
    const int causal = (flags & RMM_FLAG_CAUSAL) ? 1 : 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (t <= 2048)
        e = rmm::launch_softmax<8, 4>(S, P, s2, partials, counters, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                      row_blocks, s);
    else if (t <= 4096)
        e = rmm::launch_softmax<16, 4>(S, P, s2, partials, counters, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                       row_blocks, s);
    else
        e = rmm::launch_softmax<32, 2>(S, P, s2, partials, counters, heads, n, t, lds, stride_s, ldp, stride_p, causal,
                                       row_blocks, s);
    return e == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
}

}  // extern "C"
