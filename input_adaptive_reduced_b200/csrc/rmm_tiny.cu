// rmm_tiny.cu -- the whole RMM op in one launch for tiny fp32 problems.
//
// "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
// LLM Inference" (§3.2): s_j^2 = sum_i A[i,j]^2, I = TopK(s, k) (ties to the
// lower index, ascending), Y = A[:, I] B[I, :].  For n <= 64 rows and d <= 256
// columns the op is a few microseconds of latency-bound work, so it runs as a
// single kernel.  Grid (ceil(m / 32), ceil(n / 16)): every CTA stages all of
// A in shared memory, sums the squares of each column in row order (one
// thread per column), takes the TopK in one warp (warp_topk_bits), stages the
// kept rows of B for its 32 columns, and forms its 16 x 32 block of Y with
// fp32 FMAs over the kept indices in ascending order.  CTA (0, 0) writes I.
// (With every index kept the op takes the general path: one product launch.)
#include <cstdint>
#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kTinyThreads = 256;
constexpr int kTinyCols = 32;  // columns of Y per CTA
constexpr int kTinyRows = 16;  // rows of Y per CTA

// dynamic shared memory: A (n d floats), then B[I, c0 : c0 + 32] (k x 32 floats)
template <int J>  // d <= 32 J
__global__ void __launch_bounds__(kTinyThreads) tiny_rmm_kernel(const float* __restrict__ A, const float* __restrict__ B,
                                                                float* __restrict__ Y, int32_t* __restrict__ I_out,
                                                                const int32_t* __restrict__ I_given, int n, int d,
                                                                int m, int k, int64_t lda, int64_t ldb, int64_t ldy,
                                                                float alpha) {
    extern __shared__ float4 smem4[];
    float* sA = reinterpret_cast<float*>(smem4);  // row-major, row stride d
    float* sB = sA + n * d;                       // [k][32]; n d is a multiple of 4
    __shared__ float s2[32 * J];
    __shared__ int32_t sI[32 * J];
    __shared__ float sAk[kTinyRows * 32 * J];  // [16][k]: this CTA's rows of A[:, I]
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c0 = blockIdx.x * kTinyCols, r0 = blockIdx.y * kTinyRows;
    // A into shared memory, every 16-byte copy in flight at once (d and lda
    // are multiples of 4)
    const int dv = d / 4;
    for (int e = tid; e < n * dv; e += kTinyThreads) {
        const int r = e / dv, c = e - r * dv;
        cp_async_16(smem_u32(sA + r * d + 4 * c), A + r * lda + 4 * c, 16u);
    }
    cp_async_wait_all();
    __syncthreads();
    if (I_given) {  // an index outside [0, d) (a caller's error) reads nothing and adds nothing
        for (int t = tid; t < k; t += kTinyThreads) sI[t] = __ldg(I_given + t);
    } else {
        // column scores: thread f sums column f in row order
        for (int f = tid; f < d; f += kTinyThreads) {
            float s = 0.f;
            for (int r = 0; r < n; ++r) s = fmaf(sA[r * d + f], sA[r * d + f], s);
            s2[f] = s;
        }
        __syncthreads();
        if (warp == 0) {  // the TopK, the kept indices in order
            uint32_t key[J];
            bool valid[J];
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int f = lane + 32 * j;
                valid[j] = f < d;
                key[j] = valid[j] ? __float_as_uint(s2[f]) : 0u;
            }
            const uint32_t kept = warp_topk_bits<J>(key, valid, (uint32_t)k, lane);
            uint32_t before = 0;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const bool in = (kept >> j) & 1u;
                const unsigned b = __ballot_sync(0xffffffffu, in);
                if (in) sI[before + __popc(b & ((1u << lane) - 1u))] = lane + 32 * j;
                before += __popc(b);
            }
        }
    }
    __syncthreads();
    if (blockIdx.x == 0 && blockIdx.y == 0 && I_out && !I_given)
        for (int t = tid; t < k; t += kTinyThreads) I_out[t] = sI[t];
    // the kept rows of B for this CTA's columns (m is a multiple of 4: a
    // 16-byte group is all inside or all past the last column)
    for (int e = tid; e < k * (kTinyCols / 4); e += kTinyThreads) {
        const int t = e >> 3, c = (e & 7) * 4;
        const bool in = c0 + c < m && sI[t] >= 0 && sI[t] < d;  // else the copy fills zeros
        cp_async_16(smem_u32(sB + t * kTinyCols + c), in ? B + (int64_t)sI[t] * ldb + c0 + c : B, in ? 16u : 0u);
    }
    cp_async_wait_all();
    __syncthreads();
    // this CTA's rows of A[:, I], contiguous (k <= 256 floats a row)
    for (int e = tid; e < kTinyRows * k; e += kTinyThreads) {
        const int rl = e / k, t = e - rl * k;
        const int j = sI[t];
        sAk[rl * 32 * J + t] = r0 + rl < n && j >= 0 && j < d ? sA[(r0 + rl) * d + j] : 0.f;
    }
    __syncthreads();
    // Y[r, c0 + 2 g .. + 1] = alpha sum_t A[r, I_t] B[I_t, c0 + 2 g .. + 1], t ascending
    const int r = r0 + (tid >> 4), g = tid & 15;
    if (r >= n) return;
    float2 acc = make_float2(0.f, 0.f);
    const float* ar = sAk + (tid >> 4) * 32 * J;
#pragma unroll 8
    for (int t = 0; t < k; ++t) {
        const float a = ar[t];
        const float2 b = reinterpret_cast<const float2*>(sB + t * kTinyCols)[g];
        acc.x = fmaf(a, b.x, acc.x);
        acc.y = fmaf(a, b.y, acc.y);
    }
    const int c = c0 + 2 * g;
    if (c < m) *reinterpret_cast<float2*>(Y + (int64_t)r * ldy + c) = make_float2(alpha * acc.x, alpha * acc.y);
}

}  // namespace

bool tiny_fits(const rmm_problem& p, int64_t k) {
    const bool given = (p.flags & RMM_FLAG_USE_GIVEN_INDICES) != 0;
    return (given || k < p.d) && p.mode == RMM_LINEAR && p.dtype == RMM_F32 && p.heads == 1 && p.n >= 1 && p.n <= kTinyMaxRows &&
           p.d >= 4 && p.d <= 256 && p.d % 4 == 0 && p.lda % 4 == 0 && p.m >= 1 && p.m % 4 == 0 &&
           p.ldb % 4 == 0 && p.ldy % 4 == 0 &&
           (p.flags & (RMM_FLAG_GIVEN_SCORES | RMM_FLAG_EMIT_SCORES)) == 0;
}

template <int J>
cudaError_t launch_tiny_j(const TinyArgs& a, cudaStream_t s) {
    const size_t smem = ((size_t)a.n * a.d + (size_t)a.k * kTinyCols) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(tiny_rmm_kernel<J>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(((size_t)kTinyMaxRows + kTinyCols) * 32 * J * sizeof(float)));
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.m + kTinyCols - 1) / kTinyCols), (unsigned)((a.n + kTinyRows - 1) / kTinyRows));
    return launch_pdl(tiny_rmm_kernel<J>, grid, dim3(kTinyThreads), smem, s, a.A, a.B, a.Y, a.I_out, a.I_given, a.n,
                      a.d, a.m, a.k, a.lda, a.ldb, a.ldy, a.alpha);
}

cudaError_t launch_tiny(const TinyArgs& a, cudaStream_t s) {
    if (a.d <= 64) return launch_tiny_j<2>(a, s);
    if (a.d <= 128) return launch_tiny_j<4>(a, s);
    return launch_tiny_j<8>(a, s);
}

}  // namespace rmm
