// rmm_pack.cu -- staging of the gathered operand columns A[:, I] of Reduced
// Matrix Multiplication ("Reduced Matrix Multiplication: Input-Adaptive
// Matrix-Product Reduction for LLM Inference", §3.2: the product runs over the
// retained slice A[:, I] only).  A row-major operand keeps the contraction
// axis contiguous, so its retained columns are element-granular and cannot be
// fetched by tensor-memory-access tiles; this pass compacts them into a dense
// K-major buffer (rows x roundup(k, 8)) that the tensor-core GEMM then reads
// with TMA.  Used for A in every mode and for K in the QK mode.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kPackThreads = 256;
constexpr int kPackRows = 16;  // rows per CTA; the 8 indices of a thread are reused across them

// grid (ceil(ld_dst / (8*256)), ceil(rows / 16), heads).  Thread t owns output
// columns [8t, 8t+8) of its CTA's slice; it loads their 8 source indices once
// and writes 16-byte (bf16) or 2 x 16-byte (fp32) rows of the packed buffer.
// The body of one CTA of the grid; (bx, by, h) is its block index.
template <typename T>
__device__ __forceinline__ void pack_block(const T* __restrict__ src, int64_t rows, int64_t d, int64_t ld_src,
                                           int64_t stride_src, int group, const int32_t* __restrict__ I,
                                           int64_t I_stride, int64_t k, T* __restrict__ dst, int64_t ld_dst,
                                           int64_t stride_dst, int64_t bx, int64_t by, int h) {
    const int64_t t0 = (bx * kPackThreads + threadIdx.x) * 8;
    if (t0 >= ld_dst) return;
    int32_t idx[8];
    bool live[8];
    const int32_t* Ih = I + (int64_t)h * I_stride;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        live[v] = t0 + v < k;
        int32_t j = live[v] ? __ldg(Ih + t0 + v) : 0;
        idx[v] = min(max(j, 0), (int32_t)(d - 1));  // keep every load in bounds
    }
    const T* sh = src + (int64_t)(h / group) * stride_src;
    T* dh = dst + (int64_t)h * stride_dst;
    const int64_t r_beg = by * kPackRows;
    const int64_t r_end = min(rows, r_beg + kPackRows);
    // four rows per round: thirty-two independent element loads in flight per thread
    for (int64_t r = r_beg; r < r_end; r += 4) {
        const int nq = (int)(r_end - r < 4 ? r_end - r : 4);
        __align__(16) T vals[4][8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const T* sq = sh + (r + (q < nq ? q : 0)) * ld_src;
#pragma unroll
            for (int v = 0; v < 8; ++v) vals[q][v] = live[v] ? sq[idx[v]] : T(0.f);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (q >= nq) break;
            T* o = dh + (r + q) * ld_dst + t0;
            if constexpr (sizeof(T) == 1) {
                *reinterpret_cast<uint2*>(o) = *reinterpret_cast<const uint2*>(vals[q]);
            } else if constexpr (sizeof(T) == 2) {
                *reinterpret_cast<uint4*>(o) = *reinterpret_cast<const uint4*>(vals[q]);
            } else {
                reinterpret_cast<uint4*>(o)[0] = reinterpret_cast<const uint4*>(vals[q])[0];
                reinterpret_cast<uint4*>(o)[1] = reinterpret_cast<const uint4*>(vals[q])[1];
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(
    const T* __restrict__ src, int64_t rows, int64_t d, int64_t ld_src, int64_t stride_src, int group,
    const int32_t* __restrict__ I, int64_t I_stride, int64_t k, T* __restrict__ dst, int64_t ld_dst,
    int64_t stride_dst) {
    pdl_wait();
    pdl_trigger();
    pack_block(src, rows, d, ld_src, stride_src, group, I, I_stride, k, dst, ld_dst, stride_dst, blockIdx.x,
               blockIdx.y, (int)blockIdx.z);
}

// Transposing variant for fp32 operands: dst[h][c][t] = src[h / group][I[h][t]][c]
// (t < k; 0 for k <= t < ld_dst), i.e. the gathered rows B[I, :] of a row-major
// d x m matrix written K-major (m x ld_dst).  32 x 32 tiles through shared memory.
template <typename T>
__global__ void __launch_bounds__(256) pack_rows_transposed_kernel(
    const T* __restrict__ src, int64_t d, int64_t cols, int64_t ld_src, int64_t stride_src, int group,
    const int32_t* __restrict__ I, int64_t I_stride, int64_t k, T* __restrict__ dst, int64_t ld_dst,
    int64_t stride_dst) {
    pdl_wait();
    pdl_trigger();
    __shared__ T tile[32][33];
    const int h = blockIdx.z;
    const int64_t t0 = (int64_t)blockIdx.x * 32, c0 = (int64_t)blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    const T* sh = src + (int64_t)(h / group) * stride_src;
    const int32_t* Ih = I ? I + (int64_t)h * I_stride : nullptr;
    for (int r = ty; r < 32; r += 8) {
        const int64_t t = t0 + r, c = c0 + tx;
        T v = T(0.f);
        if (t < k && c < cols) {
            int64_t j = Ih ? (int64_t)__ldg(Ih + t) : t;
            j = j < 0 ? 0 : (j >= d ? d - 1 : j);
            v = sh[j * ld_src + c];
        }
        tile[r][tx] = v;
    }
    __syncthreads();
    T* dh = dst + (int64_t)h * stride_dst;
    for (int r = ty; r < 32; r += 8) {
        const int64_t c = c0 + r, t = t0 + tx;
        if (c < cols && t < ld_dst) dh[c * ld_dst + t] = tile[tx][r];
    }
}

// Row gather for bf16 B operands: dst[h][t][:] = src[h / group][I[h][t]][:]
// for t < k (rows of `cols` elements).  grid (ceil(k / kRowsPerCta), heads);
// the CTA copies its rows with 16-byte loads and stores, four independent
// chunks in flight per thread.  The retained rows are contiguous segments of B,
// so both sides are fully coalesced.
constexpr int kRowsPerCta = 8;

template <typename T, int U = 4>
__device__ __forceinline__ void pack_rows_block(const T* __restrict__ src, int64_t d, int64_t cols, int64_t ld_src,
                                                int64_t stride_src, int group, const int32_t* __restrict__ I,
                                                int64_t I_stride, int64_t k, T* __restrict__ dst, int64_t ld_dst,
                                                int64_t stride_dst, int64_t bx, int h) {
    constexpr int V = 16 / sizeof(T);
    const int cpr = (int)(cols / V);
    const int64_t t0 = bx * kRowsPerCta;
    const int64_t left = k - t0;
    const int nrows = left < kRowsPerCta ? (int)left : kRowsPerCta;
    const int total = nrows * cpr;
    const T* sh = src + (int64_t)(h / group) * stride_src;
    T* dh = dst + (int64_t)h * stride_dst;
    const int32_t* Ih = I + (int64_t)h * I_stride + t0;
    for (int base = threadIdx.x; base < total; base += U * 256) {
        uint4 v[U];
        int64_t out[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int idx = base + u * 256;
            out[u] = -1;
            if (idx < total) {
                const int r = idx / cpr;
                const int c = idx - r * cpr;
                int64_t j = __ldg(Ih + r);
                j = j < 0 ? 0 : (j >= d ? d - 1 : j);
                v[u] = __ldg(reinterpret_cast<const uint4*>(sh + j * ld_src) + c);
                out[u] = (t0 + r) * ld_dst + (int64_t)c * V;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (out[u] >= 0) *reinterpret_cast<uint4*>(dh + out[u]) = v[u];
    }
}

template <typename T>
__global__ void __launch_bounds__(256) pack_rows_kernel(
    const T* __restrict__ src, int64_t d, int64_t cols, int64_t ld_src, int64_t stride_src, int group,
    const int32_t* __restrict__ I, int64_t I_stride, int64_t k, T* __restrict__ dst, int64_t ld_dst,
    int64_t stride_dst) {
    pdl_wait();
    pdl_trigger();
    pack_rows_block(src, d, cols, ld_src, stride_src, group, I, I_stride, k, dst, ld_dst, stride_dst, blockIdx.x,
                    (int)blockIdx.y);
}

// Both staging copies of an op in one launch: the CTAs of pack_kernel's grid
// (A[:, I]) first, then those of pack_rows_kernel's grid (B[I, :]), over one
// 1-D grid.  The A gather runs while the score pass's reads of A may still sit
// in L2, and the row copy's first CTAs fill the SMs that the gather's last wave
// leaves idle, where a second launch would wait for the whole gather to end.
// At this kernel's register count (3 CTAs per SM, against 8 for the lone row
// copy) each row-copy thread keeps eight 16-byte loads in flight.
template <typename T>
__global__ void __launch_bounds__(256, 3) pack_ab_kernel(PackArgs a, PackArgs b, int64_t a_x, int64_t a_y, int64_t n_a,
                                                         int64_t b_x) {
    pdl_wait();
    pdl_trigger();
    const int64_t i = blockIdx.x;
    if (i < n_a) {
        const int64_t x = i % a_x, yz = i / a_x;
        pack_block((const T*)a.src, a.rows, a.d, a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (T*)a.dst,
                   a.ld_dst, a.stride_dst, x, yz % a_y, (int)(yz / a_y));
    } else {
        const int64_t j = i - n_a;
        pack_rows_block<T, 8>((const T*)b.src, b.d, b.rows, b.ld_src, b.stride_src, b.group, b.I, b.I_stride, b.k,
                              (T*)b.dst, b.ld_dst, b.stride_dst, j % b_x, (int)(j / b_x));
    }
}

// Rows of B with the unkept ones zeroed, per query head: dst[h][t][:] =
// src[h / group][t][:] if t is in I[h] (ascending, unique) else 0, for t <
// rows_out (rows t >= d are zero).  grid (ceil(rows_out / 64), heads).  An
// ascending set of unique indices in [0, d) has I[t] in [t, t + d - k], so the
// indices that fall in rows [r0, r0 + 64) sit at positions [r0 - (d - k),
// r0 + 64): the CTA scans that window with coalesced loads, marks its kept
// rows, and reads only those.
constexpr int kMaskRows = 64;

template <typename T>
__global__ void __launch_bounds__(256) mask_rows_kernel(
    const T* __restrict__ src, int64_t d, int64_t cols, int64_t ld_src, int64_t stride_src, int group,
    const int32_t* __restrict__ I, int64_t I_stride, int64_t k, T* __restrict__ dst, int64_t ld_dst,
    int64_t stride_dst, int64_t rows_out, uint8_t* __restrict__ block_any) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = 16 / sizeof(T);
    __shared__ int keep[kMaskRows];
    const int h = blockIdx.y;
    const int64_t r0 = (int64_t)blockIdx.x * kMaskRows;
    const int32_t* Ih = I + (int64_t)h * I_stride;
    if (threadIdx.x < kMaskRows) keep[threadIdx.x] = 0;
    __syncthreads();
    const int64_t t_beg = r0 - (d - k) > 0 ? r0 - (d - k) : 0;
    const int64_t t_end = r0 + kMaskRows < k ? r0 + kMaskRows : k;
    for (int64_t t = t_beg + threadIdx.x; t < t_end; t += 256) {
        const int64_t j = __ldg(Ih + t);
        if (j >= r0 && j < r0 + kMaskRows && j < d) keep[j - r0] = 1;
    }
    __syncthreads();
    // whether any row of this block is kept (the product skips blocks with none)
    const int any = __syncthreads_or(threadIdx.x < kMaskRows ? keep[threadIdx.x] : 0);
    if (block_any && threadIdx.x == 0) block_any[(int64_t)h * gridDim.x + blockIdx.x] = any ? 1 : 0;
    const int cpr = (int)(cols / V);
    const int64_t left = rows_out - r0;
    const int nrows = left < kMaskRows ? (int)left : kMaskRows;
    const T* sh = src + (int64_t)(h / group) * stride_src;
    T* dh = dst + (int64_t)h * stride_dst;
    for (int idx = threadIdx.x; idx < nrows * cpr; idx += 256) {
        const int r = idx / cpr;
        const int c = idx - r * cpr;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (keep[r]) v = __ldg(reinterpret_cast<const uint4*>(sh + (r0 + r) * ld_src) + c);
        *reinterpret_cast<uint4*>(dh + (r0 + r) * ld_dst + (int64_t)c * V) = v;
    }
}

// Narrow variant (packed width <= kNarrowMax, e.g. attention heads with
// d_h = 128): the CTA caches the head's indices in shared memory once and its
// threads walk (row, 8-column chunk) pairs, so every thread has work.
constexpr int kNarrowMax = 1024;
constexpr int kNarrowRows = 64;

template <typename T>
__global__ void __launch_bounds__(256) pack_narrow_kernel(
    const T* __restrict__ src, int64_t rows, int64_t d, int64_t ld_src, int64_t stride_src, int group,
    const int32_t* __restrict__ I, int64_t I_stride, int64_t k, T* __restrict__ dst, int64_t ld_dst,
    int64_t stride_dst) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t sidx[kNarrowMax];
    const int h = blockIdx.y;
    const int cpr = (int)(ld_dst / 8);
    for (int t = threadIdx.x; t < (int)ld_dst; t += 256) {
        int32_t j = t < k ? __ldg(I + (int64_t)h * I_stride + t) : -1;
        sidx[t] = j < 0 ? -1 : (j >= d ? (int32_t)(d - 1) : j);
    }
    __syncthreads();
    const int64_t r0 = (int64_t)blockIdx.x * kNarrowRows;
    const int nr = (int)min((int64_t)kNarrowRows, rows - r0);
    const T* sh = src + (int64_t)(h / group) * stride_src;
    T* dh = dst + (int64_t)h * stride_dst;
    for (int e = threadIdx.x; e < nr * cpr; e += 256) {
        const int r = e / cpr, c = e - r * cpr;
        const T* srow = sh + (r0 + r) * ld_src;
        __align__(16) T vals[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int32_t j = sidx[8 * c + v];
            vals[v] = j >= 0 ? srow[j] : T(0.f);
        }
        T* o = dh + (r0 + r) * ld_dst + 8 * c;
        if constexpr (sizeof(T) == 1) {
            *reinterpret_cast<uint2*>(o) = *reinterpret_cast<const uint2*>(vals);
        } else if constexpr (sizeof(T) == 2) {
            *reinterpret_cast<uint4*>(o) = *reinterpret_cast<const uint4*>(vals);
        } else {
            reinterpret_cast<uint4*>(o)[0] = reinterpret_cast<const uint4*>(vals)[0];
            reinterpret_cast<uint4*>(o)[1] = reinterpret_cast<const uint4*>(vals)[1];
        }
    }
}

// grid (ceil(rows / 64), heads), 256 threads: the head's index set becomes a
// bit mask in shared memory; each thread copies 16-byte groups of a row,
// zeroing the columns that are not kept.
template <typename T>
__global__ void __launch_bounds__(256) mask_columns_kernel(const T* __restrict__ src, int64_t rows, int64_t d,
                                                           int64_t ld_src, int64_t stride_src,
                                                           const int32_t* __restrict__ I, int64_t I_stride,
                                                           int64_t k, T* __restrict__ dst, int64_t ld_dst,
                                                           int64_t stride_dst) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = 16 / sizeof(T);
    __shared__ uint32_t keep[kNarrowMax / 32];
    const int h = blockIdx.y;
    for (int w = threadIdx.x; w < kNarrowMax / 32; w += 256) keep[w] = 0u;
    __syncthreads();
    for (int64_t t = threadIdx.x; t < k; t += 256) {
        const int32_t j = __ldg(I + (int64_t)h * I_stride + t);
        if (j >= 0 && j < d) atomicOr(&keep[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    const int cpr = (int)(d / V);
    const int64_t r0 = (int64_t)blockIdx.x * 64;
    const int nr = (int)(rows - r0 < 64 ? rows - r0 : 64);
    const T* sh = src + (int64_t)h * stride_src;
    T* dh = dst + (int64_t)h * stride_dst;
    for (int e = threadIdx.x; e < nr * cpr; e += 256) {
        const int r = e / cpr, c = e - r * cpr;
        uint4 v = __ldg(reinterpret_cast<const uint4*>(sh + (r0 + r) * ld_src) + c);
        T* vals = reinterpret_cast<T*>(&v);
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int j = c * V + u;
            if (!((keep[j >> 5] >> (j & 31)) & 1u)) vals[u] = T(0.f);
        }
        reinterpret_cast<uint4*>(dh + (r0 + r) * ld_dst)[c] = v;
    }
}

}  // namespace

cudaError_t launch_mask_columns(const PackArgs& a, cudaStream_t s) {
    if (a.d > kNarrowMax) return cudaErrorInvalidValue;
    dim3 g((unsigned)((a.rows + 63) / 64), (unsigned)a.heads);
    if (g.x == 0) return cudaSuccess;
    if (a.dtype == 1)
        return launch_pdl(mask_columns_kernel<float>, g, dim3(256), 0, s, (const float*)a.src, a.rows, a.d, a.ld_src,
                          a.stride_src, a.I, a.I_stride, a.k, (float*)a.dst, a.ld_dst, a.stride_dst);
    return launch_pdl(mask_columns_kernel<__nv_bfloat16>, g, dim3(256), 0, s, (const __nv_bfloat16*)a.src, a.rows,
                      a.d, a.ld_src, a.stride_src, a.I, a.I_stride, a.k, (__nv_bfloat16*)a.dst, a.ld_dst,
                      a.stride_dst);
}

cudaError_t launch_pack_rows(const PackArgs& a, cudaStream_t s) {
    if (a.k == 0 || a.rows == 0) return cudaSuccess;
    dim3 grid((unsigned)((a.k + kRowsPerCta - 1) / kRowsPerCta), (unsigned)a.heads);
    if (a.dtype == 2)
        return launch_pdl(pack_rows_kernel<__nv_fp8_e4m3>, grid, dim3(256), 0, s, (const __nv_fp8_e4m3*)a.src, a.d,
                          a.rows, a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (__nv_fp8_e4m3*)a.dst,
                          a.ld_dst, a.stride_dst);
    if (a.dtype == 1)
        return launch_pdl(pack_rows_kernel<float>, grid, dim3(256), 0, s, (const float*)a.src, a.d, a.rows, a.ld_src,
                          a.stride_src, a.group, a.I, a.I_stride, a.k, (float*)a.dst, a.ld_dst, a.stride_dst);
    return launch_pdl(pack_rows_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, (const __nv_bfloat16*)a.src, a.d,
                      a.rows, a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (__nv_bfloat16*)a.dst,
                      a.ld_dst, a.stride_dst);
}

bool pack_ab_one_launch(int dtype, int64_t ld_a) { return (dtype == 0 || dtype == 2) && ld_a > kNarrowMax; }

cudaError_t launch_pack_ab(const PackArgs& a, const PackArgs& b, cudaStream_t s) {
    if (!pack_ab_one_launch(a.dtype, a.ld_dst) || b.dtype != a.dtype) return cudaErrorInvalidValue;
    const int64_t a_x = (a.ld_dst + 8 * kPackThreads - 1) / (8 * kPackThreads);
    const int64_t a_y = (a.rows + kPackRows - 1) / kPackRows;
    const int64_t n_a = a_x * a_y * a.heads;
    const int64_t b_x = (b.k + kRowsPerCta - 1) / kRowsPerCta;
    const int64_t n_b = b.rows == 0 ? 0 : b_x * b.heads;
    const int64_t total = n_a + n_b;
    if (total == 0) return cudaSuccess;
    if (total > 0x7fffffff) return cudaErrorInvalidValue;
    if (a.dtype == 2)
        return launch_pdl(pack_ab_kernel<__nv_fp8_e4m3>, dim3((unsigned)total), dim3(256), 0, s, a, b, a_x, a_y,
                          n_a, b_x);
    return launch_pdl(pack_ab_kernel<__nv_bfloat16>, dim3((unsigned)total), dim3(256), 0, s, a, b, a_x, a_y, n_a,
                      b_x);
}

cudaError_t launch_mask_rows(const PackArgs& a, int64_t rows_out, cudaStream_t s, uint8_t* block_any) {
    dim3 grid((unsigned)((rows_out + kMaskRows - 1) / kMaskRows), (unsigned)a.heads);
    if (grid.x == 0 || a.rows == 0) return cudaSuccess;
    if (a.dtype == 1)
        return launch_pdl(mask_rows_kernel<float>, grid, dim3(256), 0, s, (const float*)a.src, a.d, a.rows, a.ld_src,
                          a.stride_src, a.group, a.I, a.I_stride, a.k, (float*)a.dst, a.ld_dst, a.stride_dst,
                          rows_out, block_any);
    return launch_pdl(mask_rows_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, (const __nv_bfloat16*)a.src, a.d,
                      a.rows, a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (__nv_bfloat16*)a.dst,
                      a.ld_dst, a.stride_dst, rows_out, block_any);
}

cudaError_t launch_pack_rows_transposed(const PackArgs& a, cudaStream_t s) {
    // a.rows = columns of the source (m), a.d = rows of the source, a.I may be null (identity)
    dim3 grid((unsigned)((a.ld_dst + 31) / 32), (unsigned)((a.rows + 31) / 32), (unsigned)a.heads);
    if (grid.y == 0) return cudaSuccess;
    if (a.dtype == 1)
        return launch_pdl(pack_rows_transposed_kernel<float>, grid, dim3(256), 0, s, (const float*)a.src, a.d,
                          a.rows, a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (float*)a.dst, a.ld_dst,
                          a.stride_dst);
    return launch_pdl(pack_rows_transposed_kernel<__nv_bfloat16>, grid, dim3(256), 0, s,
                      (const __nv_bfloat16*)a.src, a.d, a.rows, a.ld_src, a.stride_src, a.group, a.I, a.I_stride,
                      a.k, (__nv_bfloat16*)a.dst, a.ld_dst, a.stride_dst);
}

cudaError_t launch_pack(const PackArgs& a, cudaStream_t s) {
    using F8 = __nv_fp8_e4m3;
    if (a.ld_dst <= kNarrowMax) {
        dim3 g((unsigned)((a.rows + kNarrowRows - 1) / kNarrowRows), (unsigned)a.heads);
        if (g.x == 0) return cudaSuccess;
        if (a.dtype == 2)
            return launch_pdl(pack_narrow_kernel<F8>, g, dim3(256), 0, s, (const F8*)a.src, a.rows, a.d, a.ld_src,
                              a.stride_src, a.group, a.I, a.I_stride, a.k, (F8*)a.dst, a.ld_dst, a.stride_dst);
        if (a.dtype == 1)
            return launch_pdl(pack_narrow_kernel<float>, g, dim3(256), 0, s, (const float*)a.src, a.rows, a.d,
                              a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (float*)a.dst, a.ld_dst,
                              a.stride_dst);
        return launch_pdl(pack_narrow_kernel<__nv_bfloat16>, g, dim3(256), 0, s, (const __nv_bfloat16*)a.src, a.rows,
                          a.d, a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (__nv_bfloat16*)a.dst,
                          a.ld_dst, a.stride_dst);
    }
    dim3 grid((unsigned)((a.ld_dst + 8 * kPackThreads - 1) / (8 * kPackThreads)),
              (unsigned)((a.rows + kPackRows - 1) / kPackRows), (unsigned)a.heads);
    if (grid.y == 0) return cudaSuccess;
    if (a.dtype == 2)
        return launch_pdl(pack_kernel<F8>, grid, dim3(kPackThreads), 0, s, (const F8*)a.src, a.rows, a.d, a.ld_src,
                          a.stride_src, a.group, a.I, a.I_stride, a.k, (F8*)a.dst, a.ld_dst, a.stride_dst);
    if (a.dtype == 1)
        return launch_pdl(pack_kernel<float>, grid, dim3(kPackThreads), 0, s, (const float*)a.src, a.rows, a.d,
                          a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (float*)a.dst, a.ld_dst,
                          a.stride_dst);
    return launch_pdl(pack_kernel<__nv_bfloat16>, grid, dim3(kPackThreads), 0, s, (const __nv_bfloat16*)a.src, a.rows,
                      a.d, a.ld_src, a.stride_src, a.group, a.I, a.I_stride, a.k, (__nv_bfloat16*)a.dst, a.ld_dst,
                      a.stride_dst);
}

}  // namespace rmm
