// rmm_select.cu -- activation-aware index selection of Reduced Matrix
// Multiplication: column scores s_j = ||A[:, j]||_2 and I = TopK(s, k)
// ("Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
// LLM Inference", §3.2 "Activation-aware dimension selection"; the same rule
// per attention head in §3.3).
//
// Scores are kept squared (ordering by s^2 equals ordering by s) in fp32.
// Every column is summed in the same fixed order regardless of its position,
// so equal columns give bit-equal scores and the result does not depend on
// the launch.  Selection compares the fp32 bit patterns (monotone for
// non-negative values) with a 4-pass radix select; among equal scores the
// lower index is kept, and I is written in ascending order.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct Vec16<__nv_fp8_e4m3> {  // 8-bit E4M3 codes, decoded exactly (the low-bit form)
    static constexpr int N = 16;
    __device__ static void load(const __nv_fp8_e4m3* p, float (&x)[16]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 lo(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffffu), __NV_E4M3));
            const __half2 hi(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3));
            const float2 a = __half22float2(lo), b = __half22float2(hi);
            x[4 * i] = a.x;
            x[4 * i + 1] = a.y;
            x[4 * i + 2] = b.x;
            x[4 * i + 3] = b.y;
        }
    }
};
template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ static void load(const float* p, float (&x)[4]) {
        const float4 u = __ldg(reinterpret_cast<const float4*>(p));
        x[0] = u.x;
        x[1] = u.y;
        x[2] = u.z;
        x[3] = u.w;
    }
};

// ------------------------------------------------------------------ colnorm
// grid (ceil(d / (32*V)), nsplit, heads), 16 warps.  Warp w of split s sums
// rows r0+w, r0+w+16, ... of its 32*V columns in increasing row order (eight
// independent 16-byte loads in flight per thread); the 16 warp partials are
// added in warp order and written as the split's partial.  The last CTA of a
// column block to finish (device-scope counter) adds the nsplit partials of
// its columns in split order and writes the final fp32 scores, then resets
// the counter for the next call.  The order of every sum is fixed and the
// same for every column.
constexpr int kMaxSplit = 64;

constexpr int kColWarps = 16;

template <typename T>
__global__ void __launch_bounds__(32 * kColWarps) colnorm_kernel(const T* __restrict__ A, int64_t n, int64_t d,
                                                      int64_t lda, int64_t stride_a,
                                                      int64_t rows_per_split, int nsplit,
                                                      float* __restrict__ partials,
                                                      unsigned* __restrict__ counters,
                                                      float* __restrict__ s2, int causal_rows) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = Vec16<T>::N;
    constexpr int COLS = 32 * V;
    constexpr int U = 8;
    constexpr int W = kColWarps;
    __shared__ float red[W][COLS];
    __shared__ bool last;
    const int h = blockIdx.z, split = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t col = (int64_t)blockIdx.x * COLS + lane * V;
    const int64_t r0 = (int64_t)split * rows_per_split;
    const int64_t r1 = min(n, r0 + rows_per_split);
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    if (col < d) {
        const T* base = A + (int64_t)h * stride_a + col;
        int64_t r = r0 + warp;
        // Rows above this column block are zero when A is causal: start at the
        // first row of the warp's class (rows r0 + warp + W j) at or below the
        // block's first column.  Skipped terms are exact zeros, so every sum
        // keeps its value and order.
        const int64_t c0 = (int64_t)blockIdx.x * COLS;
        if (causal_rows && r < c0) r += (c0 - r + W - 1) / W * W;
        for (; r + W * (U - 1) < r1; r += W * U) {
            float x[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u) Vec16<T>::load(base + (r + W * u) * lda, x[u]);
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int v = 0; v < V; ++v) acc[v] = fmaf(x[u][v], x[u][v], acc[v]);
        }
        for (; r < r1; r += W) {
            float x0[V];
            Vec16<T>::load(base + r * lda, x0);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = fmaf(x0[v], x0[v], acc[v]);
        }
    }
#pragma unroll
    for (int v = 0; v < V; ++v) red[warp][lane * V + v] = acc[v];
    __syncthreads();
    for (int c = threadIdx.x; c < COLS; c += 32 * W) {
        float sum = red[0][c];
#pragma unroll
        for (int w = 1; w < W; ++w) sum += red[w][c];
        const int64_t gcol = (int64_t)blockIdx.x * COLS + c;
        if (gcol < d) partials[((int64_t)h * nsplit + split) * d + gcol] = sum;
    }
    // last CTA of this column block: fixed-order sum over the splits
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned* ctr = counters + (int64_t)h * gridDim.x + blockIdx.x;
        last = atomicAdd(ctr, 1u) == (unsigned)(nsplit - 1);
        if (last) *ctr = 0u;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int c = threadIdx.x; c < COLS; c += 32 * W) {
        const int64_t gcol = (int64_t)blockIdx.x * COLS + c;
        if (gcol >= d) continue;
        const float* pc = partials + (int64_t)h * nsplit * d + gcol;
        float sum = 0.f;
        for (int b = 0; b < nsplit; b += 16) {  // 16 independent loads in flight, added in split order
            float v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = b + u < nsplit ? __ldcg(pc + (int64_t)(b + u) * d) : 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (b + u < nsplit) sum = (b + u == 0) ? v[u] : sum + v[u];
        }
        s2[(int64_t)h * d + gcol] = sum;
    }
}

// ------------------------------------------------------------------ TopK core
// Works on keys[0..d) in shared memory (fp32 bit patterns of s^2 >= 0; d a
// multiple of 4, 16-byte aligned) with a 1024-thread block.  Three radix
// passes over bits [31:21], [20:10] and [9:0] find the exact k-th largest key
// T and how many keys equal to T are kept; then the indices are emitted in
// ascending order.  Every pass reads four keys per 16-byte shared load.
constexpr int kSubHist = 4;  // warps w, w+4, ... share a histogram copy: 4x less atomic contention

struct TopkShared {
    uint32_t hist[kSubHist][2048];
    uint32_t warp_tot[32];
    uint32_t prefix;
    uint32_t remaining;
    uint32_t warp_gt[32];
    uint32_t warp_eq[32];
    uint32_t eq_before[32];
    uint32_t sel_before[32];
};

__device__ __forceinline__ void hist_clear(TopkShared& sh) {
    for (int b = threadIdx.x; b < kSubHist * 2048; b += 1024) (&sh.hist[0][0])[b] = 0;
}

__device__ __forceinline__ void hist_add(uint32_t* myhist, uint32_t key, uint32_t mask, uint32_t prefix, int shift,
                                         uint32_t bins) {
    if ((key & mask) == prefix) atomicAdd(&myhist[(key >> shift) & (bins - 1)], 1u);
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += y;
    }
    return v;
}

// first_done: the sub-histograms already hold the first pass over all keys.
// mask_out (or nullptr): bit j of word j / 32 set iff column j is selected,
// for the ceil(d / 32) words that cover [0, d); the emission's ballots over 32
// consecutive columns are these words.
__device__ void radix_select_and_emit(const uint32_t* keys, int64_t d, int64_t k, int32_t* out, TopkShared& sh,
                                      bool first_done, uint32_t* mask_out) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint4* keys4 = reinterpret_cast<const uint4*>(keys);
    const int64_t d4 = d >> 2;
    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);  // bits [31:21], [20:10], [9:0]
        const int nb = pass == 2 ? 1024 : 2048;
        if (pass > 0 || !first_done) {
            hist_clear(sh);
            __syncthreads();
            uint32_t* myhist = sh.hist[warp & (kSubHist - 1)];
            for (int64_t q = tid; q < d4; q += 1024) {
                const uint4 v = keys4[q];
                hist_add(myhist, v.x, mask, prefix, shift, (uint32_t)nb);
                hist_add(myhist, v.y, mask, prefix, shift, (uint32_t)nb);
                hist_add(myhist, v.z, mask, prefix, shift, (uint32_t)nb);
                hist_add(myhist, v.w, mask, prefix, shift, (uint32_t)nb);
            }
            __syncthreads();
        }
        // thread t owns bins nb-1-2t and nb-2-2t: a block scan in descending bin order
        const int b_hi = nb - 1 - 2 * tid, b_lo = b_hi - 1;
        uint32_t c0 = 0, c1 = 0;
#pragma unroll
        for (int c = 0; c < kSubHist; ++c) {
            if (b_hi >= 0) c0 += sh.hist[c][b_hi];
            if (b_lo >= 0) c1 += sh.hist[c][b_lo];
        }
        const uint32_t tot = c0 + c1;
        const uint32_t incl = warp_incl_scan(tot, lane);
        if (lane == 31) sh.warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const uint32_t w = sh.warp_tot[lane];
            sh.warp_tot[lane] = warp_incl_scan(w, lane) - w;  // exclusive prefix of the warp totals
        }
        __syncthreads();
        const uint32_t excl = sh.warp_tot[warp] + incl - tot;
        if (tot > 0 && excl < remaining && remaining <= excl + tot) {
            const bool hi = excl + c0 >= remaining;
            const uint32_t b = (uint32_t)(hi ? b_hi : b_lo);
            sh.prefix = prefix | (b << shift);
            sh.remaining = remaining - (hi ? excl : excl + c0);
        }
        __syncthreads();
        prefix = sh.prefix;
        remaining = sh.remaining;
        mask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    const uint32_t T = prefix;      // the k-th largest key
    const uint32_t r = remaining;   // how many keys equal to T are kept (lowest indices)

    // Each warp owns a contiguous segment (a multiple of 128 keys).  It counts
    // four keys per lane and step, and emits 32 keys per step in order.
    const int64_t seg = ((d + 31) / 32 + 127) / 128 * 128;
    const int64_t beg = (int64_t)warp * seg;
    const int64_t end = min(d, beg + seg);
    uint32_t gt = 0, eq = 0;
    for (int64_t j0 = beg; j0 < end; j0 += 128) {
        const int64_t j = j0 + 4 * lane;
        if (j < end) {  // end is a multiple of 4: all four keys are in range
            const uint4 v = keys4[j >> 2];
            gt += (v.x > T) + (v.y > T) + (v.z > T) + (v.w > T);
            eq += (v.x == T) + (v.y == T) + (v.z == T) + (v.w == T);
        }
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    if (lane == 0) {
        sh.warp_gt[warp] = gt;
        sh.warp_eq[warp] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t e = sh.warp_eq[lane], g = sh.warp_gt[lane];
        const uint32_t eb = warp_incl_scan(e, lane) - e;
        const uint32_t take_eq = eb >= r ? 0u : min(e, r - eb);
        const uint32_t sel = g + take_eq;
        sh.eq_before[lane] = eb;
        sh.sel_before[lane] = warp_incl_scan(sel, lane) - sel;
    }
    __syncthreads();
    uint32_t eq_run = sh.eq_before[warp], sel_run = sh.sel_before[warp];
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int64_t j0 = beg; j0 < end; j0 += 32) {
        const int64_t j = j0 + lane;
        const uint32_t key = j < end ? keys[j] : 0u;
        const bool is_gt = j < end && key > T;
        const bool is_eq = j < end && key == T;
        const unsigned em = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t rank = eq_run + __popc(em & lt_mask);
        const bool sel = is_gt || (is_eq && rank < r);
        const unsigned sm = __ballot_sync(0xffffffffu, sel);
        const uint32_t pos = sel_run + __popc(sm & lt_mask);
        if (sel && pos < (uint32_t)k) out[pos] = (int32_t)j;
        if (mask_out && lane == 0) mask_out[j0 >> 5] = sm;  // j0 is a multiple of 32 below end
        eq_run += __popc(em);
        sel_run += __popc(sm);
    }
}

// ------------------------------------------------------------------ TopK
// One 1024-thread CTA per head on the final scores written by colnorm (d a
// multiple of 4): 16-byte loads, the first radix histogram built on the way
// into shared memory.
__global__ void __launch_bounds__(1024) topk_kernel(const float* __restrict__ scores, int64_t d, int64_t k,
                                                    int32_t* __restrict__ I, uint32_t* __restrict__ mask,
                                                    int64_t mask_words) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t keys[];
    __shared__ TopkShared sh;
    const int h = blockIdx.x;
    const float4* p = reinterpret_cast<const float4*>(scores + (int64_t)h * d);
    uint4* keys4 = reinterpret_cast<uint4*>(keys);
    hist_clear(sh);
    __syncthreads();
    uint32_t* myhist = sh.hist[(threadIdx.x >> 5) & (kSubHist - 1)];
    const int64_t d4 = d >> 2;
    // four independent 16-byte loads in flight per thread (the scores come from L2)
    for (int64_t q0 = threadIdx.x; q0 < d4; q0 += 4 * 1024) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = q0 + u * 1024 < d4 ? __ldcg(p + q0 + u * 1024) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (q0 + u * 1024 < d4) {
                const uint4 w = make_uint4(__float_as_uint(v[u].x), __float_as_uint(v[u].y), __float_as_uint(v[u].z),
                                           __float_as_uint(v[u].w));
                keys4[q0 + u * 1024] = w;
                atomicAdd(&myhist[w.x >> 21], 1u);
                atomicAdd(&myhist[w.y >> 21], 1u);
                atomicAdd(&myhist[w.z >> 21], 1u);
                atomicAdd(&myhist[w.w >> 21], 1u);
            }
    }
    __syncthreads();
    radix_select_and_emit(keys, d, k, I + (int64_t)h * k, sh, true, mask ? mask + h * mask_words : nullptr);
}

// ------------------------------------------------------------------ fused
// One 1024-thread CTA per head.  Threads form RG row groups x (1024/RG)
// column lanes; lane c of group g sums rows g, g+RG, ... of its 16-byte
// column vectors; the RG partials are added in group order.
template <typename T>
__global__ void __launch_bounds__(1024) normselect_kernel(const T* __restrict__ A, int64_t n,
                                                          int64_t d, int64_t lda, int64_t stride_a,
                                                          int rg, int64_t k, int32_t* __restrict__ I,
                                                          float* __restrict__ s2, uint32_t* __restrict__ mask,
                                                          int64_t mask_words) {
    pdl_wait();
    pdl_trigger();
    constexpr int V = Vec16<T>::N;
    extern __shared__ uint32_t smem[];
    uint32_t* keys = smem;                                        // d
    float* red = reinterpret_cast<float*>(smem + ((d + 3) & ~3ll)); // rg x d when rg > 1
    __shared__ TopkShared sh;
    const int h = blockIdx.x;
    const int tpr = 1024 / rg;
    const int g = threadIdx.x / tpr, tl = threadIdx.x % tpr;
    const T* Ah = A + (int64_t)h * stride_a;
    const int64_t dv = d / V;
    for (int64_t cv = tl; cv < dv; cv += tpr) {
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.f;
        int64_t r = g;
        for (; r + 3 * rg < n; r += 4 * rg) {
            float x0[V], x1[V], x2[V], x3[V];
            Vec16<T>::load(Ah + r * lda + cv * V, x0);
            Vec16<T>::load(Ah + (r + rg) * lda + cv * V, x1);
            Vec16<T>::load(Ah + (r + 2 * rg) * lda + cv * V, x2);
            Vec16<T>::load(Ah + (r + 3 * rg) * lda + cv * V, x3);
#pragma unroll
            for (int v = 0; v < V; ++v) {
                acc[v] = fmaf(x0[v], x0[v], acc[v]);
                acc[v] = fmaf(x1[v], x1[v], acc[v]);
                acc[v] = fmaf(x2[v], x2[v], acc[v]);
                acc[v] = fmaf(x3[v], x3[v], acc[v]);
            }
        }
        for (; r < n; r += rg) {
            float x0[V];
            Vec16<T>::load(Ah + r * lda + cv * V, x0);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = fmaf(x0[v], x0[v], acc[v]);
        }
        if (rg == 1) {
#pragma unroll
            for (int v = 0; v < V; ++v) keys[cv * V + v] = __float_as_uint(acc[v]);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) red[(int64_t)g * d + cv * V + v] = acc[v];
        }
    }
    __syncthreads();
    if (rg > 1) {
        for (int64_t j = threadIdx.x; j < d; j += 1024) {
            float s = red[j];
            for (int gg = 1; gg < rg; ++gg) s += red[(int64_t)gg * d + j];
            keys[j] = __float_as_uint(s);
        }
        __syncthreads();
    }
    if (s2) {
        for (int64_t j = threadIdx.x; j < d; j += 1024) s2[(int64_t)h * d + j] = __uint_as_float(keys[j]);
    }
    radix_select_and_emit(keys, d, k, I + (int64_t)h * k, sh, false, mask ? mask + h * mask_words : nullptr);
}

// ------------------------------------------------------------------ few features
// d <= 256 columns and n <= 8 rows per head (attention heads at a decode
// step): one warp per head.  Lane l sums the squares of columns l + 32 j in
// row order (fp32); warp_topk_bits finds the k largest, ties to the lower
// column, and the kept columns are emitted in order from one ballot per 32.
constexpr int kSmallMaxD = 256;
constexpr int kSmallMaxRows = 8;
constexpr int kSmallWarps = 8;

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

// J: 32-column words per head (d <= 32 J)
template <typename T, int J>
__global__ void __launch_bounds__(32 * kSmallWarps) select_small_kernel(const T* __restrict__ A, int64_t n, int64_t d,
                                                                       int64_t lda, int64_t stride_a, int heads,
                                                                       int64_t k, int32_t* __restrict__ I,
                                                                       float* __restrict__ s2, uint32_t* __restrict__ mask,
                                                                       int64_t mask_words) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = blockIdx.x * kSmallWarps + warp;
    if (h >= heads) return;  // no block-wide barrier below
    const T* Ah = A + (int64_t)h * stride_a;
    uint32_t key[J];
    bool valid[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int f = lane + 32 * j;
        valid[j] = f < d;
        float acc = 0.f;
        if (valid[j]) {
            for (int64_t r = 0; r < n; ++r) {
                const float x = to_float(Ah[r * lda + f]);
                acc = fmaf(x, x, acc);
            }
            if (s2) s2[(int64_t)h * d + f] = acc;
        }
        key[j] = __float_as_uint(acc);
    }
    const uint32_t kept_bits = warp_topk_bits<J>(key, valid, (uint32_t)k, lane);
    int32_t* Ih = I + (int64_t)h * k;
    uint32_t before = 0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int f = lane + 32 * j;
        const bool kept = (kept_bits >> j) & 1u;
        const unsigned b = __ballot_sync(0xffffffffu, kept);
        if (kept) Ih[before + __popc(b & ((1u << lane) - 1u))] = f;
        if (mask && lane == 0 && 32 * j < d) mask[(int64_t)h * mask_words + j] = b;
        before += __popc(b);
    }
}

// ------------------------------------------------------------------ QK select + mask
// One launch for the QK op's feature selection and its masked copy of Q
// (d <= 256): grid (cluster, heads), a cluster of C CTAs per query head, CTA
// c owning rows [c R, (c + 1) R).  Thread t sums the squares of the 8
// features of 16-byte column group t mod (d / 8) over rows t div (d / 8),
// + G, ... in row order (G row groups); the row groups are added in order
// in shared memory; the cluster's first CTA adds the C CTAs' sums in rank
// order through distributed shared memory (the same order for every call),
// one warp takes the TopK with warp_topk_bits, writes I and stores the
// kept-feature words into every CTA of the cluster; after a second cluster
// barrier each CTA writes its rows of Q with the unkept features set to +0.
constexpr int kQkThreads = 256;

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// (ordered after the cluster barrier by the barrier's own "memory" clobber)
__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr));
    return v;
}

__device__ __forceinline__ void st_dsmem_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

template <int J>  // d <= 32 J
__global__ void __launch_bounds__(kQkThreads, 1) qk_select_mask_kernel(
    const __nv_bfloat16* __restrict__ Q, int64_t n, int64_t d, int64_t ldq, int64_t stride_q, int64_t k,
    int32_t* __restrict__ I, __nv_bfloat16* __restrict__ Qm, int64_t ldm, int64_t stride_m, int64_t rows_per_cta) {
    __shared__ float red[kQkThreads * 8];  // [row group][feature]
    __shared__ float part[32 * J];         // this CTA's feature sums
    __shared__ uint32_t keepw[J];          // kept-feature words, from the cluster's first CTA
    pdl_wait();
    pdl_trigger();
    const uint32_t rank = cluster_ctarank(), csize = cluster_nctarank();
    const int h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = (int)(d / 8);           // 16-byte column groups per row
    const int groups = kQkThreads / cg;    // row groups
    const int c = tid % cg, g = tid / cg;
    const int64_t r0 = (int64_t)rank * rows_per_cta;
    const int64_t r1 = min(n, r0 + rows_per_cta);
    const __nv_bfloat16* Qh = Q + (int64_t)h * stride_q;
    float acc[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[v] = 0.f;
    if (g < groups) {
        const __nv_bfloat16* base = Qh + c * 8;
        int64_t r = r0 + g;
        for (; r + 7 * groups < r1; r += 8 * groups) {  // eight rows in flight, added in row order
            uint4 q[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) q[u] = __ldg(reinterpret_cast<const uint4*>(base + (r + u * groups) * ldq));
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float x = __uint_as_float((v & 1) ? (w[v >> 1] & 0xffff0000u) : (w[v >> 1] << 16));
                    acc[v] = fmaf(x, x, acc[v]);
                }
            }
        }
        for (; r < r1; r += groups) {
            const uint4 q = __ldg(reinterpret_cast<const uint4*>(base + r * ldq));
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const float x = __uint_as_float((v & 1) ? (w[v >> 1] & 0xffff0000u) : (w[v >> 1] << 16));
                acc[v] = fmaf(x, x, acc[v]);
            }
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) red[g * d + c * 8 + v] = acc[v];
    }
    __syncthreads();
    for (int f = tid; f < d; f += kQkThreads) {
        float sum = red[f];
        for (int gg = 1; gg < groups; ++gg) sum += red[gg * d + f];
        part[f] = sum;
    }
    cluster_sync_all();  // every CTA's sums are complete and visible to the cluster
    if (rank == 0 && warp == 0) {
        uint32_t key[J];
        bool valid[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int f = lane + 32 * j;
            valid[j] = f < d;
            float sum = 0.f;
            if (valid[j]) {
                // the C sums loaded together, then added in rank order
                const uint32_t a = smem_u32(&part[f]);
                float v[8];
#pragma unroll
                for (int cr = 0; cr < 8; ++cr) v[cr] = cr < (int)csize ? ld_dsmem_f32(mapa_shared(a, (uint32_t)cr)) : 0.f;
#pragma unroll
                for (int cr = 0; cr < 8; ++cr) sum += v[cr];  // +0 past the cluster's size
            }
            key[j] = __float_as_uint(sum);
        }
        const uint32_t kept_bits = warp_topk_bits<J>(key, valid, (uint32_t)k, lane);
        int32_t* Ih = I + (int64_t)h * k;
        uint32_t before = 0;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const bool kept = (kept_bits >> j) & 1u;
            const unsigned b = __ballot_sync(0xffffffffu, kept);
            if (kept) Ih[before + __popc(b & ((1u << lane) - 1u))] = lane + 32 * j;
            before += __popc(b);
            if (lane < (int)csize) st_dsmem_u32(mapa_shared(smem_u32(&keepw[j]), (uint32_t)lane), b);
        }
    }
    cluster_sync_all();  // the kept-feature words are in every CTA of the cluster
    if (g >= groups) return;
    // this thread's column group, as in the sums: the AND masks of its 8 features
    const uint32_t bits = (keepw[c >> 2] >> ((c & 3) * 8)) & 0xffu;  // features 8 c .. 8 c + 7
    uint32_t am[4];
#pragma unroll
    for (int v = 0; v < 4; ++v)
        am[v] = ((bits >> (2 * v)) & 1u ? 0x0000ffffu : 0u) | ((bits >> (2 * v + 1)) & 1u ? 0xffff0000u : 0u);
    const __nv_bfloat16* src = Qh + c * 8;
    __nv_bfloat16* dst = Qm + (int64_t)h * stride_m + c * 8;
    int64_t r = r0 + g;
    for (; r + 3 * groups < r1; r += 4 * groups) {  // four rows in flight
        uint4 q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) q[u] = __ldg(reinterpret_cast<const uint4*>(src + (r + u * groups) * ldq));
#pragma unroll
        for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(dst + (r + u * groups) * ldm) =
                make_uint4(q[u].x & am[0], q[u].y & am[1], q[u].z & am[2], q[u].w & am[3]);
    }
    for (; r < r1; r += groups) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(src + r * ldq));
        *reinterpret_cast<uint4*>(dst + r * ldm) = make_uint4(q.x & am[0], q.y & am[1], q.z & am[2], q.w & am[3]);
    }
}

// ------------------------------------------------------------------ one row
// n = 1, bf16: column j's score is a_j^2, exact in fp32, so two scores are
// equal exactly when |a_j| are, and they order as |a_j| does, i.e. as the 15
// low bits of a_j's bf16 encoding (for NaN and infinity too).  The TopK is
// then a two-digit radix select over those keys: counts of the high 8 bits
// find the bin holding the k-th largest key, counts of the low 7 bits among
// that bin's keys find the key T itself, and the kept columns (above T, then
// the lowest-indexed keys equal to T) are emitted in order.  A cluster of C
// CTAs per head splits the row into C ranges of whole 256-key steps; the
// CTAs add their counts in rank order through distributed shared memory
// (every CTA finds the same T) and exchange their kept counts to place their
// output.  256 threads, four CTAs per SM; each pass reads the CTA's range
// again (from L2).
constexpr int kRowThreads = 256;
constexpr int kRowWarps = kRowThreads / 32;

__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr));
    return v;
}

__global__ void __launch_bounds__(kRowThreads, 4) select16_kernel(const __nv_bfloat16* __restrict__ A, int64_t d,
                                                               int64_t stride_a, int64_t k,
                                                               int32_t* __restrict__ I, float* __restrict__ s2,
                                                               uint32_t* __restrict__ mask, int64_t mask_words,
                                                               int64_t seg) {
    __shared__ uint32_t hist[kRowWarps][256];  // per-warp counts; later each warp's staged indices
    __shared__ uint32_t tot1[256], tot2[128];  // this CTA's counts: high 8 bits, then low 7 bits in the bin
    __shared__ uint32_t scan_part[kRowWarps];
    __shared__ uint32_t s_bin, s_above;
    __shared__ uint32_t cta_cnt[2];            // this CTA's keys above T and equal to T
    __shared__ uint32_t warp_gt[kRowWarps], warp_eq[kRowWarps], eq_before[kRowWarps], sel_before[kRowWarps];
    pdl_wait();
    pdl_trigger();
    const uint32_t rank = cluster_ctarank(), C = cluster_nctarank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y;
    const uint16_t* a = reinterpret_cast<const uint16_t*>(A + (int64_t)h * stride_a);
    const int64_t c0 = min(d, (int64_t)rank * seg), c1 = min(d, c0 + seg);  // this CTA's keys (multiples of 8)
    const uint4* a4 = reinterpret_cast<const uint4*>(a);

    // Warp w owns a segment of whole 256-key steps of the CTA's range, the
    // same in every pass, so that its counts also place its output.
    const int64_t steps = (c1 - c0 + 255) / 256;
    const int64_t wseg = (steps + kRowWarps - 1) / kRowWarps * 256;
    const int64_t beg = min(c1, c0 + (int64_t)warp * wseg);
    const int64_t end = min(c1, beg + wseg);
    // counts of bin_of(key) over the warp's keys into its histogram (bin -1:
    // not counted; four 16-byte loads in flight per lane), then summed over
    // the warps into tot[0, bins)
    auto count = [&](int bins, uint32_t* tot, auto bin_of) {
        for (int i = tid; i < kRowWarps * 256; i += kRowThreads) (&hist[0][0])[i] = 0u;
        __syncthreads();
        for (int64_t q0 = beg / 8 + lane; q0 < end / 8; q0 += 4 * 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = q0 + u * 32 < end / 8 ? __ldg(a4 + q0 + u * 32) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (q0 + u * 32 >= end / 8) break;
                const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const int b = bin_of((w4[x >> 1] >> (16 * (x & 1))) & 0x7fffu);
                    if (b >= 0) atomicAdd(&hist[warp][b], 1u);
                }
            }
        }
        __syncthreads();
        for (int b = tid; b < bins; b += kRowThreads) {
            uint32_t sum = 0;
#pragma unroll
            for (int w = 0; w < kRowWarps; ++w) sum += hist[w][b];
            tot[b] = sum;
        }
    };
    // the warp's keys in bins above b0 (and, with eq, the count of bin b0)
    auto warp_above = [&](int bins, uint32_t b0) {
        uint32_t c = 0;
        for (int b = lane; b < bins; b += 32) c += (uint32_t)b > b0 ? hist[warp][b] : 0u;
        return __reduce_add_sync(0xffffffffu, c);
    };
    // the cluster's count of bin b (thread t takes bin bins - 1 - t), the CTAs
    // added in rank order; then the largest bin B with above0 + (keys in bins
    // >= B) >= k: s_bin = B, s_above = above0 + keys in bins > B
    auto find_bin = [&](int bins, const uint32_t* tot, uint32_t above0) {
        const int b = bins - 1 - tid;
        uint32_t g = 0;
        if (tid < bins) {
            const uint32_t addr = smem_u32(&tot[b]);
            for (uint32_t cr = 0; cr < C; ++cr) g += ld_dsmem_u32(mapa_shared(addr, cr));
        }
        const uint32_t incl = warp_incl_scan(g, lane);
        if (lane == 31) scan_part[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const uint32_t v = lane < kRowWarps ? scan_part[lane] : 0u;
            const uint32_t pi = warp_incl_scan(v, lane);
            if (lane < kRowWarps) scan_part[lane] = pi - v;
        }
        __syncthreads();
        const uint32_t upto = above0 + scan_part[warp] + incl;  // keys in bins >= b
        if (tid < bins && upto >= (uint32_t)k && upto - g < (uint32_t)k) {
            s_bin = (uint32_t)b;
            s_above = upto - g;
        }
        __syncthreads();
    };

    count(256, tot1, [](uint32_t key) { return (int)(key >> 7); });
    cluster_sync_all();  // every CTA's high-digit counts are complete
    find_bin(256, tot1, 0u);
    const uint32_t B1 = s_bin, above1 = s_above;
    const uint32_t gt_hi = warp_above(256, B1);  // this warp's keys in higher bins
    count(128, tot2, [B1](uint32_t key) { return (key >> 7) == B1 ? (int)(key & 127u) : -1; });
    cluster_sync_all();  // every CTA's low-digit counts are complete
    find_bin(128, tot2, above1);
    const uint32_t B2 = s_bin;
    const uint32_t T = (B1 << 7) | B2, r = (uint32_t)k - s_above;  // the k-th largest key; its ties kept
    // this warp's keys above T and equal to T, from its histograms
    const uint32_t gt_w = gt_hi + warp_above(128, B2), eq_w = hist[warp][B2];

    // Emission.  In a 256-key step of its segment lane l holds keys [8l, 8l + 8)
    // from one 16-byte load (d is a multiple of 8, so a lane's keys are all in
    // range or all out).  Per lane, bit x of g / e marks key x above / equal
    // to T; warp prefix sums place them, the warps' and the earlier CTAs'
    // totals place the warp.
    auto bits_of = [&](const uint4& v, uint32_t& g, uint32_t& e) {
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        g = 0u;
        e = 0u;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t k0 = w4[u] & 0x7fffu, k1 = (w4[u] >> 16) & 0x7fffu;
            g |= (uint32_t)(k0 > T) << (2 * u) | (uint32_t)(k1 > T) << (2 * u + 1);
            e |= (uint32_t)(k0 == T) << (2 * u) | (uint32_t)(k1 == T) << (2 * u + 1);
        }
    };
    if (lane == 0) {
        warp_gt[warp] = gt_w;
        warp_eq[warp] = eq_w;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t g = 0, e = 0;
        for (int w = 0; w < kRowWarps; ++w) {
            g += warp_gt[w];
            e += warp_eq[w];
        }
        cta_cnt[0] = g;
        cta_cnt[1] = e;
    }
    cluster_sync_all();  // every CTA's kept counts are complete
    if (warp == 0) {
        // the ties and the kept columns of the CTAs before this one, in rank order
        const bool before = lane < (int)rank;
        const uint32_t ga = before ? ld_dsmem_u32(mapa_shared(smem_u32(&cta_cnt[0]), (uint32_t)lane)) : 0u;
        const uint32_t ea = before ? ld_dsmem_u32(mapa_shared(smem_u32(&cta_cnt[1]), (uint32_t)lane)) : 0u;
        const uint32_t eb = warp_incl_scan(ea, lane) - ea;
        const uint32_t take = eb >= r ? 0u : min(ea, r - eb);
        const uint32_t eq_cta = __reduce_add_sync(0xffffffffu, ea);
        const uint32_t sel_cta = __reduce_add_sync(0xffffffffu, ga + take);
        // then this CTA's warps, in warp order
        const uint32_t e = lane < kRowWarps ? warp_eq[lane] : 0u;
        const uint32_t g = lane < kRowWarps ? warp_gt[lane] : 0u;
        const uint32_t ewb = eq_cta + warp_incl_scan(e, lane) - e;
        const uint32_t wtake = ewb >= r ? 0u : min(e, r - ewb);
        const uint32_t sel = g + wtake;
        const uint32_t sb = sel_cta + warp_incl_scan(sel, lane) - sel;
        if (lane < kRowWarps) {
            eq_before[lane] = ewb;
            sel_before[lane] = sb;
        }
    }
    cluster_sync_all();  // no CTA reads another's counts after this: each may finish on its own
    uint32_t eq_run = eq_before[warp], sel_run = sel_before[warp];
    int32_t* wbuf = reinterpret_cast<int32_t*>(hist[warp]);  // this warp's staged indices of a step
    int32_t* Ih = I ? I + (int64_t)h * k : nullptr;  // nullptr: only the membership words are wanted
    for (int64_t b0 = beg; b0 < end; b0 += 256) {
        const int64_t j = b0 + 8 * lane;
        const bool in = j < end;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        uint32_t g = 0u, e = 0u;
        if (in) {
            v = __ldg(reinterpret_cast<const uint4*>(a + j));
            bits_of(v, g, e);
        }
        uint32_t sel = g;
        if (__any_sync(0xffffffffu, e != 0u)) {  // ties at T: the lowest indices are kept
            const uint32_t ec = __popc(e);
            const uint32_t ei = warp_incl_scan(ec, lane);
            uint32_t rk = eq_run + ei - ec;
#pragma unroll
            for (int x = 0; x < 8; ++x)
                if ((e >> x) & 1u) {
                    if (rk < r) sel |= 1u << x;
                    ++rk;
                }
            eq_run += __shfl_sync(0xffffffffu, ei, 31);
        }
        if (Ih) {
            const uint32_t sc = __popc(sel);
            const uint32_t si = warp_incl_scan(sc, lane);
            uint32_t pos = si - sc;
#pragma unroll
            for (int x = 0; x < 8; ++x)
                if ((sel >> x) & 1u) wbuf[pos++] = (int32_t)(j + x);
            __syncwarp();
            const uint32_t nsel = __shfl_sync(0xffffffffu, si, 31);
            for (uint32_t x = lane; x < nsel; x += 32) Ih[sel_run + x] = wbuf[x];
            __syncwarp();  // wbuf is refilled by the next step
            sel_run += nsel;
        }
        if (mask) {  // four lanes' 8 bits make one 32-key word
            uint32_t w = sel << (8 * (lane & 3));
            w |= __shfl_xor_sync(0xffffffffu, w, 1);
            w |= __shfl_xor_sync(0xffffffffu, w, 2);
            if (in && (lane & 3) == 0) mask[(int64_t)h * mask_words + (j >> 5)] = w;
        }
        if (s2 && in) {  // s2 is only 4-byte aligned
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            float* dst = s2 + (int64_t)h * d + j;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float x0 = __uint_as_float(w4[u] << 16), x1 = __uint_as_float(w4[u] & 0xffff0000u);
                dst[2 * u] = x0 * x0;
                dst[2 * u + 1] = x1 * x1;
            }
        }
    }
}

__global__ void identity_kernel(int32_t* __restrict__ I, int64_t k, int heads) {
    pdl_wait();
    pdl_trigger();
    const int64_t total = k * heads;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x)
        I[i] = (int32_t)(i % k);
}

int normselect_row_groups(int64_t d, int dtype) {
    const int64_t dv = d / (dtype == 1 ? 4 : 8);
    int rg = 1;
    while (rg * 2 * dv <= 1024 && rg < 1024) rg *= 2;
    return rg;
}

}  // namespace

size_t topk_smem_bytes(int64_t d) { return (size_t)d * 4; }

size_t normselect_smem_bytes(int64_t d, int dtype) {
    const int rg = normselect_row_groups(d, dtype);
    size_t bytes = (size_t)((d + 3) & ~3ll) * 4;
    if (rg > 1) bytes += (size_t)rg * d * 4;
    return bytes;
}

cudaError_t launch_colnorm(const SelectArgs& a, cudaStream_t s) {
    if (a.nsplit < 1 || a.nsplit > kMaxSplit) return cudaErrorInvalidValue;
    const int V = a.dtype == 1 ? 4 : a.dtype == 2 ? 16 : 8;  // elements per 16-byte load
    dim3 grid((unsigned)((a.d + 32 * V - 1) / (32 * V)), (unsigned)a.nsplit, (unsigned)a.heads);
    if (a.dtype == 2)
        return launch_pdl(colnorm_kernel<__nv_fp8_e4m3>, grid, dim3(32 * kColWarps), 0, s,
                          (const __nv_fp8_e4m3*)a.A, a.n, a.d, a.lda, a.stride_a, a.rows_per_split, a.nsplit,
                          a.partials, a.counters, a.scores, a.causal_rows);
    if (a.dtype == 1)
        return launch_pdl(colnorm_kernel<float>, grid, dim3(32 * kColWarps), 0, s, (const float*)a.A, a.n, a.d,
                          a.lda, a.stride_a, a.rows_per_split, a.nsplit, a.partials, a.counters, a.scores,
                          a.causal_rows);
    return launch_pdl(colnorm_kernel<__nv_bfloat16>, grid, dim3(32 * kColWarps), 0, s, (const __nv_bfloat16*)a.A,
                      a.n, a.d, a.lda, a.stride_a, a.rows_per_split, a.nsplit, a.partials, a.counters, a.scores,
                      a.causal_rows);
}

cudaError_t launch_topk(const SelectArgs& a, cudaStream_t s) {
    const size_t smem = topk_smem_bytes(a.d);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_kernel, dim3(a.heads), dim3(1024), smem, s, (const float*)a.scores, a.d, a.k, a.I, a.mask,
                      a.mask_words);
}

cudaError_t launch_normselect(const SelectArgs& a, cudaStream_t s) {
    const int rg = normselect_row_groups(a.d, a.dtype);
    const size_t smem = normselect_smem_bytes(a.d, a.dtype);
    cudaError_t e;
    if (a.dtype == 1) {
        e = cudaFuncSetAttribute(normselect_kernel<float>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(normselect_kernel<float>, dim3(a.heads), dim3(1024), smem, s, (const float*)a.A, a.n, a.d,
                       a.lda, a.stride_a, rg, a.k, a.I, a.s2, a.mask, a.mask_words);
    } else {
        e = cudaFuncSetAttribute(normselect_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(normselect_kernel<__nv_bfloat16>, dim3(a.heads), dim3(1024), smem, s,
                       (const __nv_bfloat16*)a.A, a.n, a.d, a.lda, a.stride_a, rg, a.k, a.I, a.s2, a.mask,
                       a.mask_words);
    }
    return e;
}

bool select_small_fits(int64_t n, int64_t d) { return n >= 1 && n <= kSmallMaxRows && d <= kSmallMaxD; }

template <typename T, int J>
cudaError_t launch_small_j(const SelectArgs& a, cudaStream_t s) {
    const dim3 grid((unsigned)((a.heads + kSmallWarps - 1) / kSmallWarps));
    return launch_pdl(select_small_kernel<T, J>, grid, dim3(32 * kSmallWarps), 0, s, (const T*)a.A, a.n, a.d, a.lda,
                      a.stride_a, a.heads, a.k, a.I, a.s2, a.mask, a.mask_words);
}

template <typename T>
cudaError_t launch_small_t(const SelectArgs& a, cudaStream_t s) {
    if (a.d <= 64) return launch_small_j<T, 2>(a, s);
    if (a.d <= 128) return launch_small_j<T, 4>(a, s);
    return launch_small_j<T, 8>(a, s);
}

cudaError_t launch_select_small(const SelectArgs& a, cudaStream_t s) {
    if (!select_small_fits(a.n, a.d)) return cudaErrorInvalidValue;
    return a.dtype == 1 ? launch_small_t<float>(a, s) : launch_small_t<__nv_bfloat16>(a, s);
}

cudaError_t launch_select16(const SelectArgs& a, cudaStream_t s) {
    if (a.dtype != 0 || a.n != 1 || a.d > 65535 || a.d % 8 != 0 || a.heads < 1 || a.heads > 65535)
        return cudaErrorInvalidValue;
    // CTAs per head: up to 8, while the heads leave room (about four CTAs per
    // SM) and every CTA keeps at least 2048 keys
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return cudaErrorInvalidValue;
    int C = 1;
    while (C < 8 && (int64_t)a.heads * 2 * C <= 4LL * sms && a.d / (2 * C) >= 2048) C *= 2;
    const int64_t seg = ((a.d + C - 1) / C + 255) / 256 * 256;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)a.heads);
    cfg.blockDim = dim3(kRowThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, select16_kernel, (const __nv_bfloat16*)a.A, (int64_t)a.d, (int64_t)a.stride_a,
                              (int64_t)a.k, a.I, a.s2, a.mask, (int64_t)a.mask_words, seg);
}

bool qk_select_mask_fits(int dtype, int64_t d) { return dtype == 0 && d >= 8 && d <= 256 && d % 8 == 0; }

// CTAs per head: about two CTAs per SM over all heads, at least 16 rows each,
// at most 8 (the portable cluster size).
int qk_select_cluster(int64_t heads, int64_t n, int sms) {
    int c = 1;
    while (c < 8 && heads * c < 2LL * sms && n / (2 * c) >= 16) c *= 2;
    return c;
}

template <int J>
cudaError_t launch_qk_select_mask_j(const QkMaskArgs& a, cudaStream_t s) {
    const int64_t rows = (a.n + a.cluster - 1) / a.cluster;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)a.cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.cluster, (unsigned)a.heads);
    cfg.blockDim = dim3(kQkThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, qk_select_mask_kernel<J>, (const __nv_bfloat16*)a.Q, a.n, a.d, a.ldq, a.stride_q,
                              a.k, a.I, (__nv_bfloat16*)a.Qm, a.ldm, a.stride_m, rows);
}

cudaError_t launch_qk_select_mask(const QkMaskArgs& a, cudaStream_t s) {
    if (!qk_select_mask_fits(0, a.d) || a.k < 1 || a.k > a.d || a.n < 1 || a.heads < 1 || a.heads > 65535 ||
        (a.cluster != 1 && a.cluster != 2 && a.cluster != 4 && a.cluster != 8))
        return cudaErrorInvalidValue;
    if (a.d <= 64) return launch_qk_select_mask_j<2>(a, s);
    if (a.d <= 128) return launch_qk_select_mask_j<4>(a, s);
    return launch_qk_select_mask_j<8>(a, s);
}

cudaError_t launch_identity(int32_t* I, int64_t k, int heads, cudaStream_t s) {
    const int64_t total = k * heads;
    const int64_t want = (total + 255) / 256;
    const int blocks = (int)(want < 1024 ? (want > 0 ? want : 1) : 1024);
    return launch_pdl(identity_kernel, dim3(blocks), dim3(256), 0, s, I, k, heads);
}

}  // namespace rmm
