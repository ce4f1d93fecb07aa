// rmm_decode.cu -- attention at a decode step: a few query rows per head
// against t cached keys and values ("Reduced Matrix Multiplication:
// Input-Adaptive Matrix-Product Reduction for LLM Inference", Appendix D.1,
// the decode case: the score product's cost falls from O(tD) to
// O(rho_feat t D), the value product's from O(t d_v) to O(rho_tok t d_v); the
// K cache is still read in full to form the scores).
//
// Both ops take the query heads of one KV head g (h = g * group + hl) and
// their n rows together, qv = hl * n + i < group * n <= 8, so that every K or
// V row is read once per KV head, not once per query head.  Both are bound by
// reading the cache; the contraction per cache row (8 query vectors x d_h or
// d_v) runs on warp-level bf16 MMAs (mma.sync m16n8k16, fp32 accumulation),
// which keep the instructions per 256-byte row at a few where per-lane dot
// products with shuffle reductions would need dozens and leave the SM issue
// bound before HBM is.
//
// qk: S[h][i][j] = alpha * sum_{f in I_h} Q[h][i][f] K[g][j][f].  The query
//   vectors, with the features outside I_h set to zero, are the MMA's 8-column
//   operand; K as stored is the 16-row operand, so the contraction runs over
//   every feature and each zeroed term adds an exact zero.  I_h is selected in
//   the kernel from the query rows it loads (each CTA ranks its group's d_h
//   features; the first CTA of a KV head writes I), unless a given I is passed.
// pv: O[h][i][:] = sum_{t in T_h} P[h][i][t] V[g][t][:].  A CTA takes a range of
//   tokens, forms the union of the group's token sets over it from the
//   selection's membership bits, gathers only those V rows, and weighs row t
//   for query vector qv by P[h][i][t] if t is in T_h, else by zero.  The
//   ranges' fp32 partial sums are added in range order by the last CTA of the
//   KV head (device-scope counter, reset by that CTA), so the result does not
//   depend on timing.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm_internal.h"

namespace rmm {
namespace {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// 16-byte global -> shared copy; src_bytes = 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
// c += a (16 x 16, row) * b (16 x 8, col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(bf16 lo, bf16 hi) {
    return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}
__device__ __forceinline__ uint4 pack8(const float* y) {
    uint4 o;
    o.x = pack_bf16x2(__float2bfloat16_rn(y[0]), __float2bfloat16_rn(y[1]));
    o.y = pack_bf16x2(__float2bfloat16_rn(y[2]), __float2bfloat16_rn(y[3]));
    o.z = pack_bf16x2(__float2bfloat16_rn(y[4]), __float2bfloat16_rn(y[5]));
    o.w = pack_bf16x2(__float2bfloat16_rn(y[6]), __float2bfloat16_rn(y[7]));
    return o;
}

// ------------------------------------------------------------------ qk
// grid (X, kv_heads), 4 warps, persistent: CTA x walks the KV head's ROWS-row
// tiles x, x + X, ... with kQkStages tiles of K in flight, so that loads stay
// in flight across tiles and the query setup is paid once.  Shared memory:
// the K stages [kQkStages][ROWS][D + 8] (rows padded by 16 bytes:
// conflict-free ldmatrix), the 8 masked query vectors [8][D + 8] and the
// score tile [8][ROWS + 4] fp32.
constexpr int kQkStages = 3;
template <int D>
__host__ __device__ constexpr int qk_rows() { return D == 256 ? 64 : 128; }
template <int D>
constexpr size_t qk_smem() {
    return (size_t)(kQkStages * qk_rows<D>() + 8) * (D + 8) * 2 + (size_t)8 * (qk_rows<D>() + 4) * 4;
}

template <int D>
__global__ void __launch_bounds__(128) decode_qk_kernel(const DecodeArgs a) {
    constexpr int ROWS = qk_rows<D>();
    constexpr int CPR = D / 8;      // 16-byte chunks per K row
    constexpr int LDS = D + 8;      // shared row stride (elements)
    constexpr int MT = ROWS / 64;   // 16-row MMA tiles per warp
    constexpr int KS = D / 16;      // MMA k-steps
    extern __shared__ __align__(16) unsigned char dsmem[];
    bf16* ks = reinterpret_cast<bf16*>(dsmem);
    bf16* qs = ks + kQkStages * ROWS * LDS;
    float* ys = reinterpret_cast<float*>(qs + 8 * LDS);
    const int g = blockIdx.y;
    const int64_t tiles = (a.m + ROWS - 1) / ROWS;
    const int qvn = a.group * a.n;
    pdl_wait();
    const bf16* Kg = a.B + (int64_t)g * a.stride_b;
    auto issue = [&](int64_t tile, int stage) {
        bf16* dst = ks + stage * ROWS * LDS;
        const int64_t j0 = tile * ROWS;
        for (int c = threadIdx.x; c < ROWS * CPR; c += 128) {
            const int r = c / CPR, q = c - r * CPR;
            const int64_t j = j0 + r;
            const bool in = j < a.m;
            cp_async16(dst + r * LDS + q * 8, Kg + (in ? j : 0) * a.ldb + q * 8, in ? 16 : 0);
        }
    };
#pragma unroll
    for (int i = 0; i < kQkStages - 1; ++i) {
        const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
        if (tile < tiles) issue(tile, i);
        cp_async_commit();
    }
    pdl_trigger();
    // The query vectors with the features outside I_h zeroed.  One round of
    // loads: the group's query rows into registers and, from I, a flag per
    // kept feature; then the masked tile is written.  (Under a full HBM stream
    // each dependent round trip to L2 lengthens the CTA's life and so cuts the
    // K bytes in flight.)
    constexpr int QPT = 8 * (D / 2) / 128;  // 32-bit words of the 8 vectors per thread
    __shared__ uint8_t kept[8][D];
    for (int e = threadIdx.x; e < 8 * D / 4; e += 128)
        reinterpret_cast<uint32_t*>(&kept[0][0])[e] = a.I ? 0u : 0x01010101u;
    __syncthreads();
    uint32_t qreg[QPT];
#pragma unroll
    for (int j = 0; j < QPT; ++j) {
        const int e = threadIdx.x + j * 128;
        const int qv = e / (D / 2), f = (e - qv * (D / 2)) * 2;
        qreg[j] = 0u;
        if (qv < qvn) {
            const int hl = qv / a.n, i = qv - hl * a.n;
            qreg[j] = *reinterpret_cast<const uint32_t*>(a.A + (int64_t)(g * a.group + hl) * a.stride_a +
                                                         (int64_t)i * a.lda + f);
        }
    }
    // the group's rows of I are consecutive: entry e = hl * k + pos of the group
    // sits at g * group * k + e; group * k <= 8 * D entries, IPT per thread
    constexpr int IPT = 8 * D / 128;
    int32_t fk[IPT];
    const int nI = a.I ? a.group * (int)a.k : 0;
    const int32_t* Ig = a.I ? a.I + (int64_t)g * a.group * a.k : nullptr;
#pragma unroll
    for (int j = 0; j < IPT; ++j) {
        const int e = threadIdx.x + j * 128;
        fk[j] = e < nI ? __ldg(Ig + e) : -1;
    }
#pragma unroll
    for (int j = 0; j < IPT; ++j) {
        const int e = threadIdx.x + j * 128;
        if (e < nI && fk[j] >= 0 && fk[j] < D) kept[e / (int)a.k][fk[j]] = 1;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (a.fused_select) {
        // The selection of each head's k features, in the CTA: the raw query
        // rows go to shared memory, warp w selects the features of heads w,
        // w + 4 (fp32 sums of squares in row order; warp_topk_bits: the k
        // largest, ties to the lower feature) and the first CTA of the KV head
        // writes I in order.
#pragma unroll
        for (int j = 0; j < QPT; ++j) {
            const int e = threadIdx.x + j * 128;
            const int qv = e / (D / 2), f = (e - qv * (D / 2)) * 2;
            *reinterpret_cast<uint32_t*>(qs + qv * LDS + f) = qreg[j];
        }
        __syncthreads();
        constexpr int J = D / 32;
        for (int hl = warp; hl < a.group; hl += 4) {
            uint32_t key[J];
            bool valid[J];
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int f = lane + 32 * j;
                float sc = 0.f;
                for (int i = 0; i < a.n; ++i) {
                    const float x = __bfloat162float(qs[(hl * a.n + i) * LDS + f]);
                    sc = fmaf(x, x, sc);
                }
                key[j] = __float_as_uint(sc);
                valid[j] = true;
            }
            const uint32_t kept_bits = warp_topk_bits<J>(key, valid, (uint32_t)a.k, lane);
            uint32_t before = 0;
            const bool emit = a.I_out && blockIdx.x == 0;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int f = lane + 32 * j;
                const bool kp = (kept_bits >> j) & 1u;
                kept[hl][f] = kp ? 1 : 0;
                if (emit) {
                    const unsigned b = __ballot_sync(0xffffffffu, kp);
                    if (kp) a.I_out[(int64_t)(g * a.group + hl) * a.k + before + __popc(b & ((1u << lane) - 1u))] = f;
                    before += __popc(b);
                }
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < QPT; ++j) {
        const int e = threadIdx.x + j * 128;
        const int qv = e / (D / 2), f = (e - qv * (D / 2)) * 2;
        const int hl = qv < qvn ? qv / a.n : 0;
        const uint32_t lo = kept[hl][f] ? 0x0000ffffu : 0u, hi = kept[hl][f + 1] ? 0xffff0000u : 0u;
        *reinterpret_cast<uint32_t*>(qs + qv * LDS + f) = qreg[j] & (lo | hi);
    }
    __syncthreads();
    uint32_t bq[KS][2];
#pragma unroll
    for (int s = 0; s < KS; ++s) {
        bq[s][0] = *reinterpret_cast<const uint32_t*>(qs + (lane >> 2) * LDS + s * 16 + (lane & 3) * 2);
        bq[s][1] = *reinterpret_cast<const uint32_t*>(qs + (lane >> 2) * LDS + s * 16 + 8 + (lane & 3) * 2);
    }
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {
    const int64_t ahead = tile + (int64_t)(kQkStages - 1) * gridDim.x;
    if (ahead < tiles) issue(ahead, (it + kQkStages - 1) % kQkStages);
    cp_async_commit();
    cp_async_wait<kQkStages - 1>();
    __syncthreads();  // this tile's K is in; the previous tile's scores are stored
    const bf16* kt = ks + (it % kQkStages) * ROWS * LDS;
    const int64_t j0 = tile * ROWS;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int r0 = warp * (ROWS / 4) + mt * 16;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const bf16* arow = kt + (r0 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + (lane >> 4) * 8;
#pragma unroll
        for (int s = 0; s < KS; ++s) {
            uint32_t af[4];
            ldsm_x4(af, arow + s * 16);
            mma_16816(acc, af, bq[s][0], bq[s][1]);
        }
        const int r = r0 + (lane >> 2), qv = (lane & 3) * 2;
        ys[qv * (ROWS + 4) + r] = acc[0] * a.alpha;
        ys[(qv + 1) * (ROWS + 4) + r] = acc[1] * a.alpha;
        ys[qv * (ROWS + 4) + r + 8] = acc[2] * a.alpha;
        ys[(qv + 1) * (ROWS + 4) + r + 8] = acc[3] * a.alpha;
    }
    __syncthreads();  // the scores are in ys; this stage is free for the next issue
    for (int c = threadIdx.x; c < qvn * (ROWS / 8); c += 128) {
        const int qv = c / (ROWS / 8), q = c - qv * (ROWS / 8);
        const int64_t j = j0 + q * 8;
        if (j >= a.m) continue;  // t is a multiple of 8
        const int hl = qv / a.n, i = qv - hl * a.n;
        bf16* out = a.Y + (int64_t)(g * a.group + hl) * a.stride_y + (int64_t)i * a.ldy + j;
        *reinterpret_cast<uint4*>(out) = pack8(ys + qv * (ROWS + 4) + q * 8);
    }
    }
}

// ------------------------------------------------------------------ pv
// grid (ceil(t / a.tokens), kv_heads), 4 warps.  a.tokens (128, 256 or 512)
// tokens per CTA; the union of the group's kept tokens over them is listed in
// shared memory and cut into k-steps of 16 rows, dealt to the warps in turn.
// Each warp stages its steps' V rows with cp.async (kPvStages - 1 steps in
// flight while it multiplies another) and
// accumulates a 16 x DV tile (rows = query vectors, 8 used) over them.
constexpr int kPvMaxTok = 512;
constexpr int kPvStages = 2;
// dynamic shared memory: the per-warp V stages (reused for the warp sums), then
// the staged P rows of the qvn query vectors over a range of `tokens`
template <int DV>
__host__ __device__ constexpr size_t pv_stage_bytes() {
    return (size_t)4 * kPvStages * 16 * (DV + 8) * 2;
}
template <int DV>
size_t pv_smem(int qvn, int tokens) {
    return pv_stage_bytes<DV>() + (size_t)qvn * (tokens + 8) * 2;
}

template <int DV>
__global__ void __launch_bounds__(128) decode_pv_kernel(const DecodeArgs a) {
    constexpr int CPR = DV / 8;   // 16-byte chunks per V row
    constexpr int LDS = DV + 8;
    constexpr int NT = DV / 8;    // MMA n-tiles
    extern __shared__ __align__(16) unsigned char dsmem[];
    bf16* vs = reinterpret_cast<bf16*>(dsmem);           // [4 warps][stages][16][LDS]
    float* red = reinterpret_cast<float*>(dsmem);        // [4 warps][8][DV] after the loop
    bf16* ps = reinterpret_cast<bf16*>(dsmem + pv_stage_bytes<DV>());  // [qvn][tokens + 8]
    __shared__ uint32_t mw[8][kPvMaxTok / 32];           // membership words per group head
    __shared__ int32_t tok[kPvMaxTok];                   // union of the group's tokens, ascending
    __shared__ uint8_t bits[kPvMaxTok];                  // which group heads kept each listed token
    __shared__ uint32_t excl[kPvMaxTok / 32];
    __shared__ int n_union;
    __shared__ unsigned last;
    const int g = blockIdx.y;
    const int qvn = a.group * a.n;
    const int64_t t0 = (int64_t)blockIdx.x * a.tokens;
    const int tn = (int)(a.d - t0 < a.tokens ? a.d - t0 : a.tokens);  // a multiple of 8
    const int nw = (tn + 31) / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    // P rows of the query vectors over [t0, t0 + tn)
    for (int c = threadIdx.x; c < qvn * (tn / 8); c += 128) {
        const int qv = c / (tn / 8), q = c - qv * (tn / 8);
        const int hl = qv / a.n, i = qv - hl * a.n;
        cp_async16(ps + qv * (a.tokens + 8) + q * 8, a.A + (int64_t)(g * a.group + hl) * a.stride_a + (int64_t)i * a.lda + t0 + q * 8,
                   16);
    }
    cp_async_commit();
    pdl_trigger();
    for (int e = threadIdx.x; e < 8 * (kPvMaxTok / 32); e += 128) {
        const int hl = e / (kPvMaxTok / 32), w = e - hl * (kPvMaxTok / 32);
        uint32_t word = 0u;
        if (hl < a.group && w < nw) {
            if (a.mask) {
                word = a.mask[(int64_t)(g * a.group + hl) * a.mask_words + t0 / 32 + w];
            } else {
                const int left = tn - 32 * w;
                word = left >= 32 ? ~0u : ((1u << left) - 1u);
            }
        }
        mw[hl][w] = word;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of the union's popcounts over the words
        uint32_t cnt = 0u;
        if (lane < kPvMaxTok / 32 && lane < nw) {
            uint32_t u = 0u;
            for (int hl = 0; hl < a.group; ++hl) u |= mw[hl][lane];
            cnt = __popc(u);
        }
        uint32_t inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane < kPvMaxTok / 32) excl[lane] = inc - cnt;
        if (lane == 31) n_union = (int)inc;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < tn; x += 128) {
        const int w = x >> 5, b = x & 31;
        uint32_t u = 0u, hb = 0u;
        for (int hl = 0; hl < a.group; ++hl) {
            const uint32_t bit = (mw[hl][w] >> b) & 1u;
            u |= mw[hl][w];
            hb |= bit << hl;
        }
        if (hb) {
            const int pos = (int)excl[w] + __popc(u & ((1u << b) - 1u));
            tok[pos] = (int)(t0 + x);
            bits[pos] = (uint8_t)hb;
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    const int nu = n_union;
    const int steps = (nu + 15) / 16;
    const bf16* Vg = a.B + (int64_t)g * a.stride_b;
    bf16* myv = vs + warp * kPvStages * 16 * LDS;
    auto issue = [&](int s, int stage) {
        bf16* dst = myv + stage * 16 * LDS;
        for (int c = lane; c < 16 * CPR; c += 32) {
            const int r = c / CPR, q = c - r * CPR;
            const int pos = s * 16 + r;
            const bool in = pos < nu;
            cp_async16(dst + r * LDS + q * 8, Vg + (int64_t)(in ? tok[pos] : 0) * a.ldb + q * 8, in ? 16 : 0);
        }
    };
    // the A operand of one k-step: rows = query vectors (lane / 4 < 8; rows 8..15
    // are zero), columns = the step's 16 listed tokens
    auto a_frag = [&](int s, uint32_t (&af)[4]) {
        const int qv = lane >> 2;
        const int hl = qv < qvn ? qv / a.n : 0;
        const int kk = (lane & 3) * 2;
        uint32_t v[2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            bf16 e[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int pos = s * 16 + kk + half * 8 + u;
                bf16 w = __float2bfloat16_rn(0.f);
                if (qv < qvn && pos < nu && ((bits[pos] >> hl) & 1u)) w = ps[qv * (a.tokens + 8) + tok[pos] - (int)t0];
                e[u] = w;
            }
            v[half] = pack_bf16x2(e[0], e[1]);
        }
        af[0] = v[0];
        af[1] = 0u;
        af[2] = v[1];
        af[3] = 0u;
    };
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    // warp w takes the steps w, w + 4, ...; its i-th step uses stage i % kPvStages
#pragma unroll
    for (int i = 0; i < kPvStages - 1; ++i) {
        if (warp + 4 * i < steps) issue(warp + 4 * i, i);
        cp_async_commit();
    }
    int it = 0;
    for (int s = warp; s < steps; s += 4, ++it) {
        const int ahead = s + 4 * (kPvStages - 1);
        if (ahead < steps) issue(ahead, (it + kPvStages - 1) % kPvStages);
        cp_async_commit();
        cp_async_wait<kPvStages - 1>();
        __syncwarp();
        uint32_t af[4];
        a_frag(s, af);
        const bf16* vt = myv + (it % kPvStages) * 16 * LDS;
        const bf16* brow = vt + ((lane & 7) + ((lane >> 3) & 1) * 8) * LDS + (lane >> 4) * 8;
#pragma unroll
        for (int p = 0; p < NT / 2; ++p) {
            uint32_t bf[4];
            ldsm_x4_trans(bf, brow + p * 16);
            mma_16816(acc[2 * p], af, bf[0], bf[1]);
            mma_16816(acc[2 * p + 1], af, bf[2], bf[3]);
        }
        __syncwarp();  // the stage read here is refilled by the next iteration's issue
    }
    cp_async_wait<0>();
    __syncthreads();  // every warp is done with its V stages: reuse them for the sums
    {
        const int qv = lane >> 2, f = (lane & 3) * 2;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            red[(warp * 8 + qv) * DV + nt * 8 + f] = acc[nt][0];
            red[(warp * 8 + qv) * DV + nt * 8 + f + 1] = acc[nt][1];
        }
    }
    __syncthreads();
    const int nparts = gridDim.x;
    for (int e = threadIdx.x; e < qvn * DV; e += 128) {
        const int qv = e / DV, f = e - qv * DV;
        const float v = ((red[qv * DV + f] + red[(8 + qv) * DV + f]) + red[(16 + qv) * DV + f]) +
                        red[(24 + qv) * DV + f];
        if (nparts == 1) {
            const int hl = qv / a.n, i = qv - hl * a.n;
            a.Y[(int64_t)(g * a.group + hl) * a.stride_y + (int64_t)i * a.ldy + f] = __float2bfloat16_rn(v);
        } else {
            a.partials[((int64_t)g * nparts + blockIdx.x) * (8 * DV) + e] = v;
        }
    }
    if (nparts == 1) return;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&a.counters[g], 1u) == (unsigned)nparts - 1u;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int e = threadIdx.x; e < qvn * DV; e += 128) {
        float v = 0.f;
        const float* pp = a.partials + (int64_t)g * nparts * (8 * DV) + e;
        for (int c = 0; c < nparts; ++c) v += __ldcg(pp + (int64_t)c * (8 * DV));
        const int qv = e / DV, f = e - qv * DV;
        const int hl = qv / a.n, i = qv - hl * a.n;
        a.Y[(int64_t)(g * a.group + hl) * a.stride_y + (int64_t)i * a.ldy + f] = __float2bfloat16_rn(v);
    }
    if (threadIdx.x == 0) a.counters[g] = 0u;
}

}  // namespace

bool decode_qk_supported(int64_t d) { return d == 64 || d == 128 || d == 256; }
bool decode_pv_supported(int64_t dv) { return dv == 64 || dv == 128; }

int decode_pv_tokens(int64_t t, int64_t kv_heads, int num_sms) {
    int tokens = kPvMaxTok;
    while (tokens > 128 && kv_heads * ((t + tokens - 1) / tokens) < 2LL * num_sms) tokens /= 2;
    return tokens;
}

template <int D>
cudaError_t launch_qk_d(const DecodeArgs& a, cudaStream_t s) {
    const int64_t tiles = (a.m + qk_rows<D>() - 1) / qk_rows<D>();
    // one persistent wave: about two CTAs per SM over all KV heads
    int64_t x = 2LL * (a.sms > 0 ? a.sms : 1) / a.kv_heads;
    x = x < 1 ? 1 : (x > tiles ? tiles : x);
    const cudaError_t e = cudaFuncSetAttribute(decode_qk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)qk_smem<D>());
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_qk_kernel<D>, dim3((unsigned)x, (unsigned)a.kv_heads), dim3(128), qk_smem<D>(), s, a);
}

cudaError_t launch_decode_qk(const DecodeArgs& a, cudaStream_t s) {
    if (a.m == 0) return cudaSuccess;
    switch (a.d) {
        case 64: return launch_qk_d<64>(a, s);
        case 128: return launch_qk_d<128>(a, s);
        case 256: return launch_qk_d<256>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_pv(const DecodeArgs& a, cudaStream_t s) {
    if (a.d == 0 || a.tokens <= 0 || a.tokens > kPvMaxTok) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)((a.d + a.tokens - 1) / a.tokens), a.kv_heads);
    const int qvn = a.group * a.n;
    if (a.m == 64) return launch_pdl(decode_pv_kernel<64>, grid, dim3(128), pv_smem<64>(qvn, a.tokens), s, a);
    if (a.m == 128) return launch_pdl(decode_pv_kernel<128>, grid, dim3(128), pv_smem<128>(qvn, a.tokens), s, a);
    return cudaErrorInvalidValue;
}

}  // namespace rmm
