// rmm_attn.cu -- fused RMM attention: the three steps of "Reduced Matrix
// Multiplication: Input-Adaptive Matrix-Product Reduction for LLM Inference"
// §3.3 "Attention" without writing the score matrix S or the weights P:
//   features  I_h = TopK of Q_h's column norms;  S = alpha Q_h[:, I_h] K_g[:, I_h]^T + M
//   weights   P = softmax(S) over each query row
//   tokens    T_h = TopK of P's column norms;    O_h = P[:, T_h] V_g[T_h, :]
// Token selection needs the column norms of the final P before any output is
// formed, and every row's normalisation before any column norm, so the score
// blocks are recomputed in three passes of one kernel (the paper's own
// kernels were not fully fused; App. B.7):
//   kRowStats  per query row the maximum m_i and the exponential sum l_i of
//              its scaled scores (online over the key blocks);
//   kColScores per key the sum over 32 rows of P[i][t]^2 with
//              P = exp(S - m_i) / l_i, written per 32-row slice; a second
//              kernel adds the slices in order, and TopK picks T_h;
//   kOutput    O = sum over the key blocks holding a kept token of
//              (P masked to T_h, rounded to bf16) V, on the tensor cores.
// The feature selection and the copy of Q with the unkept features zeroed
// come from one cluster launch, as in the library's QK op (the contraction
// then runs over all d_h with exact zeros).
//
// One CTA computes 128 query rows of one head: warp 0 loads by TMA (Q once,
// then K (and V) blocks of 128 keys), warp 1 issues tcgen05.mma, and 8 row
// warps, two per TMEM lane quadrant, each own 32 rows x 64 keys of every block
// (one row per thread).  The score passes put S = Q K^T into one of two TMEM
// buffers while the row warps read the other.  The output pass keeps one S
// buffer in two 64-key halves, one per key group of row warps: a half's row
// warps read their scores and write P as bf16 pairs over them, and the PV
// product (O in TMEM) takes that P as its A operand, while the other half is
// being scored or exponentiated.  Every pass fits two CTAs on an SM.  Every
// wait is bounded.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kRowStats = 0;
constexpr int kColScores = 1;
constexpr int kOutput = 2;

constexpr int BQ = 128;    // query rows per CTA
constexpr int BKEY = 128;  // keys per block
constexpr int DH = 128;    // head dimension of Q and K
constexpr int DV = 128;    // value dimension
constexpr int ATOM = 128 * 128;  // one 64-column swizzle atom of 128 rows (bytes)
constexpr uint32_t kColO = 128;  // output pass: O accumulator columns (S and then P in [0, 128))
constexpr int TILE = 2 * ATOM;   // a 128 x 128 bf16 operand tile

struct __align__(64) AttnParams {
    CUtensorMap map_q;  // masked Q: {d_h, n, heads}, box {64, 128, 1}
    CUtensorMap map_k;   // K: {d_h, n, kv_heads}, box {64, 128, 1} (score passes)
    CUtensorMap map_kh;  // output pass: K with a {64, 64, 1} box (half a key block)
    CUtensorMap map_vh;  // output pass: V {d_v, n, kv_heads} with a {64, 64, 1} box
    __nv_bfloat16* O;   // [heads][n][ldo]
    int64_t ldo, stride_o;
    float* row_m;       // [heads][n]: maximum of the row's scaled scores (base-2 units)
    float* row_l;       // [heads][n]: sum over the row of 2^(x - m)
    float* col_part;    // [heads][4 q_blocks][n]: per 32-row slice, sum of P^2 per key
    const uint32_t* tok_mask;  // [heads][mask_words]: bit t set iff token t is kept
    int64_t mask_words;
    int n, heads, group, q_blocks, k_blocks, causal;
    float scale_log2;   // alpha * log2(e): the scores are taken in base 2
    int* err;
};

template <int MODE>
struct AttnCfg {
    static constexpr bool OUT = MODE == kOutput;
    // Row warps: RW / 4 per TMEM lane quadrant, each owning CH 32-key chunks of
    // every key block.  Every pass runs 8 (64 keys each) and fits two CTAs on
    // an SM.  The score-only passes keep two S buffers and two K stages.  The
    // output pass keeps one S buffer, whose two 64-key halves (one per key
    // group of row warps) run S -> P -> PV on their own barriers, P written over
    // the scores it came from; K and V have one stage each, loaded and released
    // by halves, so that one half's exponentials overlap the other half's
    // products and the next block's scores.
    static constexpr int RW = 8;
    static constexpr int CQ = RW / 4;      // key groups per block
    static constexpr int CH = 4 / CQ;      // 32-key chunks per warp and block
    static constexpr int NT = 32 * (2 + RW);
    static constexpr int MINB = 2;         // CTAs per SM
    static constexpr int STAGES = OUT ? 1 : 2;  // K stages
    static constexpr int V_BYTES = OUT ? TILE : 0;  // one V stage
    static constexpr int STAT_BYTES = MODE == kRowStats ? 2 * CQ * BQ * 4 : 0;  // per-group (m, l) of each row
    static constexpr size_t SMEM = 1024 + TILE + STAGES * (size_t)TILE + V_BYTES + STAT_BYTES + 256;
    // TMEM columns: score passes two S buffers [0, 256); output pass one S
    // buffer [0, 128), whose 32-key chunks take their bf16 P pairs in their
    // first 16 columns, and O [128, 256)
    static constexpr uint32_t TMEM_COLS = 256;
};

// Query block of CTA b: the longest causal key ranges first.
__device__ __forceinline__ void attn_block(const AttnParams& p, int& h, int& qb) {
    const int b = blockIdx.x;
    const int r = b / p.heads;
    h = b - r * p.heads;
    qb = p.causal ? p.q_blocks - 1 - r : r;
}

constexpr int kMaxKeyBlocks = (int)(kMaxSelectD / BKEY);  // key blocks of the longest sequence

// Output pass: whether key block kb holds a kept token (bit kb of used_bits,
// filled from the token mask when the CTA starts).
__device__ __forceinline__ bool block_used(const uint32_t* used_bits, int kb) {
    return (used_bits[kb >> 5] >> (kb & 31)) & 1u;
}

template <int MODE>
__global__ void __launch_bounds__(AttnCfg<MODE>::NT, AttnCfg<MODE>::MINB) attn_pass_kernel(const __grid_constant__ AttnParams p) {
    using C = AttnCfg<MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + TILE;                          // STAGES K tiles
    uint8_t* sV = sK + C::STAGES * TILE;              // output pass: one V tile
    float* stat = reinterpret_cast<float*>(sV + C::V_BYTES);  // [2][CQ][BQ] (row statistics)
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stat) + C::STAT_BYTES);
    // [2] each: score passes index K stages and S buffers by 2; the output pass
    // indexes the halves of its one K stage, V stage and S buffer
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = bars + 3;
    uint64_t* s_full = bars + 5;
    uint64_t* s_empty = bars + 7;                 // output pass: the half's P has been read
    uint64_t* p_full = bars + 9;                  // output pass: the half's P written
    uint64_t* v_full = bars + 11;
    uint64_t* v_empty = bars + 13;
    uint64_t* o_full = bars + 15;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(o_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&s_full[s], 1);
            // score passes: one arrival per row warp once its scores are in
            // registers; output pass: the MMA's commit after the half's PV product
            mbar_init(&s_empty[s], C::OUT ? 1 : C::RW);
            mbar_init(&p_full[s], C::RW / 2);  // the row warps of the half
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(o_full, 1);
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_map(&p.map_q);
        if (C::OUT) {
            tma_prefetch_map(&p.map_kh);
            tma_prefetch_map(&p.map_vh);
        } else {
            tma_prefetch_map(&p.map_k);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_wait();
    pdl_trigger();

    int h, qb;
    attn_block(p, h, qb);
    const int g = h / p.group;
    const int q0 = qb * BQ;
    const int kb_end = p.causal ? min(qb + 1, p.k_blocks) : p.k_blocks;
    __shared__ uint32_t used_bits[(kMaxKeyBlocks + 31) / 32];
    if constexpr (C::OUT) {
        // which key blocks hold a kept token (the token mask is written by the
        // selection that runs before this pass)
        const uint32_t* w = p.tok_mask + (int64_t)h * p.mask_words;
        for (int kb0 = warp * 32; kb0 < kb_end; kb0 += C::NT) {
            const int kb = kb0 + lane;
            uint32_t any = 0;
            if (kb < kb_end) {
#pragma unroll
                for (int i = 0; i < BKEY / 32; ++i) {
                    const int64_t wi = (int64_t)kb * (BKEY / 32) + i;
                    if (wi < p.mask_words) any |= __ldg(w + wi);
                }
            }
            const uint32_t bits = __ballot_sync(0xffffffffu, any != 0u);
            if (lane == 0) used_bits[kb0 >> 5] = bits;
        }
        __syncthreads();
    }
    auto used = [&](int kb) { return !C::OUT || block_used(used_bits, kb); };

    if (warp == 0) {
        // ---------------------------------------------------------------- loads
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, TILE);
            tma_load_3d(sQ, &p.map_q, q_full, 0, q0, h);
            tma_load_3d(sQ + ATOM, &p.map_q, q_full, 64, q0, h);
            uint32_t it = 0;
            bool ok = true;
            for (int kb = 0; kb < kb_end && ok; ++kb) {
                if (!used(kb)) continue;
                const int s = it % C::STAGES;
                const uint32_t ph = (it / C::STAGES) & 1u;
                if constexpr (C::OUT) {
                    // each half of K once the previous block's scores of that
                    // half are done, then each half of V once the previous
                    // block's PV product of that half has read it; a half is
                    // rows hh * 64 .. +64 of both 64-column swizzle atoms
                    for (int hh = 0; hh < 2 && ok; ++hh) {
                        if (!mbar_wait(&k_empty[hh], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&k_full[hh], TILE / 2);
                        tma_load_3d(sK + hh * (ATOM / 2), &p.map_kh, &k_full[hh], 0, kb * BKEY + hh * 64, g);
                        tma_load_3d(sK + ATOM + hh * (ATOM / 2), &p.map_kh, &k_full[hh], 64, kb * BKEY + hh * 64, g);
                    }
                    for (int hh = 0; hh < 2 && ok; ++hh) {
                        if (!mbar_wait(&v_empty[hh], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&v_full[hh], TILE / 2);
                        tma_load_3d(sV + hh * (ATOM / 2), &p.map_vh, &v_full[hh], 0, kb * BKEY + hh * 64, g);
                        tma_load_3d(sV + ATOM + hh * (ATOM / 2), &p.map_vh, &v_full[hh], 64, kb * BKEY + hh * 64, g);
                    }
                } else {
                    if (!mbar_wait(&k_empty[s], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) break;
                    uint8_t* dst = sK + s * TILE;
                    mbar_arrive_expect_tx(&k_full[s], TILE);
                    tma_load_3d(dst, &p.map_k, &k_full[s], 0, kb * BKEY, g);
                    tma_load_3d(dst + ATOM, &p.map_k, &k_full[s], 64, kb * BKEY, g);
                }
                ++it;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc(kKindF16, false, BKEY, 128);      // S = Q K^T
            constexpr uint32_t idesc_sh = umma_idesc(kKindF16, false, BKEY / 2, 128); // half of S
            constexpr uint32_t idesc_o = umma_idesc(kKindF16, true, DV, 128);         // O += P V (V MN-major)
            const uint32_t q_addr = smem_u32(sQ);
            bool ok = mbar_wait(q_full, 0u, abort_flag, p.err, kErrTimeoutMma);
            if constexpr (C::OUT) {
                // S half hh of the j-th used key block into TMEM columns
                // hh * 64 .. +64, once K's half has landed and the previous
                // block's PV product of that half has read its P
                auto issue_s = [&](uint32_t j, int hh) -> bool {
                    if (!mbar_wait(&k_full[hh], j & 1u, abort_flag, p.err, kErrTimeoutMma) ||
                        !mbar_wait(&s_empty[hh], (j & 1u) ^ 1u, abort_flag, p.err, kErrTimeoutMma))
                        return false;
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(sK) + hh * (ATOM / 2);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk) {
                        const uint64_t adesc = sw128_desc(q_addr + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
                        const uint64_t bdesc = sw128_desc(k_addr + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
                        umma<kKindF16>(tmem_base + hh * (BKEY / 2), adesc, bdesc, idesc_sh, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[hh]);
                    umma_commit(&k_empty[hh]);  // K's half consumed
                    return true;
                };
                // O += P V over the half's 64 keys, once its row warps have
                // written P over the scores and V's half has landed
                auto issue_pv = [&](uint32_t j, int hh) -> bool {
                    if (!mbar_wait(&p_full[hh], j & 1u, abort_flag, p.err, kErrTimeoutMma) ||
                        !mbar_wait(&v_full[hh], j & 1u, abort_flag, p.err, kErrTimeoutMma))
                        return false;
                    tc_fence_after();
                    const uint32_t v_addr = smem_u32(sV);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        // keys 16 kk .. +16: chunk kk / 2, its P columns (kk % 2) * 8 .. +8
                        const int kk = hh * 4 + q;
                        const uint64_t bdesc = sw128_desc(v_addr + kk * 16 * 128, ATOM, 1024);
                        umma_ts(tmem_base + kColO, tmem_base + (kk >> 1) * 32 + (kk & 1) * 8, bdesc, idesc_o,
                                (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&s_empty[hh]);  // the half's P read: it may take the next scores
                    umma_commit(&v_empty[hh]);
                    return true;
                };
                auto next_used = [&](int kb) {
                    while (kb < kb_end && !used(kb)) ++kb;
                    return kb;
                };
                // order: S(0, 0), S(0, 1), then per block j: PV(j, 0), S(j+1, 0),
                // PV(j, 1), S(j+1, 1)
                int kb = next_used(0);
                uint32_t j = 0;
                if (ok && kb < kb_end) ok = issue_s(0, 0) && issue_s(0, 1);
                while (ok && kb < kb_end) {
                    const int kn = next_used(kb + 1);
                    ok = issue_pv(j, 0);
                    if (ok && kn < kb_end) ok = issue_s(j + 1, 0);
                    if (ok) ok = issue_pv(j, 1);
                    if (ok && kn < kb_end) ok = issue_s(j + 1, 1);
                    kb = kn;
                    ++j;
                }
                umma_commit(o_full);
            } else {
                uint32_t it = 0;
                for (int kb = 0; kb < kb_end && ok; ++kb) {
                    if (!used(kb)) continue;
                    const int s = it % C::STAGES;  // K stage
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    const int sb = it & 1;         // S buffer
                    const uint32_t sph = (it >> 1) & 1u;
                    if (!mbar_wait(&k_full[s], ph, abort_flag, p.err, kErrTimeoutMma) ||
                        !mbar_wait(&s_empty[sb], sph ^ 1u, abort_flag, p.err, kErrTimeoutMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(sK + s * TILE);
                    const uint32_t d_tmem = tmem_base + sb * BKEY;
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk) {
                        const uint64_t adesc = sw128_desc(q_addr + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
                        const uint64_t bdesc = sw128_desc(k_addr + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
                        umma<kKindF16>(d_tmem, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[sb]);
                    umma_commit(&k_empty[s]);  // K consumed by this block's scores
                    ++it;
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- rows
        const int quad = warp & 3;         // TMEM lane quadrant: rows quad*32 .. +32
        const int cq = (warp - 2) >> 2;    // key group: chunks cq*CH .. +CH of every block
        const int r_loc = quad * 32 + lane;
        const int row = q0 + r_loc;
        const bool row_ok = row < p.n;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        // Every weight is 2^(x - b) with x = scale * score and b = m + log2(l)
        // the row's base (one exp per weight, no division); rows past n and
        // rows without a key get b = +inf, so that all their weights are 0.
        float m = -INFINITY, l = 0.f, b = INFINITY;
        if (MODE != kRowStats && row_ok) {
            m = p.row_m[(int64_t)h * p.n + row];
            l = p.row_l[(int64_t)h * p.n + row];
            if (l > 0.f) b = m + log2f(l);
        }
        const float scale = p.scale_log2;
        const uint32_t* mask_h = p.tok_mask ? p.tok_mask + (int64_t)h * p.mask_words : nullptr;
        // output pass: lane j holds this warp's mask words (one per chunk) of key
        // block 32 * keep_base + j
        uint32_t keep_reg[C::CH];
#pragma unroll
        for (int c = 0; c < C::CH; ++c) keep_reg[c] = 0u;
        int keep_base = -1;
        // One 32-key chunk (chunk cc of key block kb, in buffer sb) of this row.
        auto chunk = [&](int kb, int cc, int sb, const uint32_t (&raw)[32]) {
            const int k0 = kb * BKEY + cc * 32;  // the chunk's first key
            // which of the 32 keys of this row count: all, none, or some (the
            // diagonal block and the last block)
            const bool all_in = row_ok && k0 + 31 < p.n && (!p.causal || k0 + 31 <= row);
            const bool none_in = !row_ok || k0 >= p.n || (p.causal && k0 > row);
            // one uniform test per chunk: every key counts, or some are masked
            const bool uniform = __all_sync(0xffffffffu, all_in);
            auto valid = [&](int i) { return !none_in && k0 + i < p.n && (!p.causal || k0 + i <= row); };
            auto sc = [&](int i) { return __uint_as_float(raw[i]); };
            if constexpr (MODE == kRowStats) {
                if (uniform) {
                    // the largest scaled score is the scale times the largest
                    // (or, for a negative scale, the smallest) raw score: rounding
                    // keeps the order; each weight is then one fma and one ex2
                    float mc[4] = {sc(0), sc(1), sc(2), sc(3)};
                    if (scale >= 0.f) {
#pragma unroll
                        for (int i = 4; i < 32; ++i) mc[i & 3] = fmaxf(mc[i & 3], sc(i));
                        mc[0] = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
                    } else {
#pragma unroll
                        for (int i = 4; i < 32; ++i) mc[i & 3] = fminf(mc[i & 3], sc(i));
                        mc[0] = fminf(fminf(mc[0], mc[1]), fminf(mc[2], mc[3]));
                    }
                    const float mn = fmaxf(m, mc[0] * scale);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i & 3] += fast_exp2(fmaf(sc(i), scale, -mn));
                    l = fmaf(l, fast_exp2(m - mn), (acc[0] + acc[1]) + (acc[2] + acc[3]));
                    m = mn;
                } else if (!none_in) {
                    float x[32];  // x = scale * score, -inf where masked
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = valid(i) ? sc(i) * scale : -INFINITY;
                    float mc[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
                    for (int i = 4; i < 32; ++i) mc[i & 3] = fmaxf(mc[i & 3], x[i]);
                    const float mn = fmaxf(m, fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])));
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i & 3] += fast_exp2(x[i] - mn);  // 2^-inf = 0
                    l = fmaf(l, fast_exp2(m - mn), (acc[0] + acc[1]) + (acc[2] + acc[3]));
                    m = mn;
                }
            } else if constexpr (MODE == kColScores) {
                float z = 0.f;
                if (__any_sync(0xffffffffu, !none_in)) {
                    // P^2 = 2^(2 (x - b)) in one fma and one ex2; 0 where masked
                    const float s2 = 2.f * scale, nb2 = -2.f * b;
                    float q[32];
                    if (uniform) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) q[i] = fast_exp2(fmaf(sc(i), s2, nb2));
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) q[i] = fast_exp2(valid(i) ? fmaf(sc(i), s2, nb2) : -INFINITY);
                    }
                    z = warp_column_sums(q, lane);  // this warp's 32 rows, summed per key
                }
                const int key = k0 + lane;
                if (key < p.n) p.col_part[((int64_t)h * p.q_blocks * 4 + qb * 4 + quad) * p.n + key] = z;
            } else {
                // P masked to the kept tokens, rounded to bf16, written over the
                // chunk's first 16 score columns (in registers by now)
                if ((kb >> 5) != keep_base) {  // the same for every lane
                    keep_base = kb >> 5;
#pragma unroll
                    for (int c = 0; c < C::CH; ++c) {
                        const int64_t wi = (int64_t)(keep_base * 32 + lane) * (BKEY / 32) + cq * C::CH + c;
                        keep_reg[c] = wi < p.mask_words ? __ldg(mask_h + wi) : 0u;
                    }
                }
                const uint32_t keep_bits = __shfl_sync(0xffffffffu, keep_reg[cc - cq * C::CH], kb & 31);
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) w[e] = 0u;
                if (keep_bits != 0u) {  // the same for every lane: a chunk without a kept token stays 0
                    // bit i: key k0 + i is kept and inside this row's causal range
                    const int lim = none_in ? 0 : min(32, min(p.n, p.causal ? row + 1 : p.n) - k0);
                    const uint32_t live = keep_bits & (lim >= 32 ? 0xffffffffu : ((1u << lim) - 1u));
                    // each weight is 2^(x - b), x - b in one fma
                    if (__all_sync(0xffffffffu, live == 0xffffffffu)) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(fast_exp2(fmaf(sc(2 * e), scale, -b)),
                                                                            fast_exp2(fmaf(sc(2 * e + 1), scale, -b)));
                            w[e] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float p0 = ((live >> (2 * e)) & 1u) ? fast_exp2(fmaf(sc(2 * e), scale, -b)) : 0.f;
                            const float p1 =
                                ((live >> (2 * e + 1)) & 1u) ? fast_exp2(fmaf(sc(2 * e + 1), scale, -b)) : 0.f;
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                            w[e] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                    }
                }
                // keys 2e, 2e + 1 of the chunk -> one 32-bit column of this row's lane
                tmem_st_32x32b_x16(tmem_base + lane_base + cc * 32, w);
            }
        };
        uint32_t it = 0;
        bool ok = true;
        for (int kb = 0; kb < kb_end && ok; ++kb) {
            if (!used(kb)) continue;
            // S buffer (the output pass has one, and waits for its key group's half)
            const int sb = C::OUT ? 0 : (int)(it & 1u);
            const uint32_t ph = C::OUT ? (it & 1u) : ((it >> 1) & 1u);
            ++it;
            if (!mbar_wait(&s_full[C::OUT ? cq : sb], ph, abort_flag, p.err, kErrTimeoutEpilogue)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t raw[C::CH][32];
#pragma unroll
            for (int c = 0; c < C::CH; ++c)
                tmem_ld_32x32b_x32(tmem_base + lane_base + sb * BKEY + (cq * C::CH + c) * 32, raw[c]);
            tmem_ld_wait();
            if constexpr (!C::OUT) {
                // the scores are in registers: this S buffer may be overwritten
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[sb]);
            }
#pragma unroll
            for (int c = 0; c < C::CH; ++c) chunk(kb, cq * C::CH + c, sb, raw[c]);
            if constexpr (C::OUT) {
                tmem_st_wait();  // this warp's P columns are written before the MMA reads them
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[cq]);
            }
        }
        if constexpr (MODE == kRowStats) {
            // the key groups' (m, l) of each row, combined in group order;
            // every row warp reaches this barrier once, whether or not a wait gave up
            stat[cq * BQ + r_loc] = m;
            stat[C::CQ * BQ + cq * BQ + r_loc] = l;
            asm volatile("bar.sync 1, %0;" ::"n"(32 * C::RW) : "memory");
            if (cq == 0 && row_ok) {
                float mr = stat[r_loc];
#pragma unroll
                for (int j = 1; j < C::CQ; ++j) mr = fmaxf(mr, stat[j * BQ + r_loc]);
                float lr = 0.f;
#pragma unroll
                for (int j = 0; j < C::CQ; ++j) {
                    const float mj = stat[j * BQ + r_loc];
                    if (mj > -INFINITY) lr += stat[C::CQ * BQ + j * BQ + r_loc] * fast_exp2(mj - mr);
                }
                p.row_m[(int64_t)h * p.n + row] = mr;
                p.row_l[(int64_t)h * p.n + row] = lr;
            }
        }
        if constexpr (C::OUT) {
            const bool have = ok && it > 0;
            if (have && !mbar_wait(o_full, 0u, abort_flag, p.err, kErrTimeoutEpilogue)) ok = false;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < C::CH; ++c) {
                const int col = (cq * C::CH + c) * 32;  // this warp's output columns col .. +32
                uint32_t raw[32];
                if (have && ok) {
                    tmem_ld_32x32b_x32(tmem_base + lane_base + kColO + col, raw);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) raw[i] = 0u;  // no kept token in this row's range
                }
                if (row_ok) {
                    __nv_bfloat16* orow = p.O + (int64_t)h * p.stride_o + (int64_t)row * p.ldo + col;
#pragma unroll
                    for (int gi = 0; gi < 4; ++gi) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(raw[gi * 8 + 2 * e]),
                                                                            __uint_as_float(raw[gi * 8 + 2 * e + 1]));
                            w[e] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                        *reinterpret_cast<uint4*>(orow + gi * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// a2[h][t] = sum over the 32-row slices (in row order) of their P^2 sums;
// with the causal mask only the slices of the blocks at or below key t's
// block hold any.
__global__ void __launch_bounds__(256) attn_colscore_reduce_kernel(const float* __restrict__ part,
                                                                   float* __restrict__ a2, int n, int q_blocks,
                                                                   int causal) {
    pdl_wait();
    pdl_trigger();
    const int h = blockIdx.y;
    const int t = blockIdx.x * 256 + threadIdx.x;
    if (t >= n) return;
    const int s0 = causal ? (t / BKEY) * 4 : 0;
    const float* ph = part + (int64_t)h * q_blocks * 4 * n + t;
    float z = 0.f;
    for (int sl = s0; sl < 4 * q_blocks; ++sl) z += ph[(int64_t)sl * n];
    a2[(int64_t)h * n + t] = z;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// 3-D bf16 map {cols, rows, heads} with a {64, box_rows, 1} box and 128-byte swizzle.
bool encode_map(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int64_t heads, int64_t ld,
                int64_t stride_h, uint32_t box_rows = 128) {
    auto enc = encoder();
    if (!enc) return false;
    uint64_t head_bytes = heads > 1 ? static_cast<uint64_t>(stride_h) * 2 : static_cast<uint64_t>(ld) * 2 * rows;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2, head_bytes};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_pass(const AttnParams& p, cudaStream_t s) {
    using C = AttnCfg<MODE>;
    cudaError_t e = cudaFuncSetAttribute(attn_pass_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_pass_kernel<MODE>, dim3((unsigned)(p.q_blocks * p.heads)), dim3(C::NT), C::SMEM, s, p);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int64_t retained(double rho, int64_t d) {
    const double x = rho * static_cast<double>(d);
    const double r = std::nearbyint(x);
    int64_t k = (std::fabs(x - r) <= 1e-9 * static_cast<double>(d)) ? static_cast<int64_t>(r)
                                                                      : static_cast<int64_t>(std::ceil(x));
    return k < 1 ? 1 : (k > d ? d : k);
}

// Workspace layout of one problem (offsets in bytes, 256-aligned).
struct AttnLayout {
    int64_t kd, kt, q_blocks, mask_words;
    size_t err, I, T, qm, rm, rl, cpart, a2, mask, total;
};

AttnLayout attn_layout(const rmm_attn_problem* p) {
    AttnLayout L{};
    L.kd = retained(p->rho_d, p->d_h);
    L.kt = retained(p->rho_t, p->n);
    L.q_blocks = (p->n + BQ - 1) / BQ;
    L.mask_words = (p->n + 31) / 32;
    size_t off = 0;
    L.err = off;  // error word: a kernel that gave up on a wait records its code
    off += 256;
    L.I = off;
    off += align256(static_cast<size_t>(p->heads) * L.kd * sizeof(int32_t));
    L.T = off;
    off += align256(static_cast<size_t>(p->heads) * L.kt * sizeof(int32_t));
    L.qm = off;
    off += align256(static_cast<size_t>(p->heads) * p->n * p->d_h * 2);
    L.rm = off;
    off += align256(static_cast<size_t>(p->heads) * p->n * sizeof(float));
    L.rl = off;
    off += align256(static_cast<size_t>(p->heads) * p->n * sizeof(float));
    L.cpart = off;
    off += align256(static_cast<size_t>(p->heads) * 4 * L.q_blocks * p->n * sizeof(float));
    L.a2 = off;
    off += align256(static_cast<size_t>(p->heads) * p->n * sizeof(float));
    L.mask = off;
    off += align256(static_cast<size_t>(p->heads) * L.mask_words * sizeof(uint32_t));
    L.total = off;
    return L;
}

rmm_status validate_attn(const rmm_attn_problem* p) {
    if (!p) return RMM_ERR_INVALID_ARG;
    if (p->heads < 1 || p->kv_heads < 1 || p->heads % p->kv_heads != 0 || p->n < 0) return RMM_ERR_INVALID_ARG;
    if (p->d_h != DH || p->d_v != DV) return RMM_ERR_UNSUPPORTED;
    if (p->heads > 65535 || p->n > kMaxSelectD) return RMM_ERR_UNSUPPORTED;
    if (p->n % 8 != 0) return RMM_ERR_INVALID_ARG;  // token scores are selected in 16-byte groups
    if (p->ldq < p->d_h || p->ldk < p->d_h || p->ldv < p->d_v || p->ldo < p->d_v) return RMM_ERR_INVALID_ARG;
    if (p->ldq % 8 || p->ldk % 8 || p->ldv % 8 || p->ldo % 8) return RMM_ERR_INVALID_ARG;
    if (p->heads > 1 && (p->stride_q % 8 || p->stride_o % 8 || p->stride_q < p->n * p->ldq ||
                         p->stride_o < p->n * p->ldo))
        return RMM_ERR_INVALID_ARG;
    if (p->kv_heads > 1 && (p->stride_k % 8 || p->stride_v % 8 || p->stride_k < p->n * p->ldk ||
                            p->stride_v < p->n * p->ldv))
        return RMM_ERR_INVALID_ARG;
    if (!(p->rho_d > 0.0) || p->rho_d > 1.0 || !(p->rho_t > 0.0) || p->rho_t > 1.0) return RMM_ERR_INVALID_ARG;
    if (!std::isfinite(p->alpha)) return RMM_ERR_INVALID_ARG;
    if (p->flags & ~RMM_FLAG_CAUSAL) return RMM_ERR_INVALID_ARG;
    return RMM_OK;
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return sms;
}

}  // namespace
}  // namespace rmm

extern "C" {

size_t rmm_attention_workspace_size(const rmm_attn_problem* p) {
    if (rmm::validate_attn(p) != RMM_OK) return 0;
    return rmm::attn_layout(p).total;
}

rmm_status rmm_attention(const rmm_attn_problem* p, const void* Q, const void* K, const void* V, void* O,
                         int32_t* I_out, int32_t* T_out, void* ws, size_t ws_bytes, void* stream) {
    using namespace rmm;
    rmm_status st = validate_attn(p);
    if (st != RMM_OK) return st;
    if (p->n == 0) return RMM_OK;
    if (!Q || !K || !V || !O) return RMM_ERR_INVALID_ARG;
    for (const void* ptr : {Q, K, V, static_cast<const void*>(O)})
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return RMM_ERR_INVALID_ARG;
    if ((I_out && (reinterpret_cast<uintptr_t>(I_out) & 3u)) || (T_out && (reinterpret_cast<uintptr_t>(T_out) & 3u)))
        return RMM_ERR_INVALID_ARG;
    const int sms = device_sms();
    if (sms <= 0) return RMM_ERR_CUDA;
    const AttnLayout L = attn_layout(p);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return RMM_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int H = static_cast<int>(p->heads);
    const int64_t n = p->n;
    int32_t* I = I_out ? I_out : reinterpret_cast<int32_t*>(w + L.I);
    int32_t* T = T_out ? T_out : reinterpret_cast<int32_t*>(w + L.T);

    // 1. features: I_h = TopK of Q_h's column norms, and 2. Q with the unkept
    // features zeroed, in one cluster launch (every feature kept: Q as it is)
    cudaError_t e;
    const __nv_bfloat16* Qs = static_cast<const __nv_bfloat16*>(Q);
    int64_t ldqs = p->ldq, stride_qs = p->stride_q;
    if (L.kd == p->d_h) {
        e = launch_identity(I, L.kd, H, s);
    } else {
        QkMaskArgs qa{};
        qa.Q = Q;
        qa.n = n;
        qa.d = p->d_h;
        qa.ldq = p->ldq;
        qa.stride_q = p->stride_q;
        qa.heads = H;
        qa.k = L.kd;
        qa.I = I;
        qa.Qm = w + L.qm;
        qa.ldm = p->d_h;
        qa.stride_m = n * p->d_h;
        qa.cluster = qk_select_cluster(H, n, sms);
        e = launch_qk_select_mask(qa, s);
        Qs = reinterpret_cast<const __nv_bfloat16*>(w + L.qm);
        ldqs = p->d_h;
        stride_qs = n * p->d_h;
    }
    if (e != cudaSuccess) return RMM_ERR_CUDA;

    AttnParams ap;
    std::memset(&ap, 0, sizeof(ap));
    if (!encode_map(&ap.map_q, Qs, p->d_h, n, H, ldqs, stride_qs) ||
        !encode_map(&ap.map_k, K, p->d_h, n, p->kv_heads, p->ldk, p->stride_k) ||
        !encode_map(&ap.map_kh, K, p->d_h, n, p->kv_heads, p->ldk, p->stride_k, 64) ||
        !encode_map(&ap.map_vh, V, p->d_v, n, p->kv_heads, p->ldv, p->stride_v, 64))
        return RMM_ERR_CUDA;
    ap.O = static_cast<__nv_bfloat16*>(O);
    ap.ldo = p->ldo;
    ap.stride_o = p->stride_o;
    ap.row_m = reinterpret_cast<float*>(w + L.rm);
    ap.row_l = reinterpret_cast<float*>(w + L.rl);
    ap.col_part = reinterpret_cast<float*>(w + L.cpart);
    ap.tok_mask = reinterpret_cast<const uint32_t*>(w + L.mask);
    ap.mask_words = L.mask_words;
    ap.n = static_cast<int>(n);
    ap.heads = H;
    ap.group = static_cast<int>(p->heads / p->kv_heads);
    ap.q_blocks = static_cast<int>(L.q_blocks);
    ap.k_blocks = static_cast<int>(L.q_blocks);
    ap.causal = (p->flags & RMM_FLAG_CAUSAL) ? 1 : 0;
    ap.scale_log2 = p->alpha * 1.4426950408889634f;
    ap.err = reinterpret_cast<int*>(w + L.err);
    // 3. row statistics, 4. token scores, 5. T_h, 6. the output
    if (launch_pass<kRowStats>(ap, s) != cudaSuccess) return RMM_ERR_CUDA;
    if (launch_pass<kColScores>(ap, s) != cudaSuccess) return RMM_ERR_CUDA;
    float* a2 = reinterpret_cast<float*>(w + L.a2);
    if (launch_pdl(attn_colscore_reduce_kernel, dim3((unsigned)((n + 255) / 256), (unsigned)H), dim3(256), 0, s,
                   static_cast<const float*>(ap.col_part), a2, ap.n, ap.q_blocks, ap.causal) != cudaSuccess)
        return RMM_ERR_CUDA;
    SelectArgs ta{};
    ta.d = n;
    ta.heads = H;
    ta.k = L.kt;
    ta.I = T;
    ta.scores = a2;
    ta.mask = reinterpret_cast<uint32_t*>(w + L.mask);
    ta.mask_words = L.mask_words;
    if (launch_topk(ta, s) != cudaSuccess) return RMM_ERR_CUDA;
    if (launch_pass<kOutput>(ap, s) != cudaSuccess) return RMM_ERR_CUDA;
    return RMM_OK;
}

}  // extern "C"
