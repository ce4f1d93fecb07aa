// rmm_gemm.cu -- the reduced product of Reduced Matrix Multiplication on the
// B200 tensor cores: Y = A[:, I] B[I, :] ("Reduced Matrix Multiplication:
// Input-Adaptive Matrix-Product Reduction for LLM Inference", §3.2; per-head
// attention forms in §3.3; cost O(n k m) in §3.4 and Appendix D.1 Eq. (1)-(4)).
//
// Design (sm_100a, one CTA per SM, persistent over 128 x BN output tiles,
// 192 threads):
//   warp 0     producer.  One lane issues the TMA tile of the packed operand
//              A[:, I] (K-major).  B arrives by TMA in one of three ways:
//                kGather: the retained rows B[I, :] of a row-major d x m
//                  matrix (I == nullptr: all rows in order), four indexed
//                  rows per tile::gather4 instruction
//                  (16 lanes x BN/64 column groups per stage), written in the
//                  128-byte-swizzled MN-major layout;
//                kRows: consecutive rows (every index kept), plain tiles in
//                  the same MN-major layout;
//                kKMajor: a K-major tile of an m x K matrix (QK mode: the
//                  packed K[:, I]; fp32 problems: B[I, :] staged transposed).
//   warp 1     MMA issuer.  One thread issues tcgen05.mma (kind::f16 for bf16,
//              kind::tf32 for fp32) into a double-buffered fp32 accumulator
//              in tensor memory and commits stage releases to mbarriers.
//   warps 2-5  epilogue.  tcgen05.ld of the accumulator (one TMEM lane
//              quadrant per warp), alpha scaling, the causal -inf mask,
//              rounding to the storage dtype and 16-byte global stores.
//              Tiles that the causal mask covers entirely skip the MMA and
//              store -inf directly.
// Every wait is bounded (rmm_device.cuh); on expiry the kernel records an
// error word and returns.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kThreads = 192;  // 6 warps
constexpr int kBM = 128;

// The tensor-core operand kind of an input type, and the type the product is
// stored in (E4M3 operands give a bf16 output).
template <typename T>
struct KindOf {
    static constexpr int value = sizeof(T) == 4 ? kKindTf32 : sizeof(T) == 1 ? kKindF8 : kKindF16;
};
template <typename T>
struct OutOf {
    using type = T;
};
template <>
struct OutOf<__nv_fp8_e4m3> {
    using type = __nv_bfloat16;
};

template <typename T, int BMODE, int BN>
struct Cfg {
    static constexpr int ES = sizeof(T);
    static constexpr bool TF32 = (ES == 4);
    static constexpr int KIND = KindOf<T>::value;
    static constexpr bool B_MN = (BMODE != kBKMajor);
    static constexpr int BK = 128 / ES;        // one 128-byte swizzle row of K
    static constexpr int UK = 32 / ES;         // K per tcgen05.mma
    static constexpr int A_BYTES = kBM * 128;  // 128 rows x 128 B
    static constexpr int B_BYTES = BN * 128;   // BK rows x BN cols (MN-major) or BN rows x 128 B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (BN == 256) ? 4 : 6;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int GROUP_BYTES = BK * 128;  // one 64-column group of an MN-major B tile
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
    static_assert(!(TF32 && B_MN), "fp32 operands are staged K-major");
};

struct TileCoord {
    int h, m0, n0;
    bool skip;  // entirely above the causal diagonal
};

__device__ __forceinline__ TileCoord decode_tile(int t, const GemmParams& p, int bn) {
    TileCoord c;
    const int mt = t % p.m_tiles;
    const int rest = t / p.m_tiles;
    const int nt = rest % p.n_tiles;
    c.h = rest / p.n_tiles;
    c.m0 = mt * kBM;
    c.n0 = nt * bn;
    c.skip = p.causal && (c.n0 > c.m0 + kBM - 1);
    return c;
}

template <typename T>
__device__ __forceinline__ void store_chunk(T* yrow, int col0, int m, const float (&v)[32]) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (col0 + 8 * g < m) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * g + 2 * i], v[8 * g + 2 * i + 1]);
                    w[i] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                *reinterpret_cast<uint4*>(yrow + col0 + 8 * g) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    } else {
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            if (col0 + 4 * g < m)
                *reinterpret_cast<float4*>(yrow + col0 + 4 * g) =
                    make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        }
    }
}

template <typename T, int BMODE, int BN>
__global__ void __launch_bounds__(kThreads, 1) gather_gemm_kernel(const __grid_constant__ GemmParams p) {
    using C = Cfg<T, BMODE, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_map(&p.map_a);
        tma_prefetch_map(&p.map_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_wait();  // everything above touched only shared and tensor memory
    pdl_trigger();

    const int total = p.heads * p.m_tiles * p.n_tiles;
    const int num_kb = (p.k + C::BK - 1) / C::BK;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const TileCoord tc = decode_tile(t, p, BN);
            if (tc.skip) continue;
            const int32_t* Ih = (BMODE == kBGather && p.I) ? p.I + (int64_t)tc.h * p.I_stride : nullptr;
            const int32_t row_base = (tc.h / p.group) * p.b_head_rows;
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = it % C::STAGES;
                const uint32_t ph = (it / C::STAGES) & 1u;
                int32_t rows[4] = {0, 0, 0, 0};
                if constexpr (BMODE == kBGather) {
                    if (lane < 16) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int kidx = kb * C::BK + 4 * lane + i;
                            if (kidx < p.k) {
                                int32_t j = Ih ? __ldg(Ih + kidx) : kidx;  // no list: every index
                                j = min(max(j, 0), p.d - 1);
                                rows[i] = row_base + j;
                            } else {
                                rows[i] = p.b_rows_total;  // out of range: reads zeros
                            }
                        }
                    }
                }
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + s * C::STAGE_BYTES;
                uint8_t* sb = sa + C::A_BYTES;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
                    tma_load_3d(sa, &p.map_a, &full[s], kb * C::BK, tc.m0, tc.h);
                    if constexpr (BMODE == kBKMajor)
                        tma_load_3d(sb, &p.map_b, &full[s], kb * C::BK, tc.n0, tc.h / p.b_head_div);
                }
                __syncwarp();
                if constexpr (BMODE == kBGather) {
                    if (lane < 16) {
#pragma unroll
                        for (int g = 0; g < BN / 64; ++g)
                            tma_gather4(sb + g * C::GROUP_BYTES + lane * 4 * 128, &p.map_b, &full[s],
                                        tc.n0 + 64 * g, rows[0], rows[1], rows[2], rows[3]);
                    }
                } else if constexpr (BMODE == kBRows) {
                    if (lane < BN / 64)
                        tma_load_2d(sb + lane * C::GROUP_BYTES, &p.map_b, &full[s], tc.n0 + 64 * lane,
                                    row_base + kb * C::BK);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc(C::KIND, C::B_MN, BN);
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileCoord tc = decode_tile(t, p, BN);
                if (tc.skip) continue;
                const uint32_t acc = tcount & 1u;
                const uint32_t aph = (tcount >> 1) & 1u;
                if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, p.err, kErrTimeoutMma)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&full[s], ph, abort_flag, p.err, kErrTimeoutMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BK / C::UK; ++kk) {
                        const uint64_t adesc = sw128_desc(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = C::B_MN ? sw128_desc(b_addr + kk * C::UK * 128, C::GROUP_BYTES, 1024)
                                                       : sw128_desc(b_addr + kk * 32, 16, 1024);
                        umma<C::KIND>(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                ++tcount;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quadrant of this warp
        const int row_in_tile = q * 32 + lane;
        uint32_t tcount = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const TileCoord tc = decode_tile(t, p, BN);
            const int row = tc.m0 + row_in_tile;
            T* yrow = static_cast<T*>(p.Y) + (int64_t)tc.h * p.stride_y + (int64_t)row * p.ldy;
            if (tc.skip) {
                if (row < p.n) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = -__int_as_float(0x7f800000);
                    for (int ch = 0; ch < BN / 32; ++ch) store_chunk<T>(yrow, tc.n0 + ch * 32, p.m, v);
                }
                continue;
            }
            const uint32_t acc = tcount & 1u;
            const uint32_t aph = (tcount >> 1) & 1u;
            if (!mbar_wait(&tfull[acc], aph, abort_flag, p.err, kErrTimeoutEpilogue)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
#pragma unroll 1
            for (int ch = 0; ch < BN / 32; ++ch) {
                uint32_t raw[32];
                tmem_ld_32x32b_x32(taddr + ch * 32, raw);
                tmem_ld_wait();
                if (row < p.n) {
                    const int col0 = tc.n0 + ch * 32;
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float x = __uint_as_float(raw[i]) * p.alpha;
                        v[i] = (p.causal && col0 + i > row) ? -__int_as_float(0x7f800000) : x;
                    }
                    store_chunk<T>(yrow, col0, p.m, v);
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            ++tcount;
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ----------------------------------------------------------------------------
// CTA-pair variant (cluster of 2, tcgen05 cta_group::2).  The pair computes a
// 256 x BN tile: CTA r loads rows [m0 + 128 r, +128) of A and columns
// [n0 + (BN/2) r, +BN/2) of B into its own shared memory, and both count
// their TMA bytes on the leader's full barrier.  The leader's MMA thread
// issues M = 256 MMAs that read both CTAs' operands; each CTA's tensor memory
// receives its 128 rows x BN accumulator.  Stage releases and accumulator
// hand-offs are multicast commits to both CTAs; the peer's epilogue releases
// the accumulator with remote arrivals on the leader's barrier.  Halving B per
// CTA halves the shared-memory operand traffic of the 1-CTA 128 x BN tile.
// ----------------------------------------------------------------------------
template <typename T, int BMODE, int BN>
struct PairCfg {
    using TO = typename OutOf<T>::type;               // stored output type
    static constexpr int ES = sizeof(T);
    static constexpr bool TF32 = (ES == 4);
    static constexpr int KIND = KindOf<T>::value;
    static constexpr bool B_MN = (BMODE != kBKMajor);
    static constexpr int BK = 128 / ES;               // one 128-byte swizzle row of K
    static constexpr int UK = 32 / ES;                // K per tcgen05.mma (32 bytes)
    static constexpr int HALF_N = BN / 2;             // B columns held by one CTA
    static constexpr int A_BYTES = kBM * 128;         // 128 rows x 128 B
    static constexpr int B_BYTES = HALF_N * 128;      // BK rows x HALF_N (MN) or HALF_N rows x 128 B (K)
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = 6;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int GROUP_BYTES = BK * 128;      // one 128-byte-wide column group of an MN-major B tile
    static constexpr int GROUP_N = 128 / ES;          // B columns in one group
    // epilogue: EPI_WARPS warps, two per TMEM lane quadrant for a bf16 output
    // (each owns half of the tile's columns), with two staging buffers of 32 x 32 each
    static constexpr int EPI_WARPS = (sizeof(TO) == 2) ? 8 : 4;
    static constexpr int NT = 32 * (2 + EPI_WARPS);
    static constexpr int ROW_BYTES = 32 * (int)sizeof(TO);    // 64 (bf16) or 128 (fp32)
    static constexpr int OUT_BUF = 32 * ROW_BYTES;
    static constexpr int OUT_BYTES = EPI_WARPS * 2 * OUT_BUF;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + OUT_BYTES + 256;
    static_assert(!(TF32 && B_MN), "fp32 operands are staged K-major");
    static_assert(BMODE != kBGather, "indexed gathers use the single-CTA kernel");
};

// Write one thread's 32 output values (its row of a 32 x 32 chunk) into the
// staging buffer in the layout of a 64-byte (bf16) or 128-byte (fp32)
// swizzled TMA box: 16-byte granule g of row r sits at g ^ f(r).
template <typename T>
__device__ __forceinline__ void stage_row(uint8_t* buf, int r, const float (&v)[32]) {
    uint8_t* row = buf + r * (32 * (int)sizeof(T));
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * g + 2 * i], v[8 * g + 2 * i + 1]);
                w[i] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(row + ((g ^ ((r >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
#pragma unroll
        for (int g = 0; g < 8; ++g)
            *reinterpret_cast<float4*>(row + ((g ^ (r & 7)) << 4)) =
                make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
    }
}

// Tile order of the CTA-pair kernel: within a head, groups of p.group_m
// consecutive 256-row tiles sweep every column tile before the next group, so
// that the A rows of a group stay resident in L2 while B streams past.
__device__ __forceinline__ void pair_tile(int t, const GemmParams& p, int& h, int& mt, int& nt) {
    if (p.causal_k) {
        // row tiles carry K-work in proportion to their last row: visit every
        // head's last row tile first, so that the round-robin over the pairs
        // deals each pair one tile of every size band
        const int band = p.heads * p.n_tiles;
        mt = p.m_tiles - 1 - t / band;
        const int r = t - (t / band) * band;
        h = r / p.n_tiles;
        nt = r - h * p.n_tiles;
        return;
    }
    const int per_head = p.m_tiles * p.n_tiles;
    h = t / per_head;
    const int r = t - h * per_head;
    const int G = p.group_m;
    const int group = r / (G * p.n_tiles);
    const int within = r - group * (G * p.n_tiles);
    const int left = p.m_tiles - group * G;
    const int gm = left < G ? left : G;
    mt = group * G + within % gm;
    nt = within / gm;
}

// Work unit of the CTA-pair kernel: a whole tile, or K-part `part` of one of
// the split tail tiles (k-blocks [kb0, kb1)).  Units before `whole` are the
// tiles of the same index; the split tail follows, part-major within a tile.
struct PairUnit {
    int t, kb0, kb1, part;  // part < 0: whole tile
};

template <bool SPLIT>
__device__ __forceinline__ PairUnit pair_unit(int u, int whole, int num_kb, const GemmParams& p) {
    PairUnit w;
    if (!SPLIT || u < whole) {
        w.t = u;
        w.kb0 = 0;
        w.kb1 = num_kb;
        w.part = -1;
    } else {
        const int v = u - whole;
        w.t = whole + v / p.split_f;
        w.part = v - (v / p.split_f) * p.split_f;
        w.kb0 = w.part * num_kb / p.split_f;
        w.kb1 = (w.part + 1) * num_kb / p.split_f;
    }
    return w;
}

// End of a unit's K loop: with a causal A (A[i][j] = 0 for j > i, the K axis
// on the rows' positions), the k-blocks past the pair tile's last row are
// zero and skipped.  Causal problems have no split tail.
template <int BK>
__device__ __forceinline__ int pair_kb_end(const GemmParams& p, const PairUnit& w, int m0) {
    if (!p.causal_k) return w.kb1;
    const int last = (m0 + 2 * kBM + BK - 1) / BK;
    return last < w.kb1 ? last : w.kb1;
}

// Epilogue of one K-part of a split tail tile, for one warp (its 32 rows x
// the chunks ch = half, half + H, ...; TMEM address taddr).  The part's raw
// fp32 accumulator goes to the workspace in chunk layout [ch][g][lane][4];
// after a fence the warp counts the part, and the warp that counts the last
// one adds the parts in part order (0, 1, ..., f - 1, so every call gives the
// same bits), scales by alpha and stores the tile through the staging
// buffers (slot: the next staging buffer; returns the one after the stores).
// Split tails are planned only without the causal mask.  Kept out of line so
// that it does not shape the whole-tile epilogue's code.
template <typename T, int BN, int H>
__device__ __noinline__ uint32_t split_part_epilogue(const GemmParams& p, uint32_t taddr, int si, int part, int rank,
                                                     int q, int e, int half, int n0, int row0, int h, uint8_t* out,
                                                     uint32_t slot) {
    constexpr int OUT_BUF = 32 * 32 * (int)sizeof(T);
    const int lane = threadIdx.x & 31;
    const size_t tile_floats = (size_t)2 * kBM * BN;
    float* parts = p.split_partials + (size_t)si * p.split_f * tile_floats + ((size_t)rank * kBM + (size_t)q * 32) * BN;
#pragma unroll 1
    for (int ch = half; ch < BN / 32; ch += H) {
        if (n0 + ch * 32 >= p.m) break;
        uint32_t raw[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, raw);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(parts + (size_t)part * tile_floats + ch * 1024) + lane;
#pragma unroll
        for (int g = 0; g < 8; ++g)
            __stcg(dst + g * 32, make_float4(__uint_as_float(raw[4 * g]), __uint_as_float(raw[4 * g + 1]),
                                             __uint_as_float(raw[4 * g + 2]), __uint_as_float(raw[4 * g + 3])));
    }
    __syncwarp();
    unsigned* cnt = p.split_counters + ((size_t)si * 2 + rank) * kSplitCounterWarps + e;
    unsigned done = 0;
    if (lane == 0) {
        __threadfence();  // this part's stores before its count
        done = atomicAdd(cnt, 1u);
    }
    done = __shfl_sync(0xffffffffu, done, 0);
    if (done != (unsigned)(p.split_f - 1)) return slot;
    if (lane == 0) atomicExch(cnt, 0u);  // ready for the next launch
    __threadfence();                     // the other parts' stores after their counts
#pragma unroll 1
    for (int ch = half; ch < BN / 32; ch += H) {
        const int col0 = n0 + ch * 32;
        if (col0 >= p.m) break;
        uint32_t raw[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, raw);
        tmem_ld_wait();
        float v[32];
#pragma unroll 1
        for (int j = 0; j < p.split_f; ++j) {
            const float4* src = reinterpret_cast<const float4*>(parts + (size_t)j * tile_floats + ch * 1024) + lane;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const float4 x = j == part ? make_float4(__uint_as_float(raw[4 * g]), __uint_as_float(raw[4 * g + 1]),
                                                         __uint_as_float(raw[4 * g + 2]), __uint_as_float(raw[4 * g + 3]))
                                           : __ldcg(src + g * 32);
                v[4 * g] = j == 0 ? x.x : v[4 * g] + x.x;
                v[4 * g + 1] = j == 0 ? x.y : v[4 * g + 1] + x.y;
                v[4 * g + 2] = j == 0 ? x.z : v[4 * g + 2] + x.z;
                v[4 * g + 3] = j == 0 ? x.w : v[4 * g + 3] + x.w;
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= p.alpha;
        uint8_t* buf = out + slot * OUT_BUF;
        if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read it
        __syncwarp();
        stage_row<T>(buf, lane, v);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(&p.map_y, buf, col0, row0, h);
            bulk_commit_group();
        }
        slot ^= 1u;
    }
    return slot;
}

// ----------------------------------------------------------------------------
// Producer-fused scoring (see GemmParams::emit_s2).
// ----------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float stored_value(float x) {
    if constexpr (sizeof(T) == 2)
        return __bfloat162float(__float2bfloat16_rn(x));
    else
        return x;
}

// Row group rg's sum for columns [col0, col0 + 32) (lane = column) goes to the
// workspace; the warp that completes the chunk's row groups adds them in
// row-group order into emit_s2 and resets the chunk's counter.
__device__ __noinline__ void emit_scores_chunk(const GemmParams& p, float colsum, int h, int rg, int col0) {
    const int lane = threadIdx.x & 31;
    const int rgs = 8 * p.m_tiles;
    const bool in = col0 + lane < p.m;
    float* base = p.emit_partials + (int64_t)h * rgs * p.m + col0 + lane;
    if (in) __stcg(base + (int64_t)rg * p.m, colsum);
    __threadfence();
    __syncwarp();
    unsigned* cnt = p.emit_counters + (int64_t)h * p.n_tiles * 8 + col0 / 32;
    unsigned done = 0;
    if (lane == 0) done = atomicAdd(cnt, 1u);
    done = __shfl_sync(0xffffffffu, done, 0);
    if (done != (unsigned)(rgs - 1)) return;
    if (lane == 0) atomicExch(cnt, 0u);  // ready for the next launch
    __threadfence();                     // the other row groups' sums after their counts
    if (in) {
        float z = 0.f;
        for (int g = 0; g < rgs; ++g) z += __ldcg(base + (int64_t)g * p.m);
        p.emit_s2[(int64_t)h * p.m + col0 + lane] = z;
    }
}

// K loops of at most this many k-blocks make every epilogue warp poll the
// accumulator barrier itself.
constexpr int kAllPollMaxKb = 16;

// Optional parts of the CTA-pair kernel, compiled in only where a plan uses
// them (the plain kernel keeps the hot loops of its first form).
constexpr int kFeatEmit = 1;  // column scores of the stored output (GemmParams::emit_s2)
constexpr int kFeatSkip = 2;  // k-blocks without a kept index skipped (GemmParams::kb_keep)

template <typename T, int BMODE, int BN, bool SPLIT, int FEAT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<T, BMODE, BN>::NT, 1)
    pair_gemm_kernel(const __grid_constant__ GemmParams p) {
    using C = PairCfg<T, BMODE, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::OUT_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* epi_go = reinterpret_cast<volatile int*>(tmem_holder + 2);  // accumulator ready (epilogue)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);   // the leader's expect_tx arrival (+ both CTAs' bytes)
            mbar_init(&empty[s], 1);  // one multicast commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);   // one multicast commit
            mbar_init(&tempty[a], 2 * C::EPI_WARPS);  // epilogue warps of both CTAs (used in the leader)
        }
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_map(&p.map_a);
        tma_prefetch_map(&p.map_b);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_wait();  // everything above touched only shared and tensor memory
    pdl_trigger();

    const int total = p.heads * p.m_tiles * p.n_tiles;  // 256-row tiles
    const int num_kb = (p.k + C::BK - 1) / C::BK;
    const int whole = SPLIT ? total - p.split_tiles : total;
    const int units = SPLIT ? whole + p.split_tiles * p.split_f : total;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int u = cluster; u < units && ok; u += nclusters) {
                const PairUnit w = pair_unit<SPLIT>(u, whole, num_kb, p);
                int h, mt, nt;
                pair_tile(w.t, p, h, mt, nt);
                const int m0 = mt * 2 * kBM, n0 = nt * BN;
                if (p.causal && n0 > m0 + 2 * kBM - 1) continue;
                const int row_base = (h / p.group) * p.b_head_rows;
                const int kb_hi = pair_kb_end<C::BK>(p, w, m0);
                const uint8_t* keep = (FEAT & kFeatSkip) ? p.kb_keep + (int64_t)h * p.kb_keep_stride : nullptr;
                for (int kb = w.kb0; kb < kb_hi; ++kb) {
                    if constexpr (FEAT & kFeatSkip)
                        if (kb != w.kb0 && !keep[kb]) continue;  // no kept index in this k-block
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    ++it;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
                    tma_load_3d_pair(sa, &p.map_a, bar, kb * C::BK, m0 + (int)rank * kBM, h);
                    if constexpr (BMODE == kBKMajor) {
                        tma_load_3d_pair(sb, &p.map_b, bar, kb * C::BK, n0 + (int)rank * C::HALF_N,
                                         h / p.b_head_div);
                    } else {
#pragma unroll
                        for (int g = 0; g < C::HALF_N / C::GROUP_N; ++g)
                            tma_load_2d_pair(sb + g * C::GROUP_BYTES, &p.map_b, bar,
                                             n0 + (int)rank * C::HALF_N + C::GROUP_N * g, row_base + kb * C::BK);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = umma_idesc(C::KIND, C::B_MN, BN, 256);
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int u = cluster; u < units && ok; u += nclusters) {
                const PairUnit w = pair_unit<SPLIT>(u, whole, num_kb, p);
                int h, mt, nt;
                pair_tile(w.t, p, h, mt, nt);
                const int m0 = mt * 2 * kBM, n0 = nt * BN;
                if (p.causal && n0 > m0 + 2 * kBM - 1) continue;
                const uint32_t acc = tcount & 1u;
                const uint32_t aph = (tcount >> 1) & 1u;
                if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, p.err, kErrTimeoutMma)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                const int kb_hi = pair_kb_end<C::BK>(p, w, m0);
                const uint8_t* keep = (FEAT & kFeatSkip) ? p.kb_keep + (int64_t)h * p.kb_keep_stride : nullptr;
                for (int kb = w.kb0; kb < kb_hi; ++kb) {
                    if constexpr (FEAT & kFeatSkip)
                        if (kb != w.kb0 && !keep[kb]) continue;  // the producer skips it too
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    ++it;
                    if (!mbar_wait(&full[s], ph, abort_flag, p.err, kErrTimeoutMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BK / C::UK; ++kk) {
                        const uint64_t adesc = sw128_desc(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = C::B_MN ? sw128_desc(b_addr + kk * C::UK * 128, C::GROUP_BYTES, 1024)
                                                       : sw128_desc(b_addr + kk * 32, 16, 1024);
                        umma_pair<C::KIND>(d_tmem, adesc, bdesc, idesc, (kb != w.kb0 || kk != 0) ? 1u : 0u);
                    }
                    umma_commit_pair(&empty[s], 0x3);
                }
                if (!ok) break;
                umma_commit_pair(&tfull[acc], 0x3);
                ++tcount;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        // Warp e (of EPI_WARPS) owns TMEM lane quadrant q = (warp % 4), i.e. 32
        // rows, and column chunks ch = half, half + H, ... of the tile (H = number
        // of warps per quadrant).  Per 32-column chunk it stages its rows in a
        // swizzled shared buffer and one lane stores the 32 x 32 box by TMA (rows
        // past n and columns past m are clipped by the store itself).  Tiles the
        // causal mask covers entirely store one -inf buffer repeatedly.
        constexpr int H = C::EPI_WARPS / 4;
        const int e = warp - 2;
        const int q = warp & 3;
        const int half = e / 4;
        const int row_base = (int)rank * kBM + q * 32;
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
        const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
        uint8_t* out = smem + C::STAGES * C::STAGE_BYTES + (e * 2) * C::OUT_BUF;
        uint32_t tcount = 0, slot = 0;
        // Stage one thread's 32 values of a 32 x 32 chunk and store the chunk by TMA.
        auto emit = [&](const float (&v)[32], int col0, int row0, int h) {
            uint8_t* buf = out + slot * C::OUT_BUF;
            if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read it
            __syncwarp();
            stage_row<typename C::TO>(buf, lane, v);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(&p.map_y, buf, col0, row0, h);
                bulk_commit_group();
            }
            slot ^= 1u;
        };
        for (int u = cluster; u < units; u += nclusters) {
            const PairUnit w = pair_unit<SPLIT>(u, whole, num_kb, p);
            int h, mt, nt;
            pair_tile(w.t, p, h, mt, nt);
            const int m0 = mt * 2 * kBM, n0 = nt * BN;
            const int row0 = m0 + row_base;
            const int row = row0 + lane;
            const bool skip = p.causal && n0 > m0 + 2 * kBM - 1;
            uint32_t acc = 0, taddr = 0;
            if (!skip) {
                acc = tcount & 1u;
                const uint32_t aph = (tcount >> 1) & 1u;
                if (pair_kb_end<C::BK>(p, w, m0) - w.kb0 <= kAllPollMaxKb) {
                    // short K loop: the epilogue is the critical path, every warp polls
                    if (!mbar_wait(&tfull[acc], aph, abort_flag, p.err, kErrTimeoutEpilogue)) break;
                } else {
                    // long K loop: one warp polls so that the others leave the issue
                    // slots to the producer and MMA warps; they sleep on a named barrier
                    if (e == 0) *epi_go = mbar_wait(&tfull[acc], aph, abort_flag, p.err, kErrTimeoutEpilogue) ? 1 : 0;
                    asm volatile("bar.sync 1, %0;" ::"n"(32 * C::EPI_WARPS) : "memory");
                    if (!*epi_go) break;
                }
                tc_fence_after();
                taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            }
            if (SPLIT && row0 < p.n && w.part >= 0) {
                slot = split_part_epilogue<typename C::TO, BN, H>(p, taddr, w.t - whole, w.part, (int)rank, q, e, half, n0, row0,
                                                     h, out, slot);
            } else if (row0 < p.n) {
                bool inf_staged = false;
#pragma unroll 1
                for (int ch = half; ch < BN / 32; ch += H) {
                    const int col0 = n0 + ch * 32;
                    if (col0 >= p.m) break;
                    if (skip) {
                        uint8_t* buf = out + slot * C::OUT_BUF;
                        if (!inf_staged) {
                            float v[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = -__int_as_float(0x7f800000);
                            if (lane == 0) bulk_wait_group_read<0>();
                            __syncwarp();
                            stage_row<typename C::TO>(buf, lane, v);
                            fence_proxy_async_smem();
                            __syncwarp();
                            inf_staged = true;
                        }
                        if (lane == 0) {
                            tma_store_3d(&p.map_y, buf, col0, row0, h);
                            bulk_commit_group();
                        }
                        continue;  // the same buffer serves every chunk of the tile
                    }
                    uint32_t raw[32];
                    tmem_ld_32x32b_x32(taddr + ch * 32, raw);
                    float v[32];
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float x = __uint_as_float(raw[i]) * p.alpha;
                        v[i] = (p.causal && col0 + i > row) ? -__int_as_float(0x7f800000) : x;
                    }
                    emit(v, col0, row0, h);
                    if constexpr (FEAT & kFeatEmit) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const float y = stored_value<typename C::TO>(v[i]);
                            v[i] = row < p.n ? y * y : 0.f;
                        }
                        emit_scores_chunk(p, warp_column_sums(v, lane), h, (mt * 2 + (int)rank) * 4 + q, col0);
                    }
                }
                if (skip && inf_staged) slot ^= 1u;  // the -inf buffer may still be read: use the other one next
            } else if ((FEAT & kFeatEmit) && !skip) {
                // no rows of this warp's slice exist: its row group adds zeros
#pragma unroll 1
                for (int ch = half; ch < BN / 32; ch += H) {
                    const int col0 = n0 + ch * 32;
                    if (col0 >= p.m) break;
                    emit_scores_chunk(p, 0.f, h, (mt * 2 + (int)rank) * 4 + q, col0);
                }
            }
            if (!skip) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
                ++tcount;
            }
        }
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // both CTAs done with each other's shared and tensor memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

template <typename T, int BMODE, int BN, bool SPLIT, int FEAT>
cudaError_t launch_pair_inst(const GemmParams& p, int num_sms, cudaStream_t s) {
    using C = PairCfg<T, BMODE, BN>;
    auto kern = pair_gemm_kernel<T, BMODE, BN, SPLIT, FEAT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    const int total = p.heads * p.m_tiles * p.n_tiles;
    const int units = total - p.split_tiles + p.split_tiles * p.split_f;
    const int clusters = units < num_sms / 2 ? units : num_sms / 2;
    if (clusters <= 0) return cudaSuccess;
    return launch_pdl(kern, dim3(2 * clusters), dim3(C::NT), C::SMEM, s, p);
}

// The instantiation a launch needs: split tail or not, emission (never with a
// split tail) and block skipping (bf16 row tiles only) as the plan set them.
template <typename T, int BMODE, int BN>
cudaError_t launch_pair(const GemmParams& p, int num_sms, cudaStream_t s) {
    const bool split = p.split_tiles > 0, emit = p.emit_s2 != nullptr, skip = p.kb_keep != nullptr;
    if (emit && split) return cudaErrorInvalidValue;
    if constexpr (BMODE == kBRows) {
        if (skip && emit) return launch_pair_inst<T, BMODE, BN, false, kFeatEmit | kFeatSkip>(p, num_sms, s);
        if (skip) return split ? launch_pair_inst<T, BMODE, BN, true, kFeatSkip>(p, num_sms, s)
                               : launch_pair_inst<T, BMODE, BN, false, kFeatSkip>(p, num_sms, s);
    } else {
        if (skip) return cudaErrorInvalidValue;
    }
    if (emit) return launch_pair_inst<T, BMODE, BN, false, kFeatEmit>(p, num_sms, s);
    return split ? launch_pair_inst<T, BMODE, BN, true, 0>(p, num_sms, s)
                 : launch_pair_inst<T, BMODE, BN, false, 0>(p, num_sms, s);
}

template <typename T, int BMODE, int BN>
cudaError_t launch_one(const GemmParams& p, int num_sms, cudaStream_t s) {
    using C = Cfg<T, BMODE, BN>;
    auto kern = gather_gemm_kernel<T, BMODE, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    const int total = p.heads * p.m_tiles * p.n_tiles;
    const int grid = total < num_sms ? total : num_sms;
    if (grid <= 0) return cudaSuccess;
    return launch_pdl(kern, dim3(grid), dim3(kThreads), C::SMEM, s, p);
}

template <typename T, int BMODE>
cudaError_t launch_bn(const GemmParams& p, const GemmLaunch& l, cudaStream_t s) {
    return l.bn == 256 ? launch_one<T, BMODE, 256>(p, l.num_sms, s) : launch_one<T, BMODE, 128>(p, l.num_sms, s);
}

}  // namespace

void pair_split_tail(int64_t tiles, int64_t num_kb, int clusters, int* split_tiles, int* split_f) {
    *split_tiles = 0;
    *split_f = 1;
    if (tiles <= 0 || clusters <= 0) return;
    // The last wave holds tiles % clusters tiles; cut each into f K-parts so
    // that the f-fold units still fit one wave, with at least 8 k-blocks a part.
    const int64_t rem = tiles % clusters;
    if (rem == 0) return;
    int64_t f = clusters / rem;
    if (f > 4) f = 4;
    if (f > num_kb / 8) f = num_kb / 8;
    if (f < 2) return;
    *split_tiles = static_cast<int>(rem);
    *split_f = static_cast<int>(f);
}

size_t gemm_smem_bytes(int dtype, int bn, bool pair) {
    if (dtype == 2)
        return bn == 256 ? PairCfg<__nv_fp8_e4m3, kBRows, 256>::SMEM : PairCfg<__nv_fp8_e4m3, kBRows, 128>::SMEM;
    if (pair) {
        if (dtype == 1) return bn == 256 ? PairCfg<float, kBKMajor, 256>::SMEM : PairCfg<float, kBKMajor, 128>::SMEM;
        return bn == 256 ? PairCfg<__nv_bfloat16, kBRows, 256>::SMEM : PairCfg<__nv_bfloat16, kBRows, 128>::SMEM;
    }
    if (dtype == 1) return bn == 256 ? Cfg<float, kBKMajor, 256>::SMEM : Cfg<float, kBKMajor, 128>::SMEM;
    return bn == 256 ? Cfg<__nv_bfloat16, kBGather, 256>::SMEM : Cfg<__nv_bfloat16, kBGather, 128>::SMEM;
}

cudaError_t launch_gemm(const GemmParams& p, const GemmLaunch& l, cudaStream_t s) {
    if (l.dtype == 2) {  // E4M3 operands: CTA pairs, B as rows (MN-major)
        if (!l.pair || l.b_mode != kBRows) return cudaErrorInvalidValue;
        return l.bn == 256 ? launch_pair<__nv_fp8_e4m3, kBRows, 256>(p, l.num_sms, s)
                           : launch_pair<__nv_fp8_e4m3, kBRows, 128>(p, l.num_sms, s);
    }
    if (l.pair) {
        if (l.dtype == 1) {
            if (l.b_mode != kBKMajor) return cudaErrorInvalidValue;
            return l.bn == 256 ? launch_pair<float, kBKMajor, 256>(p, l.num_sms, s)
                               : launch_pair<float, kBKMajor, 128>(p, l.num_sms, s);
        }
        if (l.b_mode == kBRows)
            return l.bn == 256 ? launch_pair<__nv_bfloat16, kBRows, 256>(p, l.num_sms, s)
                               : launch_pair<__nv_bfloat16, kBRows, 128>(p, l.num_sms, s);
        if (l.b_mode == kBKMajor)
            return l.bn == 256 ? launch_pair<__nv_bfloat16, kBKMajor, 256>(p, l.num_sms, s)
                               : launch_pair<__nv_bfloat16, kBKMajor, 128>(p, l.num_sms, s);
        return cudaErrorInvalidValue;
    }
    if (l.dtype == 1) {
        if (l.b_mode != kBKMajor) return cudaErrorInvalidValue;
        return launch_bn<float, kBKMajor>(p, l, s);
    }
    switch (l.b_mode) {
        case kBGather: return launch_bn<__nv_bfloat16, kBGather>(p, l, s);
        case kBRows: return launch_bn<__nv_bfloat16, kBRows>(p, l, s);
        default: return launch_bn<__nv_bfloat16, kBKMajor>(p, l, s);
    }
}

}  // namespace rmm
