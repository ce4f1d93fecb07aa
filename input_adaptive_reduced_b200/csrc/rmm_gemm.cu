// rmm_gemm.cu -- the reduced product of Reduced Matrix Multiplication on the
// B200 tensor cores: Y = A[:, I] B[I, :] ("Reduced Matrix Multiplication:
// Input-Adaptive Matrix-Product Reduction for LLM Inference", §3.2; per-head
// attention forms in §3.3; cost O(n k m) in §3.4 and Appendix D.1 Eq. (1)-(4)).
//
// Design (sm_100a, one CTA per SM, persistent over 128 x BN output tiles):
//   warps 0-3  producer: the A tile (packed A[:, I], K-major) arrives by TMA;
//              B is either gathered row by row through the index set with
//              16-byte cp.async into the 128-byte-swizzled MN-major layout
//              (LINEAR / PV: B[I, :] rows are contiguous), or arrives by TMA
//              as a K-major tile (QK: packed K[:, I]).
//   warp  8    MMA issuer: one thread issues tcgen05.mma (kind::f16 for bf16,
//              kind::tf32 for fp32) into a double-buffered fp32 accumulator in
//              tensor memory and commits stage releases to mbarriers.
//   warps 4-7  epilogue: tcgen05.ld of the accumulator (one TMEM lane quadrant
//              per warp), alpha scaling, the causal -inf mask, rounding to the
//              storage dtype and 16-byte global stores.  Tiles that the causal
//              mask covers entirely skip the MMA and store -inf directly.
// Every wait is bounded (rmm_device.cuh); on expiry the kernel records an
// error word and returns.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kThreads = 288;  // 9 warps
constexpr int kBM = 128;

template <typename T, int BN>
struct Cfg {
    static constexpr int ES = sizeof(T);
    static constexpr bool TF32 = (ES == 4);
    static constexpr int BK = 128 / ES;        // one 128-byte swizzle row of K
    static constexpr int UK = 32 / ES;         // K per tcgen05.mma
    static constexpr int A_BYTES = kBM * 128;  // 128 rows x 128 B
    static constexpr int B_BYTES = BN * 128;   // BK rows x BN cols (gather) or BN rows x 128 B (TMA)
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (BN == 256) ? 4 : 6;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int CPR = BN * ES / 16;   // 16-byte chunks per gathered B row
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
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

template <typename T, bool B_GATHER, int BN>
__global__ void __launch_bounds__(kThreads, 1) gather_gemm_kernel(const __grid_constant__ GemmParams p) {
    using C = Cfg<T, BN>;
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
            mbar_init(&full[s], B_GATHER ? 128 + 1 : 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_map(&p.map_a);
        if (!B_GATHER) tma_prefetch_map(&p.map_b);
    }
    if (warp == 8) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int total = p.heads * p.m_tiles * p.n_tiles;
    const int num_kb = (p.k + C::BK - 1) / C::BK;

    if (warp < 4) {
        // ------------------------------------------------------------ producer
        const int tid = threadIdx.x;
        if (B_GATHER || tid == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileCoord tc = decode_tile(t, p, BN);
                if (tc.skip) continue;
                const T* Bh = nullptr;
                const int32_t* Ih = nullptr;
                if constexpr (B_GATHER) {
                    Bh = static_cast<const T*>(p.B) + (int64_t)(tc.h / p.group) * p.stride_b;
                    Ih = p.I ? p.I + (int64_t)tc.h * p.I_stride : nullptr;
                }
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    if (tid == 0) {
                        mbar_arrive_expect_tx(&full[s], B_GATHER ? C::A_BYTES : C::A_BYTES + C::B_BYTES);
                        tma_load_3d(sa, &p.map_a, &full[s], kb * C::BK, tc.m0, tc.h);
                        if constexpr (!B_GATHER)
                            tma_load_3d(sb, &p.map_b, &full[s], kb * C::BK, tc.n0, tc.h / p.b_head_div);
                    }
                    if constexpr (B_GATHER) {
                        const uint32_t sb_addr = smem_u32(sb);
#pragma unroll 4
                        for (int c = tid; c < C::BK * C::CPR; c += 128) {
                            const int r = c / C::CPR;
                            const int cc = c % C::CPR;
                            const int kidx = kb * C::BK + r;
                            const bool kvalid = kidx < p.k;
                            int row = kvalid ? (Ih ? __ldg(Ih + kidx) : kidx) : 0;
                            row = min(max(row, 0), p.d - 1);
                            const int gcol = tc.n0 + cc * (16 / C::ES);
                            const bool cvalid = gcol < p.m;
                            const T* src = Bh + (int64_t)row * p.ldb + (cvalid ? gcol : 0);
                            const uint32_t dst = sb_addr + (cc >> 3) * (C::BK * 128) + r * 128 +
                                                 (((cc & 7) ^ (r & 7)) << 4);
                            cp_async_16(dst, src, (kvalid && cvalid) ? 16u : 0u);
                        }
                        cp_async_arrive_noinc(&full[s]);
                    }
                }
            }
            if constexpr (B_GATHER) cp_async_wait_all();
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc(C::TF32, B_GATHER, BN);
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
                    fence_proxy_async_smem();
                    const uint32_t a_addr = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BK / C::UK; ++kk) {
                        const uint64_t adesc = sw128_desc(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = B_GATHER
                                                   ? sw128_desc(b_addr + kk * C::UK * 128, C::BK * 128, 1024)
                                                   : sw128_desc(b_addr + kk * 32, 16, 1024);
                        umma<C::TF32>(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
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
    if (warp == 8) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <typename T, bool G, int BN>
cudaError_t launch_one(const GemmParams& p, int num_sms, cudaStream_t s) {
    using C = Cfg<T, BN>;
    auto kern = gather_gemm_kernel<T, G, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    const int total = p.heads * p.m_tiles * p.n_tiles;
    const int grid = total < num_sms ? total : num_sms;
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kThreads, C::SMEM, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t gemm_smem_bytes(int dtype, int bn) {
    if (dtype == 1) return bn == 256 ? Cfg<float, 256>::SMEM : Cfg<float, 128>::SMEM;
    return bn == 256 ? Cfg<__nv_bfloat16, 256>::SMEM : Cfg<__nv_bfloat16, 128>::SMEM;
}

cudaError_t launch_gemm(const GemmParams& p, const GemmLaunch& l, cudaStream_t s) {
    if (l.dtype == 1) {
        if (l.b_gather)
            return l.bn == 256 ? launch_one<float, true, 256>(p, l.num_sms, s)
                               : launch_one<float, true, 128>(p, l.num_sms, s);
        return l.bn == 256 ? launch_one<float, false, 256>(p, l.num_sms, s)
                           : launch_one<float, false, 128>(p, l.num_sms, s);
    }
    if (l.b_gather)
        return l.bn == 256 ? launch_one<__nv_bfloat16, true, 256>(p, l.num_sms, s)
                           : launch_one<__nv_bfloat16, true, 128>(p, l.num_sms, s);
    return l.bn == 256 ? launch_one<__nv_bfloat16, false, 256>(p, l.num_sms, s)
                       : launch_one<__nv_bfloat16, false, 128>(p, l.num_sms, s);
}

}  // namespace rmm
