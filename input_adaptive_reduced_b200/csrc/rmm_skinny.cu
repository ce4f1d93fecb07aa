// rmm_skinny.cu -- the reduced product for few rows (n <= 64: decode-sized
// token counts), where the op is a stream of the retained rows of B
// ("Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
// LLM Inference", §3.2; the per-step reselection of Appendix A makes every
// decode step pay it).
//
// Yᵀ = B[I, :]ᵀ A[:, I]ᵀ is computed with the operands swapped: the MMA's
// M = 128 runs over output columns, so the gathered rows B[I, m0:m0+128]
// form an MN-major operand that 8 cp.async warps land straight from B through
// the index set (no staging copy; this kernel is bound by the HBM read of
// B[I, :]), and the packed A[:, I] (n rows padded to NP) is a K-major TMA
// operand.  The contraction is split over CTAs so that every SM streams; each
// split writes fp32 partials and a second kernel adds them in split order.
//
//   warp 0      TMA producer of the A[:, I] tile (expect_tx on the stage)
//   warp 1      TMEM allocation and the MMA issuer (one thread)
//   warps 2-5   epilogue: tcgen05.ld of the 128 x NP accumulator
//   warps 6-13  cp.async gather of 64 retained B rows x 128 columns per stage
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kSkThreads = 448;
constexpr int kSkBK = 64;                     // bf16 K per stage (one 128-byte row)
constexpr int kSkGatherBytes = kSkBK * 256;   // 64 rows x 128 columns x 2 B
constexpr int kSkGroupBytes = kSkBK * 128;    // one 64-column group

constexpr int kSkMaxSplitIdx = 4096;          // indices of one split staged in shared memory

template <int NP>
struct SkCfg {
    static constexpr int A_BYTES = NP * 128;  // the A[:, I] tile: NP rows x 128 B
    static constexpr int STAGE_BYTES = kSkGatherBytes + A_BYTES;
    // two CTAs per SM (16 gather warps per SM): 4 stages, 3 when NP = 64
    static constexpr int STAGES = NP == 64 ? 3 : 4;
    static constexpr int TMEM_COLS = NP < 32 ? 32 : NP;
    static constexpr size_t IDX_OFF = (size_t)STAGES * STAGE_BYTES + 256;
    static constexpr size_t SMEM = 1024 + IDX_OFF + kSkMaxSplitIdx * 4;
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15])
        : "r"(taddr));
}

template <int NP>
__global__ void __launch_bounds__(kSkThreads, 2) skinny_kernel(const __grid_constant__ SkinnyParams p) {
    using C = SkCfg<NP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x % p.m_tiles;
    const int split = blockIdx.x / p.m_tiles;
    const int m0 = mt * 128;
    const int nkb = (p.k + kSkBK - 1) / kSkBK;
    const int kb_beg = (int)((int64_t)nkb * split / p.splits);
    const int kb_end = (int)((int64_t)nkb * (split + 1) / p.splits);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1 + 256);  // expect_tx arrival + 256 cp.async arrivals
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_map(&p.map_a);
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
    // this split's retained row indices, staged once (-1 past k)
    int32_t* sidx = reinterpret_cast<int32_t*>(smem + C::IDX_OFF);
    if (warp >= 6) {
        const int ptid = threadIdx.x - 6 * 32;
        const int t0 = kb_beg * kSkBK, cnt = (kb_end - kb_beg) * kSkBK;
        for (int t = ptid; t < cnt; t += 256) {
            const int kidx = t0 + t;
            int32_t j = -1;
            if (kidx < p.k) {
                j = p.I ? __ldg(p.I + kidx) : kidx;
                j = min(max(j, 0), p.d - 1);
            }
            sidx[t] = j;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the gather warps only
    }

    if (warp == 0) {
        if (lane == 0) {
            for (int kb = kb_beg, it = 0; kb < kb_end; ++kb, ++it) {
                const int s = it % C::STAGES;
                const uint32_t ph = (it / C::STAGES) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) break;
                uint8_t* sa = smem + s * C::STAGE_BYTES + kSkGatherBytes;
                mbar_arrive_expect_tx(&full[s], C::A_BYTES);
                tma_load_3d(sa, &p.map_a, &full[s], kb * kSkBK, 0, 0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // M = 128 (output columns, MN-major gathered rows), N = NP (tokens, K-major)
            constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                                       ((uint32_t)(NP >> 3) << 17) | ((128u >> 4) << 24);
            bool ok = true;
            for (int kb = kb_beg, it = 0; kb < kb_end; ++kb, ++it) {
                const int s = it % C::STAGES;
                const uint32_t ph = (it / C::STAGES) & 1u;
                if (!mbar_wait(&full[s], ph, abort_flag, p.err, kErrTimeoutMma)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                fence_proxy_async_smem();
                const uint32_t g_addr = smem_u32(smem + s * C::STAGE_BYTES);
                const uint32_t a_addr = g_addr + kSkGatherBytes;
#pragma unroll
                for (int kk = 0; kk < kSkBK / 16; ++kk) {
                    const uint64_t mdesc = sw128_desc(g_addr + kk * 16 * 128, kSkGroupBytes, 1024);
                    const uint64_t ndesc = sw128_desc(a_addr + kk * 32, 16, 1024);
                    umma<kKindF16>(tmem_base, mdesc, ndesc, idesc, (kb > kb_beg || kk > 0) ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            if (ok) umma_commit(tfull);
        }
    } else if (warp < 6) {
        // epilogue: lane row = output column m0 + 32 q + lane, columns = tokens
        const int q = warp & 3;
        const int col = m0 + q * 32 + lane;
        const bool any_k = kb_end > kb_beg;
        if (!any_k || mbar_wait(tfull, 0, abort_flag, p.err, kErrTimeoutEpilogue)) {
            tc_fence_after();
            // 16 tokens at a time: TMEM columns c16*16 .. +15 of this lane's row
#pragma unroll 1
            for (int c16 = 0; c16 < NP / 16; ++c16) {
                uint32_t raw[16];
                tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(q * 32) << 16) + c16 * 16, raw);
                tmem_ld_wait();
                if (col < p.m) {
                    if (p.splits == 1) {
                        __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(p.Y);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int tok = c16 * 16 + i;
                            const float v = any_k ? __uint_as_float(raw[i]) : 0.f;
                            if (tok < p.n) Y[(int64_t)tok * p.ldy + col] = __float2bfloat16_rn(v * p.alpha);
                        }
                    } else {
                        // [split][token][column]: a warp's lanes write consecutive columns
                        float* dst = p.partials + (int64_t)split * NP * p.m + col;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int tok = c16 * 16 + i;
                            if (tok < p.n) __stcg(dst + (int64_t)tok * p.m, any_k ? __uint_as_float(raw[i]) : 0.f);
                        }
                    }
                }
            }
        }
    } else {
        // cp.async gather of the retained rows: thread t owns 16-byte chunks
        // t, t + 256, t + 512, t + 768 of the 64 x 16 chunk stage
        const int ptid = threadIdx.x - 6 * 32;
        const __nv_bfloat16* B = static_cast<const __nv_bfloat16*>(p.B);
        for (int kb = kb_beg, it = 0; kb < kb_end; ++kb, ++it) {
            const int s = it % C::STAGES;
            const uint32_t ph = (it / C::STAGES) & 1u;
            int32_t rowj[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) rowj[i] = sidx[it * kSkBK + (ptid >> 4) + 16 * i];
            if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, kErrTimeoutProducer)) break;
            const uint32_t g_addr = smem_u32(smem + s * C::STAGE_BYTES);
            const int cc = ptid & 15;                 // 16-byte chunk within the 256-byte row slice
            const int gcol = m0 + 8 * cc;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = (ptid >> 4) + 16 * i;
                const bool valid = rowj[i] >= 0 && gcol < p.m;
                const __nv_bfloat16* src = B + (valid ? (int64_t)rowj[i] * p.ldb + gcol : 0);
                const uint32_t dst = g_addr + (cc >> 3) * kSkGroupBytes + r * 128 + (((cc & 7) ^ (r & 7)) << 4);
                cp_async_16(dst, src, valid ? 16u : 0u);
            }
            cp_async_arrive_noinc(&full[s]);
        }
        cp_async_wait_all();
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// Y[i][c] = alpha * (sum over splits, in order, of partials[s][c][i]), rounded to bf16.
template <int NP>
__global__ void __launch_bounds__(256) skinny_reduce_kernel(const float* __restrict__ partials, int splits,
                                                            int n, int m, float alpha,
                                                            __nv_bfloat16* __restrict__ Y, int64_t ldy) {
    pdl_wait();
    pdl_trigger();
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over n x m, column fastest
    if (e >= (int64_t)n * m) return;
    const int i = (int)(e / m), c = (int)(e - (int64_t)i * m);
    float sum = 0.f;
    for (int s = 0; s < splits; ++s) sum += __ldcg(partials + ((int64_t)s * NP + i) * m + c);
    Y[(int64_t)i * ldy + c] = __float2bfloat16_rn(sum * alpha);
}

template <int NP>
cudaError_t launch_np(const SkinnyParams& p, cudaStream_t s) {
    using C = SkCfg<NP>;
    cudaError_t e = cudaFuncSetAttribute(skinny_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::SMEM);
    if (e != cudaSuccess) return e;
    e = launch_pdl(skinny_kernel<NP>, dim3(p.m_tiles * p.splits), dim3(kSkThreads), C::SMEM, s, p);
    if (e != cudaSuccess || p.splits == 1) return e;
    const int64_t total = (int64_t)p.n * p.m;
    return launch_pdl(skinny_reduce_kernel<NP>, dim3((unsigned)((total + 255) / 256)), dim3(256), 0, s, p.partials,
                      p.splits, p.n, p.m, p.alpha, static_cast<__nv_bfloat16*>(p.Y), p.ldy);
}

}  // namespace

int skinny_pad(int64_t n) { return n <= 16 ? 16 : (n <= 32 ? 32 : 64); }

int skinny_splits(int64_t m, int64_t k, int num_sms, int np) {
    const int64_t m_tiles = (m + 127) / 128;
    const int64_t nkb = (k + kSkBK - 1) / kSkBK;
    int64_t lo = (nkb * kSkBK + kSkMaxSplitIdx - kSkBK - 1) / (kSkMaxSplitIdx - kSkBK);
    if (lo < 1) lo = 1;  // each split's indices fit the shared staging area
    int64_t hi = nkb < 64 ? nkb : 64;
    if (hi < lo) hi = lo;
    if (num_sms <= 0) return (int)lo;
    // Time in k-block units.  Two CTAs share an SM's bandwidth, so an SM's
    // time follows the number of CTAs it runs: ceil(CTAs / SMs) times one
    // CTA's share of K plus a fixed cost (prologue, pipeline fill, partials).
    const int64_t slots = num_sms;
    const int64_t fixed = 4 + np / 16;
    int64_t best = lo, best_cost = -1;
    for (int64_t sp = lo; sp <= hi; ++sp) {
        const int64_t waves = (m_tiles * sp + slots - 1) / slots;
        const int64_t cost = waves * ((nkb + sp - 1) / sp + fixed);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = sp;
        }
    }
    return (int)best;
}

cudaError_t launch_skinny(const SkinnyParams& p, cudaStream_t s) {
    switch (p.np) {
        case 16: return launch_np<16>(p, s);
        case 32: return launch_np<32>(p, s);
        case 64: return launch_np<64>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace rmm
