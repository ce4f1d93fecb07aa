// rmm_static.cu -- index selection without any device allocation.
//
// Some callers cannot allocate device memory at the point where they need an
// index set: code that runs while a memory pool is frozen or being captured,
// plugins living inside another runtime's allocator, or a fixed-footprint
// serving process whose memory budget was reserved up front.  For them,
// rmm_select_no_alloc runs the same score and TopK kernels as rmm_select but
// keeps their scratch (per-split partial sums, completion counters and the
// final scores) in one file-scope device array of kNoAllocScratchBytes that
// every GPU loading this library holds until the process exits.  The caller
// passes only the input and the outputs.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

// The shared scratch.  Host code must not use this name as a device address
// (on the host it denotes a stand-in object); the address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device (looked up on the
// first call for that device).
rmm_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return RMM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RMM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return RMM_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return RMM_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" rmm_status rmm_select_no_alloc(const rmm_plan* plan, const void* A, int32_t* I, float* s2,
                                          void* stream) {
    if (!plan || !A || !I) return RMM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(A) & 15u) || (reinterpret_cast<uintptr_t>(I) & 3u) ||
        (s2 && (reinterpret_cast<uintptr_t>(s2) & 3u)))
        return RMM_ERR_INVALID_ARG;
    const rmm_problem& p = plan->p;
    if (p.d > rmm::kMaxSelectD) return RMM_ERR_UNSUPPORTED;

    // Scratch layout: completion counters | split partials | final scores.
    const int vec = 16 / plan->es;
    const int64_t colblocks = (p.d + 32 * vec - 1) / (32 * vec);
    const size_t counter_bytes = align256(static_cast<size_t>(p.heads) * colblocks * sizeof(unsigned));
    const size_t partial_bytes = align256(static_cast<size_t>(p.heads) * plan->nsplit * p.d * sizeof(float));
    const size_t score_bytes = align256(static_cast<size_t>(p.heads) * p.d * sizeof(float));
    if (counter_bytes + partial_bytes + score_bytes > kNoAllocScratchBytes) return RMM_ERR_UNSUPPORTED;

    void* base = nullptr;
    const rmm_status st = scratch_address(&base);
    if (st != RMM_OK) return st;
    unsigned char* scratch = static_cast<unsigned char*>(base);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // The counters must start at zero; the partials and scores are fully
    // overwritten by every call.
    if (cudaMemsetAsync(scratch, 0, counter_bytes, s) != cudaSuccess) return RMM_ERR_CUDA;

    rmm::SelectArgs a{};
    a.A = A;
    a.dtype = p.dtype;
    a.n = p.n;
    a.d = p.d;
    a.lda = p.lda;
    a.stride_a = p.stride_a;
    a.heads = static_cast<int>(p.heads);
    a.k = plan->k;
    a.I = I;
    a.s2 = s2;
    a.counters = reinterpret_cast<unsigned*>(scratch);
    a.partials = reinterpret_cast<float*>(scratch + counter_bytes);
    a.scores = s2 ? s2 : reinterpret_cast<float*>(scratch + counter_bytes + partial_bytes);
    a.nsplit = plan->nsplit;
    a.rows_per_split = plan->rows_per_split;
    a.causal_rows = p.mode == RMM_PV && (p.flags & RMM_FLAG_CAUSAL) ? 1 : 0;
    cudaError_t e = rmm::launch_colnorm(a, s);
    if (e == cudaSuccess) e = rmm::launch_topk(a, s);
    return e == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
}
