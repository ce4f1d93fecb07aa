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

#include <cuda.h>
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
struct ScratchSlot {
    unsigned long long ctx_id;  // the CUDA context the address was looked up in
    void* addr;
};
ScratchSlot g_scratch[kMaxDevices] = {};

// Unique id of the calling thread's current CUDA context (driver API, looked
// up once through the runtime's entry-point query), or 0 if unavailable.
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
        cudaGetLastError();
        looked_up = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_select_scratch on the current device and context.  It
// is looked up with cudaGetSymbolAddress on the first call in a context and
// looked up again when the context changes (after cudaDeviceReset, for
// example, the device's primary context and the address are new).
rmm_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return RMM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RMM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const unsigned long long ctx = current_context_id();
    ScratchSlot& slot = g_scratch[dev];
    if (!slot.addr || ctx == 0 || slot.ctx_id != ctx) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return RMM_ERR_CUDA;
        }
        slot.addr = p;
        slot.ctx_id = ctx;
    }
    *out = slot.addr;
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

    cudaStream_t s = static_cast<cudaStream_t>(stream);
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
    // Selections done inside one kernel per head need no scratch at all: take
    // the same kernel as rmm_select for the plan.
    if (plan->select_small || plan->select16 || plan->fused_select) {
        cudaError_t e = plan->select_small ? rmm::launch_select_small(a, s)
                        : plan->select16   ? rmm::launch_select16(a, s)
                                           : rmm::launch_normselect(a, s);
        return e == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
    }

    // Scratch layout: completion counters | split partials | final scores.
    const int vec = 16 / plan->es;
    const int64_t colblocks = (p.d + 32 * vec - 1) / (32 * vec);
    const size_t counter_bytes = align256(static_cast<size_t>(p.heads) * colblocks * sizeof(unsigned));
    const size_t partial_bytes = align256(static_cast<size_t>(p.heads) * plan->nsplit * p.d * sizeof(float));
    const size_t score_bytes = align256(static_cast<size_t>(p.heads) * p.d * sizeof(float));
    if (counter_bytes + partial_bytes + score_bytes > kNoAllocScratchBytes) return RMM_ERR_UNSUPPORTED;

    // The scratch address belongs to the current device: the stream must be
    // one of that device's streams.
    int cur = -1, sdev = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cudaStreamGetDevice(s, &sdev) != cudaSuccess) {
        cudaGetLastError();
        return RMM_ERR_CUDA;
    }
    if (sdev != cur) return RMM_ERR_INVALID_ARG;

    void* base = nullptr;
    const rmm_status st = scratch_address(&base);
    if (st != RMM_OK) return st;
    unsigned char* scratch = static_cast<unsigned char*>(base);

    // The counters must start at zero; the partials and scores are fully
    // overwritten by every call.
    if (cudaMemsetAsync(scratch, 0, counter_bytes, s) != cudaSuccess) return RMM_ERR_CUDA;

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
