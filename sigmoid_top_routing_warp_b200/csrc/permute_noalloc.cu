// permute_noalloc.cu -- moe_permute_noalloc: the dispatch-order permutation
// for callers that cannot allocate device memory at all.
//
// Such callers include plugins that a host framework hands only their input
// and output buffers, and runtimes whose memory planner owns the whole HBM
// budget and forbids any allocation outside it.  They cannot provide the
// workspace that moe_permute takes, so this variant keeps its scratch in a
// fixed array of device memory that is part of the library image.
//
// The array holds, for the multi-block path, the first row of every
// (chunk, expert) pair: at most kNoAllocScratchInts int32 values (256 KiB).
// Every GPU that loads the library holds it until the process exits.  The
// count pass of each call writes every entry that the later passes read, so
// nothing has to start at zero and stale contents of an earlier call are
// never read.  All calls share the one array: calls that overlap on the GPU
// (for example on two streams at once) race on it and must not be issued.
//
// In host code `g_noalloc_scratch` is only a host-side stand-in for the
// device array, not a device address.  The device address is looked up once
// per device with cudaGetSymbolAddress, with that device current, the first
// time the entry point runs on that device; that first call should therefore
// come before any stream capture.  The address belongs to the device's
// current CUDA context: if that context is replaced (after cudaDeviceReset,
// for example) the module may load elsewhere, so every call compares the
// current context's id with the one recorded at set-up and repeats the
// look-up when they differ.  Nothing here calls cudaMalloc, cudaFree or any
// allocating library routine.
#include "moe.h"
#include "kernels.cuh"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

namespace moe {
moe_status_t api_check_config(const moe_config_t* c);
moe_status_t api_fail(moe_status_t st, const char* msg);
void api_clear_error();
}  // namespace moe

namespace {

constexpr int kNoAllocScratchInts = MOE_PERMUTE_NOALLOC_SCRATCH_INTS;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context id of the look-up

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the calling thread's current CUDA context (0 if there is none yet).
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_ctx = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_ctx = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        looked_up = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array on the current device: looked up once
// per device, and again only if the device's context has changed since.
moe_status_t scratch_on_current_device(int32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return moe::api_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return moe::api_fail(MOE_ERR_UNSUPPORTED, "device ordinal beyond the supported range");
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            char msg[256];
            snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the permute scratch: %s",
                     cudaGetErrorString(e));
            return moe::api_fail(MOE_ERR_CUDA, msg);
        }
        g_scratch_addr[dev] = static_cast<int32_t*>(p);
        // the look-up made the device's primary context current if none was
        g_scratch_ctx[dev] = current_context_id();
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const moe_config_t* cfg, const int32_t* topk_idx,
                                            int32_t* offsets, int32_t* rows, int32_t* pos,
                                            moe_stream_t stream) {
    moe::api_clear_error();
    moe_status_t st = moe::api_check_config(cfg);
    if (st != MOE_OK) return st;
    if (!topk_idx || !offsets || !rows || !pos)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "topk_idx, offsets, rows and pos must be non-NULL");
    const long long n = (long long)cfg->T * cfg->k;
    const long long need = (long long)moe::permute_chunks((int)n) * cfg->E;
    if (need > kNoAllocScratchInts) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "moe_permute_noalloc: T*k=%lld with E=%d needs %lld scratch entries, more than "
                 "the fixed %d (use moe_permute with a workspace)",
                 n, cfg->E, need, kNoAllocScratchInts);
        return moe::api_fail(MOE_ERR_UNSUPPORTED, msg);
    }
    // T = 0 still launches: the single-block path writes offsets[0..E] = 0
    // (as moe_permute does) and reads no scratch
    int32_t* scratch = nullptr;
    st = scratch_on_current_device(&scratch);
    if (st != MOE_OK) return st;
    moe::PermuteArgs a;
    a.idx = topk_idx;
    a.offsets = offsets;
    a.rows = rows;
    a.pos = pos;
    a.chunk_base = scratch;
    a.T = cfg->T;
    a.k = cfg->k;
    a.E = cfg->E;
    cudaError_t e = moe::launch_permute(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return moe::api_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
    return MOE_OK;
}
