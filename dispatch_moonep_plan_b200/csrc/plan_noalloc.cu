// plan_noalloc.cu -- moonep_plan_noalloc: the planner with its scratch held in
// a static device array inside the library instead of a caller workspace.
//
// Who needs it: a caller that cannot hand the planner a workspace buffer.
// Examples are a framework plugin whose host framework owns all device
// memory through its own allocator and gives plugins no scratch, and a
// serving loop that reserves every buffer at start-up and must not allocate
// once it is running.  Such callers still allocate the plan's outputs (they
// are part of the layer's state), but not the planner's per-block histogram
// tables.
//
// The array below is that scratch: the per-block histogram columns, their
// prefix offsets and the per-expert totals, laid out exactly as in a caller
// workspace, for up to MOONEP_NOALLOC_MAX_E experts (4 MiB + 2 KiB).  Every
// GPU that loads the library holds it until the process exits.
//
// Host code cannot use the array's name as a device address.  The address
// belongs to the driver context the library's module is loaded in, so it is
// looked up with cudaGetSymbolAddress, with the calling device current, on
// every call made outside a stream capture, and cached per device together
// with that context.  A call inside a capture may not look anything up; it
// takes the cached address, which must belong to the current context (after
// a device reset, or under another driver context, the array lives at a new
// address and the cache is stale until a call outside capture refreshes it).
#include <cuda.h>

#include <mutex>

#include "internal.cuh"

namespace {

constexpr size_t kScratchWords =
    2 * (size_t)MOONEP_NOALLOC_MAX_E * moonep::MAX_GRID + (size_t)MOONEP_NOALLOC_MAX_E;

static __device__ __align__(256) int32_t g_plan_scratch[kScratchWords];

constexpr int kMaxDevices = 64;
struct CachedAddress {
    CUcontext ctx;
    void* addr;
};
std::mutex g_mu;
CachedAddress g_scratch_addr[kMaxDevices] = {};

const char* const kFn = "moonep_plan_noalloc";

using PFN_CtxGetCurrent = CUresult (*)(CUcontext*);

// The driver context current on this thread (nullptr if none or unknown).
CUcontext current_context() {
    static PFN_CtxGetCurrent fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_CtxGetCurrent>(f);
    }();
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// Device address of the scratch array in the current device's context.
cudaError_t scratch_address(cudaStream_t stream, void** out, const char** why) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_plan_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev].ctx = current_context();
        g_scratch_addr[dev].addr = p;
        *out = p;
        return cudaSuccess;
    }
    const CachedAddress& c = g_scratch_addr[dev];
    if (!c.addr || c.ctx == nullptr || c.ctx != current_context()) {
        *why = "inside a stream capture, but no call outside capture has looked up the scratch "
               "array's address in this device's current context yet (first call, device reset "
               "or another driver context): call it once before capturing";
        return cudaErrorStreamCaptureUnsupported;
    }
    *out = c.addr;
    return cudaSuccess;
}

}  // namespace

extern "C" int moonep_plan_noalloc(const moonep_config* c, const int32_t* topk_idx,
                                   const moonep_plan_t* plan, moonep_stream_t stream) {
    // config checks: the same rules as every other call (moonep_sizes)
    moonep_sizes_t sz;
    if (moonep_sizes(c, &sz) != MOONEP_OK)
        return moonep::set_last_error(MOONEP_ERR_INVALID_ARG, kFn, moonep_last_error());
    if (c->E > MOONEP_NOALLOC_MAX_E)
        return moonep::set_last_error(MOONEP_ERR_INVALID_ARG, kFn,
                                      "E exceeds MOONEP_NOALLOC_MAX_E (512), the size of the "
                                      "library's static planner scratch; use moonep_plan with "
                                      "a workspace");
    if (!plan || !topk_idx || !plan->expert_count || !plan->rank_load || !plan->cu_seqlens ||
        !plan->dst_row || !plan->src_of_row || !plan->status || !plan->maxvio ||
        (c->B > 0 && !plan->slot_expert))
        return moonep::set_last_error(MOONEP_ERR_INVALID_ARG, kFn,
                                      "topk_idx or a plan output pointer is NULL");
    void* scratch = nullptr;
    const char* addr_why = nullptr;
    cudaError_t e = scratch_address(static_cast<cudaStream_t>(stream), &scratch, &addr_why);
    if (e != cudaSuccess)
        return moonep::set_last_error(MOONEP_ERR_CUDA, kFn,
                                      addr_why ? addr_why : cudaGetErrorString(e));
    moonep::PlanLaunch a;
    a.R = c->R; a.S = c->S; a.E = c->E; a.K = c->K; a.B = c->B; a.rule = c->rule;
    a.idx = topk_idx;
    a.plan = *plan;
    a.plan.workspace = scratch;
    a.plan.workspace_bytes = kScratchWords * sizeof(int32_t);
    a.wait_ns = moonep::current_wait_limit_ns();
    a.barrier_extra = moonep::current_barrier_extra();
    const char* why = nullptr;
    e = moonep::launch_plan(a, static_cast<cudaStream_t>(stream), &why);
    if (e != cudaSuccess)
        return moonep::set_last_error(MOONEP_ERR_CUDA, kFn, why ? why : cudaGetErrorString(e));
    return MOONEP_OK;
}
