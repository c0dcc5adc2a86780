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
// Host code cannot use the array's name as a device address: the address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on that device, and cached.
#include <mutex>

#include "internal.cuh"

namespace {

constexpr size_t kScratchWords =
    2 * (size_t)MOONEP_NOALLOC_MAX_E * moonep::MAX_GRID + (size_t)MOONEP_NOALLOC_MAX_E;

static __device__ __align__(256) int32_t g_plan_scratch[kScratchWords];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

const char* const kFn = "moonep_plan_noalloc";

// Device address of the scratch array on the current device.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_plan_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
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
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess)
        return moonep::set_last_error(MOONEP_ERR_CUDA, kFn, cudaGetErrorString(e));
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
