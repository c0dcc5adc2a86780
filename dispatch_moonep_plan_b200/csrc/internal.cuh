// internal.cuh -- shared device helpers and launch declarations of libmoonep.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moonep.h"

namespace moonep {

// status block words
constexpr int ST_STATUS = 0;
constexpr int ST_FAIL_RANK = 1;
constexpr int ST_FAIL_SLOTS = 2;
constexpr int ST_MAX_COUNT = 3;
constexpr int ST_BARRIER1 = 4;
constexpr int ST_BARRIER2 = 5;
constexpr int ST_BAD_FLAG = 6;

constexpr int MAX_GRID = 1024;  // planner blocks; sizes the workspace

// ---- PTX wrappers ---------------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add_u32(unsigned* p, unsigned v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 16-byte streaming load that skips L1 (read-once data)
__device__ __forceinline__ uint4 ld_stream_v4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte store with the evict-first (streaming) hint
__device__ __forceinline__ void st_stream_v4(void* p, uint4 v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_stream_v2(void* p, uint2 v)
{
    asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// Read a status word written by an earlier kernel in stream order (L2 copy).
__device__ __forceinline__ int load_status(const int32_t* status)
{
    return __ldcg(status + ST_STATUS);
}

// Whether a kernel may run: the plan's status read once per block.  Kernels
// of the path can set a failure status while other blocks are starting (a
// range check reporting INTERNAL, an expert-GEMM wait running out), so
// threads reading the word on their own could disagree; the block would then
// split, with some threads gone while the rest wait on shuffles or use
// shared data those threads were to fill.  Thread 0 reads, the block agrees.
__device__ __forceinline__ bool block_status_ok(const int32_t* status)
{
    __shared__ int st;
    if (threadIdx.x == 0) st = load_status(status);
    __syncthreads();
    return st == MOONEP_STATUS_OK;
}

// A kernel's own range check found an index outside its buffers (a planner
// bug, or a plan the caller overwrote): record MOONEP_STATUS_INTERNAL in the
// status block, unless an earlier failure is already there.  The caller skips
// or clamps the access, so nothing is read or written out of range.
__device__ __forceinline__ void report_internal(int32_t* status)
{
    atomicMax(status + ST_STATUS, MOONEP_STATUS_INTERNAL);
}

// ---- launchers (one per kernel file) ---------------------------------------
struct PlanLaunch {
    int R, S, E, K, B, rule;
    const int32_t* idx;
    moonep_plan_t plan;
    unsigned long long wait_ns;
    int barrier_extra;
};
cudaError_t launch_plan(const PlanLaunch& a, cudaStream_t s, const char** why);
size_t plan_workspace_bytes(int E);

cudaError_t launch_dispatch(const moonep_config& c, const moonep_plan_t& p, const void* x,
                            void* recv, float* recv_scale, cudaStream_t s);
cudaError_t launch_combine(const moonep_config& c, const moonep_plan_t& p, const void* eo,
                           const float* w, void* y, cudaStream_t s);
cudaError_t launch_dispatch_backward(const moonep_config& c, const moonep_plan_t& p,
                                     const void* d_recv, void* dx, cudaStream_t s);
cudaError_t launch_combine_backward(const moonep_config& c, const moonep_plan_t& p, const void* dy,
                                    const void* eo, const float* w, void* d_eo, float* d_w,
                                    cudaStream_t s);
cudaError_t launch_expert_standin(const moonep_config& c, const moonep_plan_t& p,
                                  const void* recv, const float* recv_scale, int mode, void* out,
                                  cudaStream_t s);
cudaError_t launch_prefetch(const moonep_config& c, const moonep_plan_t& p,
                            void* const* views, int elem_bytes, cudaStream_t s);
cudaError_t launch_grad_reduce(const moonep_config& c, const moonep_plan_t& p,
                               float* const* views, cudaStream_t s);

cudaError_t launch_expert_gemm(const moonep_config& c, const moonep_plan_t& p, const void* x,
                               const float* x_scale, const void* w, void* y, cudaStream_t s,
                               const char** why);
bool expert_gemm_fits(const moonep_config& c);

int device_sm_count();
unsigned long long current_wait_limit_ns();
int current_barrier_extra();
int set_last_error(int code, const char* fn, const char* why);  // returns code

}  // namespace moonep
