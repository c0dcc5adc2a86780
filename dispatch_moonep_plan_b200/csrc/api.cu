// api.cu -- the extern "C" entry points declared in include/moonep.h:
// argument checks, error strings, and the hand-off to the kernel launchers.
#include <cstdint>
#include <cstdio>
#include <string>

#include "internal.cuh"

namespace moonep {
int weights_create(const moonep_config& c, int elem_bytes, moonep_weights_t* out,
                   const char** why);
int weights_destroy(moonep_weights_t* w);
}  // namespace moonep

namespace {

thread_local std::string g_err;
unsigned long long g_wait_ns = 1000000000ull;
int g_barrier_extra = 0;

int fail(int code, const char* fn, const char* why) {
    g_err = std::string(fn) + ": " + why;
    return code;
}

int cuda_fail(const char* fn, cudaError_t e, const char* why = nullptr) {
    g_err = std::string(fn) + ": " + (why ? why : cudaGetErrorString(e)) + " (" +
            cudaGetErrorName(e) + ")";
    return MOONEP_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// nullptr if the configuration is acceptable, else the reason
const char* check_config(const moonep_config* c) {
    if (!c) return "config is NULL";
    if (c->R <= 0 || c->S <= 0 || c->E <= 0 || c->K <= 0 || c->H <= 0)
        return "R, S, E, K and H must be positive";
    if (c->B < 0 || c->Hp < 0) return "B and Hp must be non-negative";
    if (c->E % c->R != 0) return "E must be a multiple of R (contiguous home experts)";
    if (c->E > MOONEP_MAX_E) return "E exceeds MOONEP_MAX_E";
    if (c->R > MOONEP_MAX_R) return "R exceeds MOONEP_MAX_R";
    if (c->B > MOONEP_MAX_B) return "B exceeds MOONEP_MAX_B";
    if (c->K > MOONEP_MAX_K) return "K exceeds MOONEP_MAX_K";
    if ((long long)c->R * c->S * c->K >= (1ll << 31)) return "R*S*K must be below 2^31";
    if (c->H % 8 != 0) return "H must be a multiple of 8 (16-byte rows)";
    if (c->payload != MOONEP_PAYLOAD_BF16 && c->payload != MOONEP_PAYLOAD_FP8)
        return "unknown payload";
    if (c->payload == MOONEP_PAYLOAD_FP8 && c->H % 128 != 0)
        return "fp8 payload needs H to be a multiple of 128";
    if (c->rule != MOONEP_RULE_INDEX_ORDER && c->rule != MOONEP_RULE_KEEP_LIGHTEST &&
        c->rule != MOONEP_RULE_LARGEST_FIRST)
        return "unknown rule";
    return nullptr;
}

// The plan outputs every call reads or writes.  The planner's workspace is
// checked by moonep_plan alone: no other call touches it.
const char* check_plan(const moonep_config* c, const moonep_plan_t* p) {
    if (!p) return "plan is NULL";
    if (!p->expert_count || !p->rank_load || !p->cu_seqlens || !p->dst_row || !p->src_of_row ||
        !p->status || !p->maxvio)
        return "a plan pointer is NULL";
    if (c->B > 0 && !p->slot_expert) return "slot_expert is NULL";
    return nullptr;
}

const char* check_workspace(const moonep_config* c, const moonep_plan_t* p) {
    if (!p->workspace) return "workspace is NULL";
    if (!aligned16(p->workspace)) return "workspace must be 16-byte aligned";
    if (p->workspace_bytes < moonep::plan_workspace_bytes(c->E)) return "workspace too small";
    return nullptr;
}

}  // namespace

namespace moonep {
unsigned long long current_wait_limit_ns() { return g_wait_ns; }
int current_barrier_extra() { return g_barrier_extra; }
int set_last_error(int code, const char* fn, const char* why) {
    const std::string reason(why);  // why may point into the current message
    return fail(code, fn, reason.c_str());
}
}  // namespace moonep

extern "C" {

int moonep_version(void) { return 100; }

const char* moonep_last_error(void) { return g_err.c_str(); }

int moonep_set_wait_limit_ns(uint64_t ns) {
    if (ns == 0) return fail(MOONEP_ERR_INVALID_ARG, "moonep_set_wait_limit_ns", "limit must be > 0");
    g_wait_ns = ns;
    return MOONEP_OK;
}

int moonep_debug_set_barrier_extra(int32_t extra) {
    if (extra < 0) return fail(MOONEP_ERR_INVALID_ARG, "moonep_debug_set_barrier_extra", "extra < 0");
    g_barrier_extra = extra;
    return MOONEP_OK;
}

int moonep_sizes(const moonep_config* c, moonep_sizes_t* o) {
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, "moonep_sizes", why);
    if (!o) return fail(MOONEP_ERR_INVALID_ARG, "moonep_sizes", "out is NULL");
    const int64_t T = (int64_t)c->R * c->S, P = T * c->K, C = (int64_t)c->S * c->K;
    const bool fp8 = c->payload == MOONEP_PAYLOAD_FP8;
    const size_t elem = fp8 ? 1 : 2;
    o->tokens = T;
    o->picks = P;
    o->rows_per_rank = C;
    o->topk_idx_bytes = (size_t)P * 4;
    o->topk_w_bytes = (size_t)P * 4;
    o->x_bytes = (size_t)T * c->H * 2;
    o->recv_bytes = (size_t)P * c->H * elem;
    o->recv_scale_bytes = fp8 ? (size_t)P * (c->H / 128) * 4 : 0;
    o->dispatch_buffer_bytes_per_rank =
        (size_t)C * c->H * elem + (fp8 ? (size_t)C * (c->H / 128) * 4 : 0);
    o->expert_out_bytes = (size_t)P * c->H * 2;
    o->y_bytes = (size_t)T * c->H * 2;
    o->expert_count_bytes = (size_t)c->E * 4;
    o->rank_load_bytes = (size_t)c->R * 4;
    o->slot_expert_bytes = (size_t)c->R * c->B * 4;
    o->cu_seqlens_bytes = (size_t)c->R * (c->E + c->B) * 4;
    o->dst_row_bytes = (size_t)P * 4;
    o->src_of_row_bytes = (size_t)P * 4;
    o->status_bytes = MOONEP_STATUS_WORDS * 4;
    o->maxvio_bytes = 8;
    o->workspace_bytes = moonep::plan_workspace_bytes(c->E);
    o->weight_row_bytes = (size_t)c->H * c->Hp * 2;
    o->prefetch_pool_bytes_per_rank = o->weight_row_bytes * c->B;
    o->weights_view_bytes = o->weight_row_bytes * (c->E + c->B);
    return MOONEP_OK;
}

int moonep_plan(const moonep_config* c, const int32_t* topk_idx, const moonep_plan_t* plan,
                moonep_stream_t stream) {
    const char* fn = "moonep_plan";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_workspace(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (!topk_idx) return fail(MOONEP_ERR_INVALID_ARG, fn, "topk_idx is NULL");
    moonep::PlanLaunch a;
    a.R = c->R; a.S = c->S; a.E = c->E; a.K = c->K; a.B = c->B; a.rule = c->rule;
    a.idx = topk_idx;
    a.plan = *plan;
    a.wait_ns = g_wait_ns;
    a.barrier_extra = g_barrier_extra;
    const char* why = nullptr;
    cudaError_t e = moonep::launch_plan(a, static_cast<cudaStream_t>(stream), &why);
    if (e != cudaSuccess) return cuda_fail(fn, e, why);
    return MOONEP_OK;
}

int moonep_dispatch(const moonep_config* c, const moonep_plan_t* plan, const void* x, void* recv,
                    float* recv_scale, moonep_stream_t stream) {
    const char* fn = "moonep_dispatch";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (!x || !recv) return fail(MOONEP_ERR_INVALID_ARG, fn, "x or recv is NULL");
    if (!aligned16(x) || !aligned16(recv))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "x and recv must be 16-byte aligned");
    if (c->payload == MOONEP_PAYLOAD_FP8) {
        if (!recv_scale) return fail(MOONEP_ERR_INVALID_ARG, fn, "fp8 payload needs recv_scale");
        if ((reinterpret_cast<uintptr_t>(recv_scale) & 3u) != 0)
            return fail(MOONEP_ERR_INVALID_ARG, fn, "recv_scale must be 4-byte aligned");
    } else if (recv_scale) {
        return fail(MOONEP_ERR_INVALID_ARG, fn, "bf16 payload takes no recv_scale");
    }
    cudaError_t e = moonep::launch_dispatch(*c, *plan, x, recv, recv_scale,
                                            static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_combine(const moonep_config* c, const moonep_plan_t* plan, const void* expert_out,
                   const float* topk_w, void* y, moonep_stream_t stream) {
    const char* fn = "moonep_combine";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (!expert_out || !topk_w || !y)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "expert_out, topk_w or y is NULL");
    if (!aligned16(expert_out) || !aligned16(y))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "expert_out and y must be 16-byte aligned");
    cudaError_t e = moonep::launch_combine(*c, *plan, expert_out, topk_w, y,
                                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_combine_backward(const moonep_config* c, const moonep_plan_t* plan, const void* dy,
                            const void* expert_out, const float* topk_w, void* d_expert_out,
                            float* d_topk_w, moonep_stream_t stream) {
    const char* fn = "moonep_combine_backward";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (!dy || !expert_out || !topk_w || !d_expert_out || !d_topk_w)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "a NULL argument");
    if (!aligned16(dy) || !aligned16(expert_out) || !aligned16(d_expert_out))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "dy, expert_out and d_expert_out must be 16-byte aligned");
    cudaError_t e = moonep::launch_combine_backward(*c, *plan, dy, expert_out, topk_w, d_expert_out,
                                                    d_topk_w, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_dispatch_backward(const moonep_config* c, const moonep_plan_t* plan, const void* d_recv,
                             void* dx, moonep_stream_t stream) {
    const char* fn = "moonep_dispatch_backward";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (!d_recv || !dx) return fail(MOONEP_ERR_INVALID_ARG, fn, "d_recv or dx is NULL");
    if (!aligned16(d_recv) || !aligned16(dx))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "d_recv and dx must be 16-byte aligned");
    cudaError_t e = moonep::launch_dispatch_backward(*c, *plan, d_recv, dx,
                                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_expert_standin(const moonep_config* c, const moonep_plan_t* plan, const void* recv,
                          const float* recv_scale, int32_t mode, void* out,
                          moonep_stream_t stream) {
    const char* fn = "moonep_expert_standin";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (!recv || !out) return fail(MOONEP_ERR_INVALID_ARG, fn, "recv or out is NULL");
    if (!aligned16(recv) || !aligned16(out))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "recv and out must be 16-byte aligned");
    if (mode != MOONEP_EXPERT_IDENTITY && mode != MOONEP_EXPERT_SCALE)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "unknown mode");
    if (c->payload == MOONEP_PAYLOAD_FP8 && !recv_scale)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "fp8 payload needs recv_scale");
    if (c->B > 0 && !plan->slot_expert)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "slot_expert is NULL");
    cudaError_t e = moonep::launch_expert_standin(*c, *plan, recv, recv_scale, mode, out,
                                                  static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_expert_gemm(const moonep_config* c, const moonep_plan_t* plan, const void* recv,
                       const float* recv_scale, const void* weights, void* out,
                       moonep_stream_t stream) {
    const char* fn = "moonep_expert_gemm";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (c->payload == MOONEP_PAYLOAD_FP8 && !recv_scale)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "fp8 payload needs recv_scale");
    if (c->payload == MOONEP_PAYLOAD_FP8 && !aligned16(recv_scale))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "recv_scale must be 16-byte aligned");
    if (c->H % 64 != 0) return fail(MOONEP_ERR_INVALID_ARG, fn, "H must be a multiple of 64");
    if (c->Hp <= 0 || c->Hp % 128 != 0)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "Hp must be a positive multiple of 128");
    if ((long long)c->R * (c->E + c->B) * c->H >= (1LL << 31))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "R*(E+B)*H must be below 2^31");
    if (!recv || !weights || !out)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "recv, weights or out is NULL");
    if (!aligned16(recv) || !aligned16(weights) || !aligned16(out))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "recv, weights and out must be 16-byte aligned");
    if (!moonep::expert_gemm_fits(*c))
        return fail(MOONEP_ERR_INVALID_ARG, fn, "too many (rank, group) pairs for shared memory");
    const char* why = nullptr;
    cudaError_t e = moonep::launch_expert_gemm(
        *c, *plan, recv, c->payload == MOONEP_PAYLOAD_FP8 ? recv_scale : nullptr, weights, out,
        static_cast<cudaStream_t>(stream), &why);
    if (e != cudaSuccess) return cuda_fail(fn, e, why);
    return MOONEP_OK;
}

int moonep_prefetch(const moonep_config* c, const moonep_plan_t* plan, void* const* rank_weights,
                    int32_t elem_bytes, moonep_stream_t stream) {
    const char* fn = "moonep_prefetch";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "elem_bytes must be 1, 2 or 4");
    if (c->Hp <= 0) return fail(MOONEP_ERR_INVALID_ARG, fn, "Hp must be positive");
    if (((long long)c->H * c->Hp * elem_bytes) % 16 != 0)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "H*Hp*elem_bytes must be a multiple of 16");
    if (!rank_weights) return fail(MOONEP_ERR_INVALID_ARG, fn, "rank_weights is NULL");
    for (int r = 0; r < c->R; ++r)
        if (!rank_weights[r] || !aligned16(rank_weights[r]))
            return fail(MOONEP_ERR_INVALID_ARG, fn, "a rank view is NULL or not 16-byte aligned");
    if (c->B == 0) return MOONEP_OK;
    cudaError_t e = moonep::launch_prefetch(*c, *plan, rank_weights, elem_bytes,
                                            static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_grad_reduce(const moonep_config* c, const moonep_plan_t* plan, float* const* rank_grads,
                       moonep_stream_t stream) {
    const char* fn = "moonep_grad_reduce";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (const char* why = check_plan(c, plan)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (c->Hp <= 0) return fail(MOONEP_ERR_INVALID_ARG, fn, "Hp must be positive");
    if (((long long)c->H * c->Hp * 4) % 16 != 0)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "H*Hp*4 must be a multiple of 16");
    if (!rank_grads) return fail(MOONEP_ERR_INVALID_ARG, fn, "rank_grads is NULL");
    for (int r = 0; r < c->R; ++r)
        if (!rank_grads[r] || !aligned16(rank_grads[r]))
            return fail(MOONEP_ERR_INVALID_ARG, fn, "a rank view is NULL or not 16-byte aligned");
    if (c->B == 0) return MOONEP_OK;
    cudaError_t e = moonep::launch_grad_reduce(*c, *plan, rank_grads,
                                               static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_plan_status(const moonep_plan_t* plan, moonep_stream_t stream, int32_t* out) {
    const char* fn = "moonep_plan_status";
    if (!plan || !plan->status || !out) return fail(MOONEP_ERR_INVALID_ARG, fn, "NULL argument");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(out, plan->status, 4 * sizeof(int32_t),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(fn, e);
    return MOONEP_OK;
}

int moonep_weights_create(const moonep_config* c, int32_t elem_bytes, moonep_weights_t* out) {
    const char* fn = "moonep_weights_create";
    if (const char* why = check_config(c)) return fail(MOONEP_ERR_INVALID_ARG, fn, why);
    if (!out) return fail(MOONEP_ERR_INVALID_ARG, fn, "out is NULL");
    if (c->Hp <= 0) return fail(MOONEP_ERR_INVALID_ARG, fn, "Hp must be positive");
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4)
        return fail(MOONEP_ERR_INVALID_ARG, fn, "elem_bytes must be 1, 2 or 4");
    const char* why = "failed";
    int rc = moonep::weights_create(*c, elem_bytes, out, &why);
    if (rc != MOONEP_OK) return fail(rc, fn, why);
    return MOONEP_OK;
}

int moonep_weights_destroy(moonep_weights_t* w) {
    int rc = moonep::weights_destroy(w);
    if (rc != MOONEP_OK) return fail(rc, "moonep_weights_destroy", "not a live weights object");
    return MOONEP_OK;
}

}  // extern "C"
