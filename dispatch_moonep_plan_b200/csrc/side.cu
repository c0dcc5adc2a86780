// side.cu -- the two side steps around the expert computation ("Moonshot AI
// Open-Sources MoonEP ..." on ainovat.com, the paragraph on duplicated experts:
// they are prefetched before expert computation, and in the backward their
// gradients are reduced back to their home ranks; "MoonEP" on
// moses-y.github.io, "How It Is Wired", prefetch and gradient reduction).
//
// prefetch: for every used slot (r, j) with expert e = slot_expert[r][j],
//   row E+j of rank r's [E+B, H, H'] view <- row e of the home view (a bit
//   copy).  Work items are (slot, 64 KiB piece); blocks stride over them.
// grad-reduce: for every expert e with replicas, row e of its home view <-
//   ((row e + g_1) + g_2) + ... over its replicas in increasing (r, j), each
//   addition one binary32 operation.  The first replica of an expert owns the
//   expert's work items; every block derives the replica chains from the
//   slot map in shared memory.
#include "internal.cuh"

namespace moonep {
namespace {

constexpr int THREADS = 256;
constexpr long long PIECE = 64 * 1024;  // bytes per work item

struct Views {
    char* v[MOONEP_MAX_R];
};

__global__ void __launch_bounds__(THREADS) prefetch_kernel(Views views,
                                                          const int32_t* __restrict__ slot_expert,
                                                          int32_t* status,
                                                          int R, int E, int B, int Er,
                                                          long long row_bytes) {
    if (!block_status_ok(status)) return;
    const long long pieces = (row_bytes + PIECE - 1) / PIECE;
    const long long items = (long long)R * B * pieces;
    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const int slot = (int)(it / pieces);
        const long long piece = it % pieces;
        const int e = __ldg(slot_expert + slot);
        if (e < 0) continue;  // unused slot
        if (e >= E) {         // range guard
            if (threadIdx.x == 0) report_internal(status);
            continue;
        }
        const int r = slot / B, j = slot % B;
        const char* src = views.v[e / Er] + (long long)e * row_bytes + piece * PIECE;
        char* dst = views.v[r] + (long long)(E + j) * row_bytes + piece * PIECE;
        const long long n16 = min(PIECE, row_bytes - piece * PIECE) / 16;
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        uint4* d4 = reinterpret_cast<uint4*>(dst);
        constexpr int U = 4;
        for (long long i = threadIdx.x; i < n16; i += THREADS * U) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long k = i + (long long)u * THREADS;
                if (k < n16) v[u] = ld_stream_v4(s4 + k);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long k = i + (long long)u * THREADS;
                if (k < n16) d4[k] = v[u];
            }
        }
    }
}

__global__ void __launch_bounds__(THREADS) grad_reduce_kernel(Views views,
                                                             const int32_t* __restrict__ slot_expert,
                                                             int32_t* status,
                                                             int R, int E, int B, int Er,
                                                             long long row_bytes) {
    if (!block_status_ok(status)) return;
    extern __shared__ int sm[];
    const int RB = R * B;
    int* se = sm;         // [RB] slot map
    int* nxt = sm + RB;   // [RB] next replica of the same expert, -1 at the end
    int* head = nxt + RB; // [RB] 1 if this slot is its expert's first replica
    for (int q = threadIdx.x; q < RB; q += THREADS) {
        const int e = __ldg(slot_expert + q);
        if (e >= E && blockIdx.x == 0) report_internal(status);  // range guard
        se[q] = (e >= 0 && e < E) ? e : -1;
    }
    __syncthreads();
    for (int q = threadIdx.x; q < RB; q += THREADS) {
        const int e = se[q];
        int n = -1, first = 1;
        if (e >= 0) {
            for (int q2 = q + 1; q2 < RB; ++q2)
                if (se[q2] == e) { n = q2; break; }
            for (int q2 = 0; q2 < q; ++q2)
                if (se[q2] == e) { first = 0; break; }
        }
        nxt[q] = n;
        head[q] = (e >= 0) && first;
    }
    __syncthreads();

    const long long pieces = (row_bytes + PIECE - 1) / PIECE;
    const long long items = (long long)RB * pieces;
    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const int slot = (int)(it / pieces);
        if (!head[slot]) continue;
        const long long piece = it % pieces;
        const int e = se[slot];
        float4* home = reinterpret_cast<float4*>(views.v[e / Er] + (long long)e * row_bytes +
                                                 piece * PIECE);
        const long long n16 = min(PIECE, row_bytes - piece * PIECE) / 16;
        constexpr int U = 4;
        for (long long i = threadIdx.x; i < n16; i += THREADS * U) {
            float4 acc[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long k = i + (long long)u * THREADS;
                if (k < n16) acc[u] = home[k];
            }
            for (int q = slot; q >= 0; q = nxt[q]) {
                const int r = q / B, j = q % B;
                const float4* g = reinterpret_cast<const float4*>(
                    views.v[r] + (long long)(E + j) * row_bytes + piece * PIECE);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const long long k = i + (long long)u * THREADS;
                    if (k < n16) {
                        const uint4 raw = ld_stream_v4(g + k);
                        acc[u].x = __fadd_rn(acc[u].x, __uint_as_float(raw.x));
                        acc[u].y = __fadd_rn(acc[u].y, __uint_as_float(raw.y));
                        acc[u].z = __fadd_rn(acc[u].z, __uint_as_float(raw.z));
                        acc[u].w = __fadd_rn(acc[u].w, __uint_as_float(raw.w));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long k = i + (long long)u * THREADS;
                if (k < n16) home[k] = acc[u];
            }
        }
    }
}

int side_grid() {
    const int sms = device_sm_count();
    return sms * (2048 / THREADS);
}

}  // namespace

cudaError_t launch_prefetch(const moonep_config& c, const moonep_plan_t& p, void* const* views,
                            int elem_bytes, cudaStream_t s) {
    Views v;
    for (int r = 0; r < MOONEP_MAX_R; ++r) v.v[r] = r < c.R ? static_cast<char*>(views[r]) : nullptr;
    const long long row_bytes = (long long)c.H * c.Hp * elem_bytes;
    prefetch_kernel<<<side_grid(), THREADS, 0, s>>>(v, p.slot_expert, p.status, c.R, c.E, c.B,
                                                    c.E / c.R, row_bytes);
    return cudaGetLastError();
}

cudaError_t launch_grad_reduce(const moonep_config& c, const moonep_plan_t& p,
                               float* const* views, cudaStream_t s) {
    Views v;
    for (int r = 0; r < MOONEP_MAX_R; ++r)
        v.v[r] = r < c.R ? reinterpret_cast<char*>(views[r]) : nullptr;
    const long long row_bytes = (long long)c.H * c.Hp * 4;
    const size_t smem = (size_t)3 * c.R * c.B * sizeof(int);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(grad_reduce_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    grad_reduce_kernel<<<side_grid(), THREADS, smem, s>>>(v, p.slot_expert, p.status, c.R, c.E,
                                                          c.B, c.E / c.R, row_bytes);
    return cudaGetLastError();
}

}  // namespace moonep
