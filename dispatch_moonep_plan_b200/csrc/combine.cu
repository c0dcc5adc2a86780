// combine.cu -- gather each token's K expert-output rows back and reduce them
// with the router weights ("MoonEP" on moses-y.github.io, "What This Does"
// and "Real-World Use").
//
// y[t] = bf16(acc), acc = 0; for k = 0..K-1: acc = fma(w[t,k], x_k, acc),
// x_k = float(expert_out[dst_row[t,k]]), all in binary32, one rounding to
// bf16 (nearest even) at the end.  The k order is fixed, so the result does
// not depend on the launch shape.
//
// One warp per token (grid-stride).  Lane k < K holds dst_row[t,k] and
// w[t,k]; each lane owns U 16-byte chunks of the row, accumulates 8 floats per
// chunk, and the next pick's chunks are loaded while the current ones are
// accumulated.
#include <cuda_bf16.h>

#include "internal.cuh"

namespace moonep {
namespace {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // .x = a (low half)
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void accum(float* acc, float wk, const uint4& v) {
    acc[0] = __fmaf_rn(wk, bf16_lo(v.x), acc[0]);
    acc[1] = __fmaf_rn(wk, bf16_hi(v.x), acc[1]);
    acc[2] = __fmaf_rn(wk, bf16_lo(v.y), acc[2]);
    acc[3] = __fmaf_rn(wk, bf16_hi(v.y), acc[3]);
    acc[4] = __fmaf_rn(wk, bf16_lo(v.z), acc[4]);
    acc[5] = __fmaf_rn(wk, bf16_hi(v.z), acc[5]);
    acc[6] = __fmaf_rn(wk, bf16_lo(v.w), acc[6]);
    acc[7] = __fmaf_rn(wk, bf16_hi(v.w), acc[7]);
}

template <int U>
__global__ void __launch_bounds__(THREADS) combine_kernel(const uint4* __restrict__ eo,
                                                         const float* __restrict__ w,
                                                         const int32_t* __restrict__ dst_row,
                                                         uint4* __restrict__ y,
                                                         const int32_t* __restrict__ status, int T,
                                                         int K, int H8) {
    if (load_status(status) != MOONEP_STATUS_OK) return;
    const int lane = threadIdx.x & 31;
    const long long nw = (long long)gridDim.x * WARPS;
    for (long long t = (long long)blockIdx.x * WARPS + (threadIdx.x >> 5); t < T; t += nw) {
        int myrow = lane < K ? __ldg(dst_row + t * K + lane) : 0;
        if ((unsigned)myrow >= (unsigned)(T * K)) myrow = 0;  // range guard
        const float myw = lane < K ? __ldg(w + t * K + lane) : 0.0f;
        for (int c0 = 0; c0 < H8; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            uint4 cur[U], nxt[U];
            {
                const uint4* src = eo + (long long)__shfl_sync(0xffffffffu, myrow, 0) * H8;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    cur[u] = c < H8 ? ld_stream_v4(src + c) : make_uint4(0, 0, 0, 0);
                }
            }
            for (int k = 0; k < K; ++k) {
                const float wk = __shfl_sync(0xffffffffu, myw, k);
                const int krow = __shfl_sync(0xffffffffu, myrow, k + 1 < K ? k + 1 : k);
                if (k + 1 < K) {
                    const uint4* src = eo + (long long)krow * H8;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        nxt[u] = c < H8 ? ld_stream_v4(src + c) : make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) accum(acc[u], wk, cur[u]);
#pragma unroll
                for (int u = 0; u < U; ++u) cur[u] = nxt[u];
            }
            uint4* dst = y + t * H8;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < H8) {
                    uint4 o;
                    o.x = pack_bf16x2(acc[u][0], acc[u][1]);
                    o.y = pack_bf16x2(acc[u][2], acc[u][3]);
                    o.z = pack_bf16x2(acc[u][4], acc[u][5]);
                    o.w = pack_bf16x2(acc[u][6], acc[u][7]);
                    dst[c] = o;
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_combine(const moonep_config& c, const moonep_plan_t& p, const void* eo,
                           const float* w, void* y, cudaStream_t s) {
    const int T = c.R * c.S;
    const int H8 = c.H / 8;
    // Two 16-byte chunks per lane (double-buffered: 4 loads in flight) keep
    // the kernel near 56 registers, so 4 blocks of 256 stay resident per SM;
    // one resident wave of blocks strides over the tokens.  Measured against
    // four chunks per lane at 2 blocks per SM: 0.97-0.99 of the copy peak
    // instead of 0.89-0.93.
    const int sms = device_sm_count();
    long long grid = ((long long)T + WARPS - 1) / WARPS;
    const long long cap = (long long)sms * 4;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    if (H8 >= 64)
        combine_kernel<2><<<(int)grid, THREADS, 0, s>>>((const uint4*)eo, w, p.dst_row,
                                                       (uint4*)y, p.status, T, c.K, H8);
    else
        combine_kernel<1><<<(int)grid, THREADS, 0, s>>>((const uint4*)eo, w, p.dst_row,
                                                       (uint4*)y, p.status, T, c.K, H8);
    return cudaGetLastError();
}

}  // namespace moonep
