// expert_standin.cu -- a stand-in for the expert computation (the grouped GEMM
// over the [E+B, H, H'] weights selected by cu_seqlens, described on
// "Moonshot AI Open-Sources MoonEP ..." (ainovat.com), the contract
// paragraph).  It lets the tests check combine with outputs that depend on
// which expert a row was grouped under.
//
//   identity, bf16 payload: out = recv
//   identity, fp8 payload:  out = bf16(float(q) * scale)
//   scale:                  out = bf16(float(v) * (1 + e/E)), e = the expert of
//                           the row's group (a slot group's expert comes from
//                           slot_expert), v the (dequantised) payload value.
// One warp per row; the row's group is found by binary search in its rank's
// cu_seqlens.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.cuh"

namespace moonep {
namespace {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3);
    return __half2float(__half(h));
}

__global__ void __launch_bounds__(THREADS) expert_kernel(const void* __restrict__ recv,
                                                        const float* __restrict__ recv_scale,
                                                        uint4* __restrict__ out,
                                                        const int32_t* __restrict__ cu_seqlens,
                                                        const int32_t* __restrict__ slot_expert,
                                                        const int32_t* __restrict__ status,
                                                        int R, int C, int E, int B, int H8,
                                                        int mode, int fp8) {
    if (!block_status_ok(status)) return;
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)R * C;
    const long long nw = (long long)gridDim.x * WARPS;
    for (long long row = (long long)blockIdx.x * WARPS + (threadIdx.x >> 5); row < rows;
         row += nw) {
        float scale = 1.0f;
        if (mode == MOONEP_EXPERT_SCALE) {
            const int r = (int)(row / C), i = (int)(row % C);
            const int32_t* cu = cu_seqlens + (long long)r * (E + B);
            int lo = 0, hi = E + B;  // first group g with cu[g] > i
            while (lo < hi) {
                int mid = (lo + hi) >> 1;
                if (__ldg(cu + mid) <= i) lo = mid + 1;
                else hi = mid;
            }
            const int e = lo < E ? lo : (lo < E + B ? __ldg(slot_expert + r * B + (lo - E)) : 0);
            scale = __fadd_rn(1.0f, __fdiv_rn((float)e, (float)E));
        }
        for (int c = lane; c < H8; c += 32) {
            float f[8];
            if (fp8) {
                const uint2 q = __ldg(reinterpret_cast<const uint2*>(recv) + row * H8 + c);
                const float s = __ldg(recv_scale + row * (H8 / 16) + (c >> 4));
#pragma unroll
                for (int i = 0; i < 4; ++i) f[i] = __fmul_rn(e4m3_to_f32((q.x >> (8 * i)) & 0xff), s);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    f[4 + i] = __fmul_rn(e4m3_to_f32((q.y >> (8 * i)) & 0xff), s);
                if (mode == MOONEP_EXPERT_SCALE) {
                    // the expert sees the dequantised bf16 value
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        f[i] = __bfloat162float(__float2bfloat16_rn(f[i]));
                }
            } else {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(recv) + row * H8 + c);
                f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
                f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
            }
            if (mode == MOONEP_EXPERT_SCALE) {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(f[i], scale);
            }
            uint4 o;
            o.x = pack_bf16x2(f[0], f[1]);
            o.y = pack_bf16x2(f[2], f[3]);
            o.z = pack_bf16x2(f[4], f[5]);
            o.w = pack_bf16x2(f[6], f[7]);
            out[row * H8 + c] = o;
        }
    }
}

}  // namespace

cudaError_t launch_expert_standin(const moonep_config& c, const moonep_plan_t& p,
                                  const void* recv, const float* recv_scale, int mode, void* out,
                                  cudaStream_t s) {
    const long long rows = (long long)c.R * c.S * c.K;
    const int sms = device_sm_count();
    long long grid = (rows + WARPS - 1) / WARPS;
    const long long cap = (long long)sms * (2048 / THREADS);
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    expert_kernel<<<(int)grid, THREADS, 0, s>>>(recv, recv_scale, (uint4*)out, p.cu_seqlens,
                                                p.slot_expert, p.status, c.R, c.S * c.K, c.E, c.B,
                                                c.H / 8, mode, c.payload == MOONEP_PAYLOAD_FP8);
    return cudaGetLastError();
}

}  // namespace moonep
