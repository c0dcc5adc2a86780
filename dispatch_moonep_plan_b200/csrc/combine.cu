// combine.cu -- gather each token's K expert-output rows back and reduce them
// with the router weights ("MoonEP" on moses-y.github.io, "What This Does"
// and "Real-World Use").
//
// y[t] = bf16(acc), acc = 0; for k = 0..K-1: acc = fma(w[t,k], x_k, acc),
// x_k = float(expert_out[dst_row[t,k]]), all in binary32, one rounding to
// bf16 (nearest even) at the end.  The k order is fixed, so the result does
// not depend on the launch shape.
//
// Up to K = 8 with H a multiple of 512 and at least 4096: the K rows'
// 512-element chunks are staged in shared memory by bulk copies (one
// cp.async.bulk per row and chunk, completion on an mbarrier), two stages per
// warp, so the next chunk is in flight while this one is summed.  Otherwise
// one warp per token reads the rows with 16-byte loads: lane k < K holds
// dst_row[t,k] and w[t,k]; each lane owns U 16-byte chunks of the row and
// accumulates 8 floats per chunk; up to K = 8 it loads its chunks of all K
// rows before accumulating, above that the next pick's chunks are loaded while
// the current ones are accumulated.
#include <cuda_bf16.h>

#include <mutex>

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

template <bool WEIGHTED>
__device__ __forceinline__ float step(float acc, float wk, float v) {
    return WEIGHTED ? __fmaf_rn(wk, v, acc) : __fadd_rn(acc, v);
}

template <bool WEIGHTED>
__device__ __forceinline__ void accum(float* acc, float wk, const uint4& v) {
    acc[0] = step<WEIGHTED>(acc[0], wk, bf16_lo(v.x));
    acc[1] = step<WEIGHTED>(acc[1], wk, bf16_hi(v.x));
    acc[2] = step<WEIGHTED>(acc[2], wk, bf16_lo(v.y));
    acc[3] = step<WEIGHTED>(acc[3], wk, bf16_hi(v.y));
    acc[4] = step<WEIGHTED>(acc[4], wk, bf16_lo(v.z));
    acc[5] = step<WEIGHTED>(acc[5], wk, bf16_hi(v.z));
    acc[6] = step<WEIGHTED>(acc[6], wk, bf16_lo(v.w));
    acc[7] = step<WEIGHTED>(acc[7], wk, bf16_hi(v.w));
}


// WEIGHTED = false is the backward of dispatch: dx[t] = bf16(sum_k rows),
// binary32 additions in k order from zero.
template <int U, bool WEIGHTED>
__global__ void __launch_bounds__(THREADS) combine_kernel(const uint4* __restrict__ eo,
                                                         const float* __restrict__ w,
                                                         const int32_t* __restrict__ dst_row,
                                                         uint4* __restrict__ y,
                                                         int32_t* status, int T,
                                                         int K, int H8) {
    if (!block_status_ok(status)) return;
    const int lane = threadIdx.x & 31;
    const long long nw = (long long)gridDim.x * WARPS;
    for (long long i = (long long)blockIdx.x * WARPS + (threadIdx.x >> 5); i < T; i += nw) {
        // combine takes the tokens last to first: dispatch wrote the rows of
        // the last tokens last, so those are the rows still held in L2
        const long long t = WEIGHTED ? T - 1 - i : i;
        int myrow = lane < K ? __ldg(dst_row + t * K + lane) : 0;
        if ((unsigned)myrow >= (unsigned)(T * K)) {  // range guard: report, read row 0
            report_internal(status);
            myrow = 0;
        }
        const float myw = (WEIGHTED && lane < K) ? __ldg(w + t * K + lane) : 1.0f;
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
                for (int u = 0; u < U; ++u) accum<WEIGHTED>(acc[u], wk, cur[u]);
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

// Up to 8 picks (the usual K): every lane first loads its U chunks of all K
// rows (up to 8*U 16-byte loads in flight), then accumulates them in k order
// with the same fma chain.  Measured against the double-buffered form above:
// 1.01-1.05 of the copy peak instead of 0.91-0.98 (the loads no longer wait
// on one another; combine reads six to eight times what it writes, so it can
// pass a copy's 1:1 rate).
template <int U, int KMAX, bool WEIGHTED>
__global__ void __launch_bounds__(THREADS) combine_kfirst_kernel(const uint4* __restrict__ eo,
                                                                const float* __restrict__ w,
                                                                const int32_t* __restrict__ dst_row,
                                                                uint4* __restrict__ y,
                                                                int32_t* status, int T, int K,
                                                                int H8) {
    if (!block_status_ok(status)) return;
    const int lane = threadIdx.x & 31;
    const long long nw = (long long)gridDim.x * WARPS;
    for (long long i = (long long)blockIdx.x * WARPS + (threadIdx.x >> 5); i < T; i += nw) {
        // combine takes the tokens last to first: dispatch wrote the rows of
        // the last tokens last, so those are the rows still held in L2
        const long long t = WEIGHTED ? T - 1 - i : i;
        int myrow = lane < K ? __ldg(dst_row + t * K + lane) : 0;
        if ((unsigned)myrow >= (unsigned)(T * K)) {  // range guard: report, read row 0
            report_internal(status);
            myrow = 0;
        }
        const float myw = (WEIGHTED && lane < K) ? __ldg(w + t * K + lane) : 1.0f;
        long long base[KMAX];
        float wk[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            base[k] = (long long)__shfl_sync(0xffffffffu, myrow, k < K ? k : 0) * H8;
            wk[k] = __shfl_sync(0xffffffffu, myw, k < K ? k : 0);
        }
        for (int c0 = 0; c0 < H8; c0 += 32 * U) {
            uint4 ev[KMAX][U];
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                if (k < K)
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        ev[k][u] = c < H8 ? ld_stream_v4(eo + base[k] + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c >= H8) continue;
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
                for (int k = 0; k < KMAX; ++k)
                    if (k < K) accum<WEIGHTED>(acc, wk[k], ev[k][u]);
                uint4 o;
                o.x = pack_bf16x2(acc[0], acc[1]);
                o.y = pack_bf16x2(acc[2], acc[3]);
                o.z = pack_bf16x2(acc[4], acc[5]);
                o.w = pack_bf16x2(acc[6], acc[7]);
                y[t * H8 + c] = o;
            }
        }
    }
}

// Backward of combine: for each pick, d_eo[row] = bf16(w * float(dy[t])) (one
// binary32 product), and d_w[t,k] = sum_h dy[t,h] * eo[row,h] in binary32:
// each lane sums its own elements with an fma chain in a fixed order (its
// chunks in increasing position, the 8 elements of a chunk in order), then a
// fixed xor-shuffle tree adds the 32 lane sums, so the result depends only on
// H, not on the launch.
// Up to 8 picks (the usual K): every lane first loads its U chunks of dy and
// of all K expert-output rows (up to 9*U 16-byte loads in flight per lane),
// then does the arithmetic and the K stores.  Measured against loading each
// pick's row just before its use: 0.92-0.96 of the copy peak instead of
// 0.72-0.74 (the loads no longer wait on one another).
template <int U, int KMAX>
__global__ void __launch_bounds__(THREADS, 2) combine_bwd_kernel(const uint4* __restrict__ dy,
                                                             const uint4* __restrict__ eo,
                                                             const float* __restrict__ w,
                                                             const int32_t* __restrict__ dst_row,
                                                             uint4* __restrict__ d_eo,
                                                             float* __restrict__ d_w,
                                                             int32_t* status, int T, int K,
                                                             int H8) {
    if (!block_status_ok(status)) return;
    const int lane = threadIdx.x & 31;
    const int P = T * K;
    const long long nw = (long long)gridDim.x * WARPS;
    for (long long t = (long long)blockIdx.x * WARPS + (threadIdx.x >> 5); t < T; t += nw) {
        int myrow = lane < K ? __ldg(dst_row + t * K + lane) : 0;
        if ((unsigned)myrow >= (unsigned)P) {  // range guard: report, use row 0
            report_internal(status);
            myrow = 0;
        }
        const float myw = lane < K ? __ldg(w + t * K + lane) : 0.0f;
        long long base[KMAX];
        float wk[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            base[k] = (long long)__shfl_sync(0xffffffffu, myrow, k < K ? k : 0) * H8;
            wk[k] = __shfl_sync(0xffffffffu, myw, k < K ? k : 0);
        }
        float part[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) part[k] = 0.0f;
        for (int c0 = 0; c0 < H8; c0 += 32 * U) {
            uint4 gv[U];
            uint4 ev[KMAX][U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                gv[u] = c < H8 ? ld_stream_v4(dy + t * H8 + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                if (k < K)
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        ev[k][u] = c < H8 ? ld_stream_v4(eo + base[k] + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c >= H8) continue;
                const float g[8] = {bf16_lo(gv[u].x), bf16_hi(gv[u].x), bf16_lo(gv[u].y),
                                    bf16_hi(gv[u].y), bf16_lo(gv[u].z), bf16_hi(gv[u].z),
                                    bf16_lo(gv[u].w), bf16_hi(gv[u].w)};
#pragma unroll
                for (int k = 0; k < KMAX; ++k)
                    if (k < K) {
                        const uint4 v = ev[k][u];
                        const float e[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                                            bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
                        for (int i = 0; i < 8; ++i) part[k] = __fmaf_rn(g[i], e[i], part[k]);
                        uint4 o;
                        o.x = pack_bf16x2(__fmul_rn(wk[k], g[0]), __fmul_rn(wk[k], g[1]));
                        o.y = pack_bf16x2(__fmul_rn(wk[k], g[2]), __fmul_rn(wk[k], g[3]));
                        o.z = pack_bf16x2(__fmul_rn(wk[k], g[4]), __fmul_rn(wk[k], g[5]));
                        o.w = pack_bf16x2(__fmul_rn(wk[k], g[6]), __fmul_rn(wk[k], g[7]));
                        st_stream_v4(d_eo + base[k] + c, o);
                    }
            }
        }
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (k < K) {
                float v = part[k];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
                if (lane == 0) d_w[t * K + k] = v;
            }
        }
    }
}

// More than 8 picks: the same arithmetic, one pick's row loaded at a time.
template <int U, int KMAX>
__global__ void __launch_bounds__(THREADS) combine_bwd_seq_kernel(const uint4* __restrict__ dy,
                                                             const uint4* __restrict__ eo,
                                                             const float* __restrict__ w,
                                                             const int32_t* __restrict__ dst_row,
                                                             uint4* __restrict__ d_eo,
                                                             float* __restrict__ d_w,
                                                             int32_t* status, int T, int K,
                                                             int H8) {
    if (!block_status_ok(status)) return;
    const int lane = threadIdx.x & 31;
    const int P = T * K;
    const long long nw = (long long)gridDim.x * WARPS;
    for (long long t = (long long)blockIdx.x * WARPS + (threadIdx.x >> 5); t < T; t += nw) {
        int myrow = lane < K ? __ldg(dst_row + t * K + lane) : 0;
        if ((unsigned)myrow >= (unsigned)P) {  // range guard: report, use row 0
            report_internal(status);
            myrow = 0;
        }
        const float myw = lane < K ? __ldg(w + t * K + lane) : 0.0f;
        float part[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) part[k] = 0.0f;
        const uint4* g_src = dy + t * H8;
        for (int c0 = 0; c0 < H8; c0 += 32 * U) {
            float g[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                const uint4 v = c < H8 ? ld_stream_v4(g_src + c) : make_uint4(0, 0, 0, 0);
                g[u][0] = bf16_lo(v.x); g[u][1] = bf16_hi(v.x); g[u][2] = bf16_lo(v.y);
                g[u][3] = bf16_hi(v.y); g[u][4] = bf16_lo(v.z); g[u][5] = bf16_hi(v.z);
                g[u][6] = bf16_lo(v.w); g[u][7] = bf16_hi(v.w);
            }
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k < K) {
                    const long long row = __shfl_sync(0xffffffffu, myrow, k);
                    const float wk = __shfl_sync(0xffffffffu, myw, k);
                    const uint4* src = eo + row * H8;
                    uint4* dst = d_eo + row * H8;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        if (c < H8) {
                            const uint4 v = ld_stream_v4(src + c);
                            const float e[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y),
                                                bf16_hi(v.y), bf16_lo(v.z), bf16_hi(v.z),
                                                bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
                            for (int i = 0; i < 8; ++i) part[k] = __fmaf_rn(g[u][i], e[i], part[k]);
                            uint4 o;
                            o.x = pack_bf16x2(__fmul_rn(wk, g[u][0]), __fmul_rn(wk, g[u][1]));
                            o.y = pack_bf16x2(__fmul_rn(wk, g[u][2]), __fmul_rn(wk, g[u][3]));
                            o.z = pack_bf16x2(__fmul_rn(wk, g[u][4]), __fmul_rn(wk, g[u][5]));
                            o.w = pack_bf16x2(__fmul_rn(wk, g[u][6]), __fmul_rn(wk, g[u][7]));
                            st_stream_v4(dst + c, o);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (k < K) {
                float v = part[k];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
                if (lane == 0) d_w[t * K + k] = v;
            }
        }
    }
}


__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Combine with the rows staged by bulk copies.  Each of the block's 8 warps
// owns two stages of KMAX x CH bf16 in shared memory; for each (token, chunk)
// of its tokens (last to first, like the loads-first kernel), lane k < K
// copies row k's chunk into the stage with one cp.async.bulk, whose completion
// the stage's mbarrier counts in bytes; the following (token, chunk) is in
// flight while this one is summed.  The same fma chain in k order and one
// bf16 rounding: bit-identical to the kernels above.  Every wait is bounded;
// one that runs out sets TIMEOUT, lets the other stage's copies land (bounded)
// and stops the warp.
template <int CH, int KMAX>
__global__ void __launch_bounds__(THREADS, 1) combine_bulk_kernel(const uint16_t* __restrict__ eo,
                                                                 const float* __restrict__ w,
                                                                 const int32_t* __restrict__ dst_row,
                                                                 uint4* __restrict__ y,
                                                                 int32_t* status, int T, int K,
                                                                 int H,
                                                                 unsigned long long wait_ns) {
    static_assert(CH % 256 == 0, "whole 16-byte vectors per lane");
    if (!block_status_ok(status)) return;
    extern __shared__ __align__(1024) uint8_t stage_mem[];
    __shared__ __align__(8) uint64_t bars[WARPS][2];
    constexpr int STAGE = KMAX * CH * 2;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* buf = stage_mem + warp * 2 * STAGE;
    if (lane == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[warp][0])));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[warp][1])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    const int P = T * K;
    const int nch = H / CH;
    const long long nw = (long long)gridDim.x * WARPS;
    const long long wid = (long long)blockIdx.x * WARPS + warp;
    const long long nitems = (wid < T ? (T - 1 - wid) / nw + 1 : 0) * nch;
    // item i: chunk i % nch of token T - 1 - (wid + (i / nch) * nw)
    auto issue = [&](long long i, int st) {
        const long long t = T - 1 - (wid + (i / nch) * nw);
        const int c = (int)(i % nch);
        int row = lane < K ? __ldg(dst_row + t * K + lane) : 0;
        if (lane < K && (unsigned)row >= (unsigned)P) {  // range guard: report, read row 0
            report_internal(status);
            row = 0;
        }
        uint64_t* bar = &bars[warp][st];
        if (lane == 0)
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                             smem_u32(bar)),
                         "r"((uint32_t)(K * CH * 2))
                         : "memory");
        __syncwarp();
        // the stage was read by generic loads; order them before the copy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (lane < K) {
            const uint16_t* src = eo + (long long)row * H + (long long)c * CH;
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
                "[%3];" ::"r"(smem_u32(buf + st * STAGE + lane * CH * 2)),
                "l"(src), "r"((uint32_t)(CH * 2)), "r"(smem_u32(bar))
                : "memory");
        }
    };
    auto wait_stage = [&](int st, uint32_t parity, unsigned long long limit) -> bool {
        const unsigned long long t0 = globaltimer_ns();
        for (int it = 1;; ++it) {
            uint32_t done;
            asm volatile(
                "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
                "selp.u32 %0, 1, 0, p; }"
                : "=r"(done)
                : "r"(smem_u32(&bars[warp][st])), "r"(parity)
                : "memory");
            if (done) return true;
            if ((it & 63) == 0 && globaltimer_ns() - t0 > limit) return false;
        }
    };
    uint32_t ph[2] = {0, 0};
    if (nitems > 0) issue(0, 0);
    for (long long i = 0; i < nitems; ++i) {
        const int st = (int)(i & 1);
        if (i + 1 < nitems) issue(i + 1, st ^ 1);
        if (!wait_stage(st, ph[st], wait_ns)) {
            if (lane == 0) atomicMax(status + ST_STATUS, MOONEP_STATUS_TIMEOUT);
            if (i + 1 < nitems) wait_stage(st ^ 1, ph[st ^ 1], wait_ns);  // its copies land first
            return;
        }
        ph[st] ^= 1;
        const long long t = T - 1 - (wid + (i / nch) * nw);
        const int c = (int)(i % nch);
        const float myw = lane < K ? __ldg(w + t * K + lane) : 0.0f;
        constexpr int V = CH / 256;  // 16-byte vectors per lane
        float acc[8 * V];
#pragma unroll
        for (int j = 0; j < 8 * V; ++j) acc[j] = 0.0f;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (k < K) {
                const float wk = __shfl_sync(0xffffffffu, myw, k);
                const uint4* rowv = reinterpret_cast<const uint4*>(buf + st * STAGE + k * CH * 2);
#pragma unroll
                for (int v = 0; v < V; ++v) accum<true>(acc + 8 * v, wk, rowv[v * 32 + lane]);
            }
        }
        uint4* dst = y + (t * H + (long long)c * CH) / 8;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            uint4 o;
            o.x = pack_bf16x2(acc[8 * v + 0], acc[8 * v + 1]);
            o.y = pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]);
            o.z = pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]);
            o.w = pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]);
            dst[v * 32 + lane] = o;
        }
        __syncwarp();  // the stage is read before it is refilled
    }
}

int grid_4_per_sm(long long T) {
    const int sms = device_sm_count();
    long long grid = (T + WARPS - 1) / WARPS;
    const long long cap = (long long)sms * 4;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return (int)grid;
}

// One warp per token, up to 256 blocks per SM (about 128 registers: two
// blocks resident; the block scheduler balances the rest).
int grid_warp_per_token(long long T) {
    const int sms = device_sm_count();
    long long grid = (T + WARPS - 1) / WARPS;
    const long long cap = (long long)sms * 256;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return (int)grid;
}

}  // namespace

cudaError_t launch_dispatch_backward(const moonep_config& c, const moonep_plan_t& p,
                                     const void* d_recv, void* dx, cudaStream_t s) {
    const int T = c.R * c.S;
    const int H8 = c.H / 8;
    if (c.K <= 8) {
        combine_kfirst_kernel<2, 8, false><<<grid_warp_per_token(T), THREADS, 0, s>>>(
            (const uint4*)d_recv, nullptr, p.dst_row, (uint4*)dx, p.status, T, c.K, H8);
        return cudaGetLastError();
    }
    const int grid = grid_4_per_sm(T);
    if (H8 >= 64)
        combine_kernel<2, false><<<grid, THREADS, 0, s>>>((const uint4*)d_recv, nullptr, p.dst_row,
                                                          (uint4*)dx, p.status, T, c.K, H8);
    else
        combine_kernel<1, false><<<grid, THREADS, 0, s>>>((const uint4*)d_recv, nullptr, p.dst_row,
                                                          (uint4*)dx, p.status, T, c.K, H8);
    return cudaGetLastError();
}

cudaError_t launch_combine_backward(const moonep_config& c, const moonep_plan_t& p, const void* dy,
                                    const void* eo, const float* w, void* d_eo, float* d_w,
                                    cudaStream_t s) {
    const int T = c.R * c.S;
    const int H8 = c.H / 8;
    const int grid = grid_4_per_sm(T);
    const uint4* dy4 = (const uint4*)dy;
    const uint4* eo4 = (const uint4*)eo;
    uint4* de4 = (uint4*)d_eo;
    if (c.K <= 8) {
        // about 128 registers: 2 blocks resident per SM; one warp per token
        // (the block scheduler balances the rest) measured 1.01 of the copy
        // peak at H 2048 and 0.99 at 7168, against 0.98 / 0.96 on 8 blocks
        // per SM
        const int g8 = grid_warp_per_token(T);
        if (H8 >= 64)
            combine_bwd_kernel<2, 8><<<g8, THREADS, 0, s>>>(dy4, eo4, w, p.dst_row, de4, d_w,
                                                                p.status, T, c.K, H8);
        else
            combine_bwd_kernel<1, 8><<<g8, THREADS, 0, s>>>(dy4, eo4, w, p.dst_row, de4, d_w,
                                                                p.status, T, c.K, H8);
    } else {
        combine_bwd_seq_kernel<1, MOONEP_MAX_K><<<grid, THREADS, 0, s>>>(dy4, eo4, w, p.dst_row,
                                                                        de4, d_w, p.status, T, c.K,
                                                                        H8);
    }
    return cudaGetLastError();
}

cudaError_t launch_combine(const moonep_config& c, const moonep_plan_t& p, const void* eo,
                           const float* w, void* y, cudaStream_t s) {
    const int T = c.R * c.S;
    const int H8 = c.H / 8;
    if (c.K <= 8 && c.H % 512 == 0 && c.H >= 4096) {
        // rows staged by bulk copies, 512-element chunks, one block of 8 warps
        // per SM (128 KiB of stages): 1.057-1.061 of the copy peak at H = 4096
        // and 7168 (the loads-first kernel: 1.052-1.057), bit-identical; at
        // H = 2048 (4 chunks a token, K = 6) 0.83 against 1.00, so shorter
        // rows take the loads-first kernel; 256-element chunks on 1-3 blocks
        // per SM measured 0.66-0.97
        constexpr int CH = 512;
        const size_t smem = (size_t)WARPS * 2 * 8 * CH * 2;
        static std::mutex mu;
        static bool set[64] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        {
            std::lock_guard<std::mutex> lock(mu);
            if (dev < 0 || dev >= 64 || !set[dev]) {
                e = cudaFuncSetAttribute(combine_bulk_kernel<CH, 8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (e != cudaSuccess) return e;
                if (dev >= 0 && dev < 64) set[dev] = true;
            }
        }
        long long grid = device_sm_count();
        if (grid > T) grid = T;
        if (grid < 1) grid = 1;
        combine_bulk_kernel<CH, 8><<<(int)grid, THREADS, smem, s>>>(
            (const uint16_t*)eo, w, p.dst_row, (uint4*)y, p.status, T, c.K, c.H,
            current_wait_limit_ns());
        return cudaGetLastError();
    }
    if (c.K <= 8) {
        combine_kfirst_kernel<2, 8, true><<<grid_warp_per_token(T), THREADS, 0, s>>>(
            (const uint4*)eo, w, p.dst_row, (uint4*)y, p.status, T, c.K, H8);
        return cudaGetLastError();
    }
    // more than 8 picks:
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
        combine_kernel<2, true><<<(int)grid, THREADS, 0, s>>>((const uint4*)eo, w, p.dst_row,
                                                             (uint4*)y, p.status, T, c.K, H8);
    else
        combine_kernel<1, true><<<(int)grid, THREADS, 0, s>>>((const uint4*)eo, w, p.dst_row,
                                                             (uint4*)y, p.status, T, c.K, H8);
    return cudaGetLastError();
}

}  // namespace moonep
