// plan.cu -- the online MoonEP planner as one cooperative kernel.
//
// What it computes (the pages: "Moonshot AI Open-Sources MoonEP ..." on
// ainovat.com, the paragraphs on maxvio, on the hard S*K invariant and on
// planning redundant experts online; "MoonEP" on moses-y.github.io, "What
// This Does", rows land in their final expert-grouped position):
//   expert histogram, maxvio, per-rank kept rows, the overflow stream cut
//   into segments that fill under-full ranks in rank order, one slot per
//   (expert, receiving rank), cu_seqlens per rank, and the destination row of
//   every (token, k) pick plus its inverse.
//
// Kernel structure (one block per SM, 1024 threads, cooperative launch so
// that every block is resident and the grid-wide waits cannot deadlock):
//   A. each warp owns a contiguous run of picks and builds a private
//      histogram in shared memory (match_any aggregation); the block writes
//      its column hist[e][block].
//   -- grid-wide wait 1 --
//   B. one warp per expert scans its column over the blocks: off[e][block]
//      (exclusive) and cnt[e] (total).
//   -- grid-wide wait 2 --
//   C. every block computes the (small, O(E + R)) balance step itself from
//      cnt[], so no third wait is needed; block 0 writes the per-layer
//      outputs and each block writes cu_seqlens / slot_expert of the ranks it
//      owns; then every warp walks its picks again in (t, k) order and places
//      them: its running per-expert offsets start at off[e][block] plus the
//      counts of the block's earlier warps, so the placement is stable and
//      deterministic without any ordered atomics.
// Every wait is bounded (globaltimer); a wait that runs out records
// MOONEP_STATUS_TIMEOUT and the block returns.
#include <algorithm>

#include "internal.cuh"

namespace moonep {
namespace {

constexpr int THREADS = 1024;
constexpr int NW = THREADS / 32;
constexpr int UNR = 8;  // picks per lane loaded ahead in the streaming loops

struct PlanParams {
    int R, S, E, K, B, rule, Er, C, P;
    int stash;  // 1: the block's picks are kept in shared memory between phases
    const int32_t* idx;
    int32_t* expert_count;
    int32_t* rank_load;
    int32_t* slot_expert;
    int32_t* cu_seqlens;
    int32_t* dst_row;
    int32_t* src_of_row;
    int32_t* status;
    double* maxvio;
    int32_t* hist;  // [E][G]
    int32_t* off;   // [E][G]
    int32_t* cnt;   // [E]
    unsigned long long wait_ns;
    int barrier_extra;
};

struct Smem {
    int* whist;   // [NW][E] per-warp counts, later per-warp running offsets
    int* cnt;     // [E]
    int* kk;      // [E] kept rows of each expert on its home rank
    int* kb;      // [E] first kept row of each expert in its home rank's buffer
    int* os;      // [E] start of the expert's rows in the overflow stream
    int* nzr;     // [E+1] number of experts with overflow before e
    int* nzlist;  // [E] experts with overflow, ascending
    int* kept;    // [R]
    int* def;     // [R] C - kept
    int* segs;    // [R] start of the rank's segment in the stream
    int* sege;    // [R] end of the rank's segment
    int* nsl;     // [R] slots the rank needs
    int* fe;      // [R] first expert of the rank's segment (-1: none)
    int* rload;   // [R] home rows before balancing
    int* scratch; // [72]
    int* idx;     // [chunk] the block's picks (when stashed)
};

__host__ __device__ inline size_t smem_ints(int E, int R) {
    return (size_t)NW * E + 6 * (size_t)E + 1 + 7 * (size_t)R + 72;
}

__device__ inline Smem carve(int* base, int E, int R) {
    Smem s;
    int* p = base;
    s.whist = p; p += NW * E;
    s.cnt = p; p += E;
    s.kk = p; p += E;
    s.kb = p; p += E;
    s.os = p; p += E;
    s.nzr = p; p += E + 1;
    s.nzlist = p; p += E;
    s.kept = p; p += R;
    s.def = p; p += R;
    s.segs = p; p += R;
    s.sege = p; p += R;
    s.nsl = p; p += R;
    s.fe = p; p += R;
    s.rload = p; p += R;
    s.scratch = p; p += 72;
    s.idx = p;
    return s;
}

__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Exclusive prefix sum of one value per thread over the block.
__device__ int block_scan_excl(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = warp_incl_scan(v, lane);
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int t = lane < NW ? scratch[lane] : 0;
        t = warp_incl_scan(t, lane);
        scratch[32 + lane] = t;
    }
    __syncthreads();
    int base = warp ? scratch[32 + warp - 1] : 0;
    int tot = scratch[32 + NW - 1];
    __syncthreads();
    if (total) *total = tot;
    return base + x - v;
}

// First index i in [0, n) with a[i] > v (n if none).
__device__ __forceinline__ int upper_bound(const int* a, int n, int v) {
    int lo = 0, hi = n;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (a[mid] <= v) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// Grid-wide wait with a time limit.  Returns false if it ran out.
__device__ bool grid_wait(unsigned* ctr, unsigned target, unsigned long long limit_ns, int* flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        red_release_add_u32(ctr, 1u);
        const unsigned long long t0 = globaltimer_ns();
        int ok = 1;
        while (ld_acquire_u32(ctr) < target) {
            if (globaltimer_ns() - t0 > limit_ns) {
                ok = 0;
                break;
            }
            __nanosleep(64);
        }
        __threadfence();
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

// The balance step.  Every block runs it on the same cnt[] and reaches the
// same result.  Returns the plan status (OK or SLOT_BUDGET).
__device__ int balance(const PlanParams& p, Smem& s, int* fail_rank, int* fail_slots) {
    const int tid = threadIdx.x;
    const int E = p.E, R = p.R, Er = p.Er, C = p.C, B = p.B;
    const bool ve = tid < E;
    const int e = tid;
    const int c = ve ? s.cnt[e] : 0;
    const int first = ve ? (e / Er) * Er : 0;

    // rows of lower-priority experts of the same rank that are kept first
    int q = 0;
    if (p.rule == MOONEP_RULE_INDEX_ORDER) {
        int pre = block_scan_excl(c, s.scratch, nullptr);
        if (ve) s.kb[e] = pre;
        __syncthreads();
        if (ve) q = pre - s.kb[first];
        __syncthreads();
    } else {
        if (ve) {
            for (int i = 0; i < Er; ++i) {
                int e2 = first + i, c2 = s.cnt[e2];
                if (c2 < c || (c2 == c && e2 < e)) q += c2;
            }
        }
    }
    const long long room = (long long)C - q;
    const int k = ve ? (int)min((long long)c, max(room, 0LL)) : 0;
    if (ve) s.kk[e] = k;

    // first kept row of each expert in its home rank (index order)
    int prek = block_scan_excl(k, s.scratch, nullptr);
    if (ve) s.kb[e] = prek;
    __syncthreads();
    int kbv = ve ? prek - s.kb[first] : 0;
    __syncthreads();
    if (ve) s.kb[e] = kbv;

    // overflow stream offsets and the list of experts that overflow
    const int o = c - k;
    int osv = block_scan_excl(o, s.scratch, nullptr);
    const int flag = (ve && o > 0) ? 1 : 0;
    int nz_tot = 0;
    int nzv = block_scan_excl(flag, s.scratch, &nz_tot);
    if (ve) {
        s.os[e] = osv;
        s.nzr[e] = nzv;
        if (flag) s.nzlist[nzv] = e;
    }
    if (tid == 0) s.nzr[E] = nz_tot;
    __syncthreads();

    // ranks: kept rows, deficits, segments
    int kept = 0, load = 0;
    if (tid < R) {
        for (int i = 0; i < Er; ++i) {
            kept += s.kk[tid * Er + i];
            load += s.cnt[tid * Er + i];
        }
    }
    const int d = tid < R ? C - kept : 0;
    int segsv = block_scan_excl(d, s.scratch, nullptr);
    if (tid < R) {
        s.kept[tid] = kept;
        s.rload[tid] = load;
        s.def[tid] = d;
        s.segs[tid] = segsv;
        s.sege[tid] = segsv + d;
        int nsl = 0, fe = -1;
        if (d > 0) {
            fe = upper_bound(s.os, E, segsv) - 1;
            int le = upper_bound(s.os, E, segsv + d - 1) - 1;
            nsl = s.nzr[le] - s.nzr[fe] + 1;
        }
        s.nsl[tid] = nsl;
        s.fe[tid] = fe;
    }
    __syncthreads();
    int st = MOONEP_STATUS_OK;
    *fail_rank = -1;
    *fail_slots = 0;
    for (int r = 0; r < R; ++r) {
        if (s.nsl[r] > B) {
            st = MOONEP_STATUS_SLOT_BUDGET;
            *fail_rank = r;
            *fail_slots = s.nsl[r];
            break;
        }
    }
    return st;
}

__global__ void __launch_bounds__(THREADS, 1) plan_kernel(PlanParams p) {
    extern __shared__ int smem_raw[];
    Smem s = carve(smem_raw, p.E, p.R);
    __shared__ int wait_flag;
    __shared__ int max_count;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, b = blockIdx.x;
    const int E = p.E;
    const long long P = p.P;
    const long long clo = P * b / G, chi = P * (b + 1) / G, len = chi - clo;
    const long long wlo = clo + len * warp / NW, whi = clo + len * (warp + 1) / NW;
    int* wh = s.whist + warp * E;

    // ---- A: per-warp histograms ----------------------------------------
    for (int i = tid; i < NW * E; i += THREADS) s.whist[i] = 0;
    if (tid == 0) max_count = 0;
    __syncthreads();
    int bad = 0;
    for (long long base = wlo; base < whi; base += 32 * UNR) {
        int ev[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            long long q = base + u * 32 + lane;
            ev[u] = q < whi ? __ldg(p.idx + q) : -1;
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            long long q = base + u * 32 + lane;
            int e = ev[u];
            if (q < whi) {
                if (p.stash) s.idx[q - clo] = e;
                if (e < 0 || e >= E) {
                    bad = 1;
                    e = -1;
                }
            }
            unsigned peers = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(peers) - 1) wh[e] += __popc(peers);
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status + ST_BAD_FLAG, 1);
    __syncthreads();
    for (int e = tid; e < E; e += THREADS) {
        int t = 0;
        for (int w = 0; w < NW; ++w) t += s.whist[w * E + e];
        p.hist[(long long)e * G + b] = t;
    }

    if (!grid_wait(reinterpret_cast<unsigned*>(p.status + ST_BARRIER1),
                   (unsigned)(G + p.barrier_extra), p.wait_ns, &wait_flag)) {
        if (tid == 0) atomicMax(p.status + ST_STATUS, MOONEP_STATUS_TIMEOUT);
        return;
    }

    // ---- B: column scans over the blocks, one warp per expert -------------
    {
        const int gw = b * NW + warp, GW = G * NW;
        for (int e = gw; e < E; e += GW) {
            const int32_t* col = p.hist + (long long)e * G;
            int32_t* ocol = p.off + (long long)e * G;
            int carry = 0;
            for (int base = 0; base < G; base += 32) {
                int i = base + lane;
                int v = i < G ? __ldcg(col + i) : 0;
                int x = warp_incl_scan(v, lane);
                if (i < G) ocol[i] = carry + x - v;
                carry += __shfl_sync(0xffffffffu, x, 31);
            }
            if (lane == 0) p.cnt[e] = carry;
        }
    }

    if (!grid_wait(reinterpret_cast<unsigned*>(p.status + ST_BARRIER2), (unsigned)G, p.wait_ns,
                   &wait_flag)) {
        if (tid == 0) atomicMax(p.status + ST_STATUS, MOONEP_STATUS_TIMEOUT);
        return;
    }
    if (__ldcg(p.status + ST_BAD_FLAG)) {
        if (b == 0 && tid == 0) atomicMax(p.status + ST_STATUS, MOONEP_STATUS_BAD_INDEX);
        return;
    }

    // ---- C: balance step (every block), outputs, placement ---------------
    for (int e = tid; e < E; e += THREADS) {
        int c = __ldcg(p.cnt + e);
        s.cnt[e] = c;
        atomicMax(&max_count, c);
    }
    __syncthreads();
    int fail_rank, fail_slots;
    const int st = balance(p, s, &fail_rank, &fail_slots);

    if (b == 0) {
        for (int e = tid; e < E; e += THREADS) p.expert_count[e] = s.cnt[e];
        for (int r = tid; r < p.R; r += THREADS) p.rank_load[r] = s.rload[r];
        if (tid == 0) {
            const int mx = max_count;
            const double tbar = __ddiv_rn((double)P, (double)E);
            p.maxvio[0] = __dsub_rn(__ddiv_rn((double)mx, tbar), 1.0);
            p.status[ST_MAX_COUNT] = mx;
            p.status[ST_FAIL_RANK] = fail_rank;
            p.status[ST_FAIL_SLOTS] = fail_slots;
            atomicMax(p.status + ST_STATUS, st);
        }
    }
    if (st != MOONEP_STATUS_OK) return;

    const int R = p.R, B = p.B, Er = p.Er, C = p.C;
    for (int r = b; r < R; r += G) {
        const int kept = s.kept[r], d = s.def[r], segs = s.segs[r], sege = s.sege[r];
        const int nsl = s.nsl[r], fe = s.fe[r];
        const int nz0 = fe >= 0 ? s.nzr[fe] : 0;
        for (int g = tid; g < E + B; g += THREADS) {
            int v;
            if (g < E) {
                const int h = g / Er;
                v = h < r ? 0 : (h > r ? kept : s.kb[g] + s.kk[g]);
            } else {
                const int j = g - E;
                if (j < nsl) {
                    const int e = s.nzlist[nz0 + j];
                    const int end = min(s.os[e] + (s.cnt[e] - s.kk[e]), sege);
                    v = kept + end - segs;
                } else {
                    v = kept + d;
                }
            }
            p.cu_seqlens[(long long)r * (E + B) + g] = v;
        }
        for (int j = tid; j < B; j += THREADS)
            p.slot_expert[r * B + j] = j < nsl ? s.nzlist[nz0 + j] : -1;
    }

    // per-warp running offsets: block offset + earlier warps' counts
    for (int e = tid; e < E; e += THREADS) {
        int run = __ldcg(p.off + (long long)e * G + b);
        for (int w = 0; w < NW; ++w) {
            int t = s.whist[w * E + e];
            s.whist[w * E + e] = run;
            run += t;
        }
    }
    __syncthreads();

    const unsigned lt_mask = (1u << lane) - 1u;
    for (long long base = wlo; base < whi; base += 32 * UNR) {
        int ev[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            long long q = base + u * 32 + lane;
            ev[u] = q < whi ? (p.stash ? s.idx[q - clo] : __ldg(p.idx + q)) : -1;
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const long long q = base + u * 32 + lane;
            const int e = ev[u];
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            int pos = 0;
            if (e >= 0) pos = wh[e] + __popc(peers & lt_mask);
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) wh[e] += __popc(peers);
            __syncwarp();
            if (e >= 0) {
                const int k = s.kk[e];
                int dst = -1;
                if (pos < k) {
                    dst = (e / Er) * C + s.kb[e] + pos;
                } else {
                    const int sidx = s.os[e] + pos - k;
                    const int rho = upper_bound(s.sege, R, sidx);
                    if (rho < R) dst = rho * C + s.kept[rho] + (sidx - s.segs[rho]);
                }
                if (dst >= 0 && dst < p.P && pos < s.cnt[e]) {
                    p.dst_row[q] = dst;
                    p.src_of_row[dst] = (int)q;
                } else {
                    // never expected: report instead of writing out of range
                    atomicMax(p.status + ST_STATUS, MOONEP_STATUS_INTERNAL);
                }
            }
        }
    }
}

struct DevInfo {
    int sms = 0;
    int max_smem_optin = 0;
};

DevInfo dev_info() {
    static thread_local int cached_dev = -1;
    static thread_local DevInfo info;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != cached_dev) {
        cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&info.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cached_dev = dev;
    }
    return info;
}

}  // namespace

int device_sm_count() { return dev_info().sms; }

size_t plan_workspace_bytes(int E) {
    size_t ints = 2 * (size_t)E * MAX_GRID + (size_t)E;
    return ((ints * 4) + 255) / 256 * 256;
}

cudaError_t launch_plan(const PlanLaunch& a, cudaStream_t stream, const char** why) {
    const DevInfo info = dev_info();
    const int G = std::min(info.sms, MAX_GRID);
    PlanParams p;
    p.R = a.R; p.S = a.S; p.E = a.E; p.K = a.K; p.B = a.B; p.rule = a.rule;
    p.Er = a.E / a.R;
    p.C = a.S * a.K;
    p.P = a.R * a.S * a.K;
    p.idx = a.idx;
    p.expert_count = a.plan.expert_count;
    p.rank_load = a.plan.rank_load;
    p.slot_expert = a.plan.slot_expert;
    p.cu_seqlens = a.plan.cu_seqlens;
    p.dst_row = a.plan.dst_row;
    p.src_of_row = a.plan.src_of_row;
    p.status = a.plan.status;
    p.maxvio = a.plan.maxvio;
    int32_t* ws = static_cast<int32_t*>(a.plan.workspace);
    p.hist = ws;
    p.off = ws + (size_t)a.E * MAX_GRID;
    p.cnt = ws + 2 * (size_t)a.E * MAX_GRID;
    p.wait_ns = a.wait_ns;
    p.barrier_extra = a.barrier_extra;

    const size_t base_bytes = smem_ints(a.E, a.R) * 4;
    const long long chunk = ((long long)p.P + G - 1) / G;
    size_t smem = base_bytes;
    p.stash = 0;
    if (base_bytes + (size_t)chunk * 4 <= (size_t)info.max_smem_optin - 1024) {
        p.stash = 1;
        smem = base_bytes + (size_t)chunk * 4;
    }
    if (smem > (size_t)info.max_smem_optin) {
        *why = "planner shared memory exceeds the device limit (E or R too large)";
        return cudaErrorInvalidValue;
    }
    cudaError_t err = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, plan_kernel, THREADS, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) {
        *why = "planner block does not fit on an SM";
        return cudaErrorInvalidConfiguration;
    }
    // status block: status, fail info, wait counters and the bad-index flag
    err = cudaMemsetAsync(a.plan.status, 0, MOONEP_STATUS_WORDS * sizeof(int32_t), stream);
    if (err != cudaSuccess) return err;
    void* args[] = {&p};
    return cudaLaunchCooperativeKernel((const void*)plan_kernel, dim3(G), dim3(THREADS), args, smem,
                                       stream);
}

}  // namespace moonep
