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
// that every block is resident and the grid-wide wait cannot deadlock):
//   A. each block owns a contiguous run of picks, each warp a contiguous part
//      of it; every warp ranks its picks 32 at a time in (t, k) order: the
//      lanes holding the same expert are found (one ballot for the warp's
//      candidate expert, lane-mask words in shared memory for the rest, or
//      match.any when the words do not fit), and the group's lowest lane
//      advances the warp's count of that expert; count before the row plus
//      the lane's rank in its group is the pick's position among the warp's
//      picks of the expert, kept beside the pick in shared memory.  One
//      thread per expert then runs over the 32 warps' counts: the block's row
//      hist[block][e] and each warp's offset within the block.
//   -- one grid-wide wait; while it lasts, each block sorts its own picks
//      into expert-major order in shared memory (slot = the block's prefix
//      over experts + the warp's offset + the position in the warp) --
//   B. every block reads all rows of hist (16-byte loads when E % 4 == 0):
//      the per-expert totals, and the counts of the blocks before it (its
//      offsets).
//   C. every block computes the small O(E + R) balance step itself from the
//      totals (no further grid-wide wait is needed); block 0 writes the
//      per-layer outputs, each block writes cu_seqlens / slot_expert of the
//      ranks it owns; then the block places its picks in expert-major order:
//      slot i of expert e is the pick at position i + offset(e) among all
//      picks of e, so the placement is stable and deterministic without
//      ordered atomics.  Its row comes from one 16-byte per-expert table
//      entry (kept rows) or, for overflow, a bucket table over the overflow
//      stream.  Consecutive threads write consecutive rows of the inverse map;
//      the forward map is collected in shared memory and written out in pick
//      order.  When a block's picks do not fit in shared memory, the walk
//      reads them again in (t, k) order and ranks them row by row against
//      running per-warp offsets.
// The wait is bounded (globaltimer); when it runs out the block records
// MOONEP_STATUS_TIMEOUT and returns.
#include <algorithm>

#include "internal.cuh"

namespace moonep {
namespace {

constexpr int THREADS = 1024;
constexpr int NW = THREADS / 32;
constexpr int UNR = 8;   // picks per lane loaded ahead in the streaming loops
constexpr int BUNR = 8;  // histogram rows per thread loaded ahead in phase B
constexpr int SCAN_N = 4;
constexpr int NBKT = 512;  // buckets of the overflow stream (receiving-position lookup)

struct PlanParams {
    int R, S, E, K, B, rule, Er, C, P;
    int stash;  // 1: the block's picks are kept in shared memory between phases
    int chunk;  // shared capacity (ints) of the stash
    const int32_t* idx;
    int32_t* expert_count;
    int32_t* rank_load;
    int32_t* slot_expert;
    int32_t* cu_seqlens;
    int32_t* dst_row;
    int32_t* src_of_row;
    int32_t* status;
    double* maxvio;
    int32_t* hist;  // [G][E]
    unsigned long long wait_ns;
    int barrier_extra;
};

struct Smem {
    int* whist;   // [NW][WS] per-warp counts; then each warp's offset among the
                  //          block's picks of the expert, plus the expert's
                  //          first expert-major slot (picks kept) or the
                  //          block's offset among all its picks (not kept)
    unsigned* wmask;  // [NW][WS] per-warp lane masks of the row being ranked
                      //          (ranking by masks only); shares its space with
    int* sorted;  // [chunk] the block's picks in expert-major order: expert |
                  //         (pick - first pick of the block) << 10 (kept picks)
    int* cnt;     // [E]   picks of each expert (all blocks)
    int* bcnt;    // [E]   picks of each expert in this block
    int* bpre;    // [E]   picks of each expert in the blocks before this one
    int* kk;      // [E]   rows of each expert kept on its home rank
    int* nzlist;  // [E]   experts with overflow, in stream order
    int* bex;     // [E]   exclusive prefix of bcnt over experts (expert-major slots)
    int* pc;      // [E+1] exclusive prefix of cnt over experts
    int* pk;      // [E+1] exclusive prefix of kk over experts
    int* ov;      // [E]   rows of each expert that overflow its home rank
    int* item_at; // [E]   the expert at each position of the overflow stream's order
    int* osi;     // [E+1] start of the stream item at each position (non-decreasing)
    int* nzri;    // [E+1] items with overflow before each position
    int* ose;     // [E]   start of each expert's rows in the overflow stream
    int4* tab;    // [E]   per expert: rows kept, destination row of its first kept
                  //       pick, overflow-stream index of pick 0 (ose - kept), picks;
                  //       on the expert-major path shifted to index by slot
    int* bkt;     // [NBKT] per bucket of 2^sh consecutive overflow-stream indices:
                  //       the receiving positions of its first and last index,
                  //       first | last << 16
    int* kept;    // [R]
    int* def;     // [R] C - kept
    int* segs;    // [R] start of the rank's segment in the stream
    int* sege;    // [R] end of the rank's segment
    int* nsl;     // [R] slots the rank needs
    int* fe;      // [R] stream position of the rank's first item (-1: none)
    int* rload;   // [R] home rows before balancing
    int* recv_at; // [R] the rank at each position of the receiving order
    int* sege_at; // [R] segment end at each position of the receiving order
    int* rbase;   // [R] destination row of stream index 0 at each receiving position
    int* scratch; // [2*SCAN_N*32 + 8]
    int* stash;   // [chunk] the block's picks in (t, k) order, expert | position
                  //         in the warp << 10; later each pick's destination row
};

// Row stride of the per-warp arrays: E rounded up to an odd count of words
// (rows of neighbouring warps start in different banks).
__host__ __device__ inline int warp_stride(int E) { return E | 1; }

__host__ __device__ inline size_t smem_ints(int E, int R, bool mask, bool stash, long long chunk) {
    const size_t nw = (size_t)NW * warp_stride(E);
    const size_t c = stash ? (size_t)chunk : 0;
    const size_t u = mask ? (nw > c ? nw : c) : c;  // wmask and sorted share
    return (size_t)((E + 3) & ~3) + 4 * (size_t)E + nw + u + 6 * (size_t)E +
           4 * ((size_t)E + 1) + 2 * (size_t)E + NBKT + 10 * (size_t)R + 2 * SCAN_N * 32 + 8 + c;
}

__device__ inline Smem carve(int* base, int E, int R, bool mask, bool stash, int chunk) {
    Smem s;
    int* p = base;
    s.ov = p; p += (E + 3) & ~3;  // first and padded: read four at a time
    s.tab = reinterpret_cast<int4*>(p); p += 4 * E;  // 16-byte aligned after ov
    const int nw = NW * warp_stride(E);
    const int c = stash ? chunk : 0;
    s.whist = p; p += nw;
    s.wmask = reinterpret_cast<unsigned*>(p);
    s.sorted = p;
    p += mask ? (nw > c ? nw : c) : c;
    s.cnt = p; p += E;
    s.bcnt = p; p += E;
    s.bpre = p; p += E;
    s.kk = p; p += E;
    s.nzlist = p; p += E;
    s.bex = p; p += E;
    s.pc = p; p += E + 1;
    s.pk = p; p += E + 1;
    s.item_at = p; p += E;
    s.osi = p; p += E + 1;
    s.nzri = p; p += E + 1;
    s.ose = p; p += E;
    s.bkt = p; p += NBKT;
    s.kept = p; p += R;
    s.def = p; p += R;
    s.segs = p; p += R;
    s.sege = p; p += R;
    s.nsl = p; p += R;
    s.fe = p; p += R;
    s.rload = p; p += R;
    s.recv_at = p; p += R;
    s.sege_at = p; p += R;
    s.rbase = p; p += R;
    s.scratch = p; p += 2 * SCAN_N * 32 + 8;
    s.stash = p;
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

// Exclusive prefix sums and totals of N values per thread over the block.
template <int N>
__device__ void block_scan(const int (&v)[N], int (&excl)[N], int (&tot)[N], int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x[N];
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = warp_incl_scan(v[i], lane);
    if (lane == 31) {
#pragma unroll
        for (int i = 0; i < N; ++i) scratch[i * 32 + warp] = x[i];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            int t = lane < NW ? scratch[i * 32 + lane] : 0;
            scratch[(N + i) * 32 + lane] = warp_incl_scan(t, lane);
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int base = warp ? scratch[(N + i) * 32 + warp - 1] : 0;
        excl[i] = base + x[i] - v[i];
        tot[i] = scratch[(N + i) * 32 + NW - 1];
    }
    __syncthreads();
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

// Grid-wide barrier, in two halves so that a block can work on its own data
// between them.  Arrive (after the block's __syncthreads, which orders the
// block's writes before thread 0's next operation): thread 0 counts the block
// in with a release add at gpu scope, which makes those writes visible to
// every thread that acquires the count.
__device__ __forceinline__ void grid_arrive(unsigned* ctr) {
    if (threadIdx.x == 0) red_release_add_u32(ctr, 1u);
}

// Wait, with a time limit, until target blocks have arrived.  Returns false
// if it ran out.
__device__ bool grid_wait(unsigned* ctr, unsigned target, unsigned long long limit_ns, int* flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long t0 = globaltimer_ns();
        int ok = 1;
        // acquire loads: the other blocks' writes before their arrival are
        // visible to thread 0, and to the block after the barrier below
        while (ld_acquire_u32(ctr) < target) {
            if (globaltimer_ns() - t0 > limit_ns) {
                ok = 0;
                break;
            }
        }
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

// The balance step.  Every block runs it on the same totals and reaches the
// same result.  Returns the plan status (OK or SLOT_BUDGET).
__device__ int balance(const PlanParams& p, Smem& s, int* misc) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = p.E, R = p.R, Er = p.Er, C = p.C, B = p.B;
    const bool ve = tid < E;
    const int e = tid;
    const int c = ve ? s.cnt[e] : 0;
    const int first = ve ? (e / Er) * Er : 0;

    // q = rows of the same rank's experts that are kept before expert e
    int q = 0;
    if (p.rule == MOONEP_RULE_INDEX_ORDER && Er <= 32) {
        if (ve)
            for (int i = first; i < e; ++i) q += s.cnt[i];  // at most 31 loads
    } else if (p.rule == MOONEP_RULE_INDEX_ORDER) {
        int v1[1] = {c}, ex1[1], t1[1];
        block_scan<1>(v1, ex1, t1, s.scratch);
        if (ve) s.pc[e] = ex1[0];
        __syncthreads();
        if (ve) q = ex1[0] - s.pc[first];
    } else if (ve) {  // rules 1 and 2: lightest experts first
        for (int i = 0; i < Er; ++i) {
            const int e2 = first + i, c2 = s.cnt[e2];
            if (c2 < c || (c2 == c && e2 < e)) q += c2;
        }
    }
    const long long room = (long long)C - q;
    const int k = ve ? (int)min((long long)c, max(room, 0LL)) : 0;
    const int o = c - k;
    if (ve) {
        s.kk[e] = k;
        s.ov[e] = o;
    }
    // the overflow stream's expert order: index order (rules 0 and 1), or by
    // decreasing overflow, ties to the lower index (rule 2)
    int ip = e;
    if (p.rule == MOONEP_RULE_LARGEST_FIRST) {
        __syncthreads();
        if (ve) {  // rank by counting; four experts per (broadcast) shared load
            ip = 0;
            const int E4 = E & ~3;
            for (int e2 = 0; e2 < E4; e2 += 4) {
                const int4 o4 = *reinterpret_cast<const int4*>(s.ov + e2);
                ip += (o4.x > o) || (o4.x == o && e2 < e);
                ip += (o4.y > o) || (o4.y == o && e2 + 1 < e);
                ip += (o4.z > o) || (o4.z == o && e2 + 2 < e);
                ip += (o4.w > o) || (o4.w == o && e2 + 3 < e);
            }
            for (int e2 = E4; e2 < E; ++e2) {
                const int o2 = s.ov[e2];
                ip += (o2 > o) || (o2 == o && e2 < e);
            }
        }
    }
    if (ve) s.item_at[ip] = e;
    __syncthreads();
    // scans: c and k over experts (index order), o and "has overflow" over
    // the stream positions
    const int ei = ve ? s.item_at[tid] : 0;
    const int oi = ve ? s.ov[ei] : 0;
    const int fi = (ve && oi > 0) ? 1 : 0;
    int v[SCAN_N] = {c, k, oi, fi}, ex[SCAN_N], tot[SCAN_N];
    block_scan<SCAN_N>(v, ex, tot, s.scratch);
    if (ve) {
        s.pc[e] = ex[0];
        s.pk[e] = ex[1];
        s.osi[tid] = ex[2];
        s.nzri[tid] = ex[3];
        s.ose[ei] = ex[2];
        if (fi) s.nzlist[ex[3]] = ei;
    }
    if (tid == 0) {
        s.pc[E] = tot[0];
        s.pk[E] = tot[1];
        s.osi[E] = tot[2];
        s.nzri[E] = tot[3];
    }
    __syncthreads();

    // ranks, one warp, 32 ranks a step: kept rows and deficits; the receiving
    // order (rank order, or by decreasing deficit, ties to the lower index,
    // for rule 2); segments in that order; slots per rank
    if (warp == 0) {
        for (int r0 = 0; r0 < R; r0 += 32) {
            const int r = r0 + lane;
            if (r < R) {
                const int kept = s.pk[(r + 1) * Er] - s.pk[r * Er];
                s.kept[r] = kept;
                s.rload[r] = s.pc[(r + 1) * Er] - s.pc[r * Er];
                s.def[r] = C - kept;
            }
        }
        __syncwarp();
        for (int r0 = 0; r0 < R; r0 += 32) {
            const int r = r0 + lane;
            if (r < R) {
                int rp = r;
                if (p.rule == MOONEP_RULE_LARGEST_FIRST) {
                    const int d = s.def[r];
                    rp = 0;
                    for (int r2 = 0; r2 < R; ++r2) {
                        const int d2 = s.def[r2];
                        rp += (d2 > d) || (d2 == d && r2 < r);
                    }
                }
                s.recv_at[rp] = r;
            }
        }
        __syncwarp();
        int carry = 0;
        for (int i0 = 0; i0 < R; i0 += 32) {
            const int i = i0 + lane;
            const int r = i < R ? s.recv_at[i] : 0;
            const int d = i < R ? s.def[r] : 0;
            const int incl = warp_incl_scan(d, lane);
            const int segs = carry + incl - d;
            carry += __shfl_sync(0xffffffffu, incl, 31);
            if (i < R) {
                s.segs[r] = segs;
                s.sege[r] = segs + d;
                s.sege_at[i] = segs + d;
            }
        }
        __syncwarp();
        int fail_r = -1, fail_n = 0;
        for (int r0 = 0; r0 < R; r0 += 32) {
            const int r = r0 + lane;
            const bool vr = r < R;
            int nsl = 0, fe = -1;
            const int d = vr ? s.def[r] : 0;
            if (vr && d > 0) {
                const int segs = s.segs[r];
                fe = upper_bound(s.osi, E, segs) - 1;
                const int le = upper_bound(s.osi, E, segs + d - 1) - 1;
                nsl = s.nzri[le] - s.nzri[fe] + 1;
            }
            if (vr) {
                s.nsl[r] = nsl;
                s.fe[r] = fe;
            }
            const unsigned over = __ballot_sync(0xffffffffu, vr && nsl > B);
            if (over && fail_r < 0) {
                const int l = __ffs(over) - 1;
                fail_r = r0 + l;
                fail_n = __shfl_sync(0xffffffffu, nsl, l);
            }
        }
        if (lane == 0) {
            misc[0] = fail_r;
            misc[1] = fail_n;
        }
    }
    __syncthreads();
    return misc[0] >= 0 ? MOONEP_STATUS_SLOT_BUDGET : MOONEP_STATUS_OK;
}

// Destination row of the pick at position pos among its expert's picks (t =
// the expert's table entry), or -1 if its stream index is past every segment.
// An overflow pick's receiving position is the first whose segment ends past
// its stream index; the bucket of 2^sh indices holding it gives the positions
// of the bucket's first and last index, between which the answer lies (almost
// always one and the same).
__device__ __forceinline__ int place(const PlanParams& p, const Smem& s, const int4& t, int pos,
                                     int sh) {
    if (pos < t.x) return t.y + pos;  // kept on the home rank
    const int sidx = t.z + pos;       // index in the overflow stream
    const int bi = sidx >> sh;
    if (sidx < 0 || bi >= NBKT) return -1;
    const int bb = s.bkt[bi];
    int lo = bb & 0xffff, hi = bb >> 16;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s.sege_at[mid] <= sidx) lo = mid + 1;
        else hi = mid;
    }
    if (lo >= p.R) return -1;
    return s.rbase[lo] + sidx;
}

// Pack a pick for the walk: its expert (< 2^10) and its position among the
// warp's picks of that expert (< 2^21: a warp holds at most P / (G * 32) + 1
// < 2^31 / (148 * 32) + 1 picks).
__device__ __forceinline__ int pack_pick(int e, int off) { return e | (off << 10); }

// Stable ranking of one row (32 consecutive picks, one per lane; e = -1 for
// none) within a warp: returns the lane's position among the warp's picks of
// its expert so far (the counts in wh from earlier rows, then the row's lower
// lanes holding the same expert) and moves wh[e] past the row.
//   MASK: the lanes holding the warp's candidate expert are found by one
//   ballot; every other lane ORs its bit into its expert's mask word wm[e],
//   and after the warp's barrier one read gives the whole group, so the rank
//   does not depend on the order the atomics were carried out in.  The
//   candidate (warp-uniform) stays while it holds 4 or more lanes of a row,
//   else it becomes lane 0's expert in this row: under a heavy skew it soon
//   settles on the hot expert, whose lanes would otherwise all set bits in
//   one word, one after another.
//   The group's lowest lane advances the count and clears the word (every
//   word is zero between rows).  Top-k routing keeps the lanes sharing a word
//   few: a token's k experts are distinct, so at most ceil(31 / k) + 1 lanes
//   of a row hold one expert.
//   Otherwise match.any finds the group (its cost grows with the number of
//   distinct experts in the row, about ten times the masks' at 30).
template <bool MASK>
__device__ __forceinline__ int rank_row(int* wh, unsigned* wm, int e, int lane, unsigned lt_mask,
                                        int& cand) {
    unsigned m;
    if constexpr (MASK) {
        const unsigned mc = __ballot_sync(0xffffffffu, e >= 0 && e == cand);
        const bool inc = (mc >> lane) & 1u;
        if (e >= 0 && !inc) atomicOr(wm + e, 1u << lane);
        if (__popc(mc) < 4) cand = __shfl_sync(0xffffffffu, e, 0);
        __syncwarp();
        m = inc ? mc : (e >= 0 ? wm[e] : 0u);
    } else {
        m = __match_any_sync(0xffffffffu, e);
    }
    const int run = e >= 0 ? wh[e] : 0;
    __syncwarp();
    const int rank = __popc(m & lt_mask);
    if (e >= 0 && rank == 0) {
        wh[e] = run + __popc(m);
        if constexpr (MASK) wm[e] = 0u;
    }
    __syncwarp();
    return run + rank;
}

template <bool MASK>
__global__ void __launch_bounds__(THREADS, 1) plan_kernel(PlanParams p) {
    extern __shared__ __align__(16) int smem_raw[];
    const bool stash = p.stash != 0;
    Smem s = carve(smem_raw, p.E, p.R, MASK, stash, p.chunk);
    __shared__ int wait_flag;
    __shared__ int max_count;
    __shared__ int misc[4];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, b = blockIdx.x;
    const int E = p.E, WS = warp_stride(E);
    const long long P = p.P;
    // pick indices in 32 bits: P < 2^31, so even a row's last lane (< P + 256)
    // fits without wrapping
    const unsigned clo = (unsigned)(P * b / G), chi = (unsigned)(P * (b + 1) / G);
    const int len = (int)(chi - clo);
    const unsigned wlo = clo + (unsigned)((long long)len * warp / NW);
    const unsigned whi = clo + (unsigned)((long long)len * (warp + 1) / NW);
    int* wh = s.whist + warp * WS;
    unsigned* wm = s.wmask + warp * WS;  // used only when MASK
    const unsigned lt_mask = (1u << lane) - 1u;

    // ---- A: per-warp histograms and positions within the warp ---------------
    for (int i = tid; i < NW * WS; i += THREADS) {
        s.whist[i] = 0;
        if constexpr (MASK) s.wmask[i] = 0u;
    }
    for (int i = tid; i < E; i += THREADS) {
        s.cnt[i] = 0;
        s.bpre[i] = 0;
    }
    if (tid == 0) max_count = 0;
    __syncthreads();
    int bad = 0;
    int cand = -1;  // the warp's candidate expert (ranking by masks)
    unsigned base = wlo;
    // whole batches of UNR rows: every lane has a pick, no bounds checks
    for (; base + 32 * UNR <= whi; base += 32 * UNR) {
        int ev[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) ev[u] = __ldg(p.idx + base + u * 32 + lane);
        const int qo = (int)(base - clo) + lane;
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int e = ev[u];
            const bool ok = (unsigned)e < (unsigned)E;
            bad |= !ok;
            const int off = rank_row<MASK>(wh, wm, ok ? e : -1, lane, lt_mask, cand);
            if (stash) s.stash[qo + u * 32] = ok ? pack_pick(e, off) : -1;
        }
    }
    // the last, partial batch
    for (; base < whi; base += 32 * UNR) {
        int ev[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const unsigned q = base + u * 32 + lane;
            ev[u] = q < whi ? __ldg(p.idx + q) : -1;
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            if (base + u * 32 < whi) {  // warp-uniform: the row has picks
                const unsigned q = base + u * 32 + lane;
                const bool valid = q < whi;
                const int e = ev[u];
                const bool ok = valid && e >= 0 && e < E;
                if (valid && !ok) bad = 1;
                // a lane with no pick, or a bad index, takes no part
                const int off = rank_row<MASK>(wh, wm, ok ? e : -1, lane, lt_mask, cand);
                if (valid && stash) s.stash[q - clo] = ok ? pack_pick(e, off) : -1;
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status + ST_BAD_FLAG, 1);
    __syncthreads();
    // the block's count of each expert, and each warp's offset among the
    // block's picks of it (16 counts loaded at a time before the running sum)
    for (int e = tid; e < E; e += THREADS) {
        int run = 0;
#pragma unroll
        for (int w0 = 0; w0 < NW; w0 += 16) {
            int v[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) v[w] = s.whist[(w0 + w) * WS + e];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                s.whist[(w0 + w) * WS + e] = run;
                run += v[w];
            }
        }
        s.bcnt[e] = run;
        p.hist[(long long)b * E + e] = run;
    }
    __syncthreads();
    unsigned* const barrier = reinterpret_cast<unsigned*>(p.status + ST_BARRIER1);
    grid_arrive(barrier);

    // expert-major slots of the block's picks; this needs only the block's
    // own counts, so it runs while the other blocks finish their histograms
    if (stash) {
        int v1[1] = {tid < E ? s.bcnt[tid] : 0}, ex1[1], t1[1];
        block_scan<1>(v1, ex1, t1, s.scratch);  // E <= THREADS
        if (tid < E) {
            // each warp's first slot of expert tid
            s.bex[tid] = ex1[0];
#pragma unroll
            for (int w0 = 0; w0 < NW; w0 += 16) {
                int v[16];
#pragma unroll
                for (int w = 0; w < 16; ++w) v[w] = s.whist[(w0 + w) * WS + tid];
#pragma unroll
                for (int w = 0; w < 16; ++w) s.whist[(w0 + w) * WS + tid] = v[w] + ex1[0];
            }
        }
        __syncthreads();
        for (unsigned base = wlo; base < whi; base += 32 * UNR) {
            int v[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const unsigned q = base + u * 32 + lane;
                v[u] = q < whi ? s.stash[q - clo] : -1;
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                if (v[u] >= 0) {
                    const int e = v[u] & 1023;
                    const int ql = (int)(base - clo) + u * 32 + lane;
                    s.sorted[wh[e] + (v[u] >> 10)] = e | (ql << 10);
                }
            }
        }
    }

    if (!grid_wait(barrier, (unsigned)(G + p.barrier_extra), p.wait_ns, &wait_flag)) {
        if (tid == 0) atomicMax(p.status + ST_STATUS, MOONEP_STATUS_TIMEOUT);
        return;
    }
    if (tid == 0) misc[2] = __ldcg(p.status + ST_BAD_FLAG);
    __syncthreads();
    if (misc[2]) {
        if (b == 0 && tid == 0) atomicMax(p.status + ST_STATUS, MOONEP_STATUS_BAD_INDEX);
        return;
    }

    // ---- B: totals and this block's offsets from every block's row --------
    if ((E & 3) == 0) {
        const int E4 = E >> 2;
        const int nparts = THREADS / E4;  // >= 4 since E <= THREADS
        const int part = tid / E4, e4 = tid - part * E4;
        if (part < nparts) {
            int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
            for (int b0 = part; b0 < G; b0 += nparts * BUNR) {
                int4 v[BUNR];
#pragma unroll
                for (int u = 0; u < BUNR; ++u) {
                    const int bb = b0 + u * nparts;
                    v[u] = bb < G ? __ldcg(reinterpret_cast<const int4*>(p.hist + (long long)bb * E) + e4)
                                  : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < BUNR; ++u) {
                    tot.x += v[u].x; tot.y += v[u].y; tot.z += v[u].z; tot.w += v[u].w;
                    if (b0 + u * nparts < b) {
                        pre.x += v[u].x; pre.y += v[u].y; pre.z += v[u].z; pre.w += v[u].w;
                    }
                }
            }
            const int e = 4 * e4;
            atomicAdd(s.cnt + e, tot.x); atomicAdd(s.cnt + e + 1, tot.y);
            atomicAdd(s.cnt + e + 2, tot.z); atomicAdd(s.cnt + e + 3, tot.w);
            atomicAdd(s.bpre + e, pre.x); atomicAdd(s.bpre + e + 1, pre.y);
            atomicAdd(s.bpre + e + 2, pre.z); atomicAdd(s.bpre + e + 3, pre.w);
        }
    } else {
        const int nparts = THREADS / E;  // >= 1 since E <= THREADS
        const int part = tid / E, e = tid - part * E;
        if (part < nparts) {
            int tot = 0, pre = 0;
            for (int b0 = part; b0 < G; b0 += nparts * BUNR) {
                int v[BUNR];
#pragma unroll
                for (int u = 0; u < BUNR; ++u) {
                    const int bb = b0 + u * nparts;
                    v[u] = bb < G ? __ldcg(p.hist + (long long)bb * E + e) : 0;
                }
#pragma unroll
                for (int u = 0; u < BUNR; ++u) {
                    tot += v[u];
                    if (b0 + u * nparts < b) pre += v[u];
                }
            }
            atomicAdd(s.cnt + e, tot);
            atomicAdd(s.bpre + e, pre);
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += THREADS) atomicMax(&max_count, s.cnt[e]);
    __syncthreads();

    // ---- C: balance step (every block), outputs, placement ---------------
    const int st = balance(p, s, misc);

    if (b == 0) {
        for (int e = tid; e < E; e += THREADS) p.expert_count[e] = s.cnt[e];
        for (int r = tid; r < p.R; r += THREADS) p.rank_load[r] = s.rload[r];
        if (tid == 0) {
            const int mx = max_count;
            const double tbar = __ddiv_rn((double)P, (double)E);
            p.maxvio[0] = __dsub_rn(__ddiv_rn((double)mx, tbar), 1.0);
            p.status[ST_MAX_COUNT] = mx;
            p.status[ST_FAIL_RANK] = misc[0];
            p.status[ST_FAIL_SLOTS] = misc[1];
            atomicMax(p.status + ST_STATUS, st);
        }
    }
    if (st != MOONEP_STATUS_OK) return;

    const int R = p.R, B = p.B, Er = p.Er;
    for (int r = b; r < R; r += G) {
        const int kept = s.kept[r], d = s.def[r], segs = s.segs[r], sege = s.sege[r];
        const int nsl = s.nsl[r], fe = s.fe[r];
        const int nz0 = fe >= 0 ? s.nzri[fe] : 0;
        const int rbase = s.pk[r * Er];
        for (int g = tid; g < E + B; g += THREADS) {
            int v;
            if (g < E) {
                const int h = g / Er;
                v = h < r ? 0 : (h > r ? kept : s.pk[g] - rbase + s.kk[g]);
            } else {
                const int j = g - E;
                if (j < nsl) {
                    const int e = s.nzlist[nz0 + j];
                    const int end = min(s.ose[e] + s.ov[e], sege);
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

    // the placement tables; on the expert-major path an entry is shifted by
    // the offset sft from a slot of the block to the pick's position among
    // all picks of its expert, so that the slot itself indexes the entry
    for (int e = tid; e < E; e += THREADS) {
        const int first = (e / Er) * Er;
        const int k = s.kk[e];
        const int sft = stash ? s.bpre[e] - s.bex[e] : 0;
        s.tab[e] = make_int4(k - sft, (e / Er) * p.C + (s.pk[e] - s.pk[first]) + sft,
                             s.ose[e] - k + sft, s.cnt[e] - sft);
    }
    if (!stash) {
        // each warp's running offsets: the block's offset plus the warp's
        // offset in the block
        for (int i = tid; i < NW * E; i += THREADS) {
            const int w = i / E, e = i - w * E;
            s.whist[w * WS + e] += s.bpre[e];
        }
    }
    for (int i = tid; i < R; i += THREADS) {
        const int rho = s.recv_at[i];
        s.rbase[i] = rho * p.C + s.kept[rho] - s.segs[rho];
    }
    // the bucket width: the smallest power of two that covers the overflow
    // stream (as long as the deficits' sum) in NBKT buckets; the last NBKT
    // threads fill the buckets (the first E fill the tables above)
    int sh = 0;
    while (((long long)NBKT << sh) < (long long)s.osi[E]) ++sh;
    if (tid >= THREADS - NBKT) {
        const int i = tid - (THREADS - NBKT);
        const int first = (int)((long long)i << sh);
        const int last = (int)(((long long)(i + 1) << sh) - 1);
        s.bkt[i] = upper_bound(s.sege_at, R, first) | (upper_bound(s.sege_at, R, last) << 16);
    }
    __syncthreads();

    int internal = 0;
    if (stash) {
        // the walk in expert-major order: consecutive threads place
        // consecutive picks of one expert, whose rows are consecutive too
        // (within a receiving segment), so the inverse map is written in runs;
        // each pick's row goes to the stash, indexed by the pick
        constexpr int WU = 4;  // slots per thread in flight
        for (int i0 = tid; i0 < len; i0 += WU * THREADS) {
            int v[WU];
#pragma unroll
            for (int u = 0; u < WU; ++u) {
                const int i = i0 + u * THREADS;
                v[u] = i < len ? s.sorted[i] : -1;
            }
#pragma unroll
            for (int u = 0; u < WU; ++u) {
                if (v[u] >= 0) {
                    const int e = v[u] & 1023, ql = v[u] >> 10;
                    const int pos = i0 + u * THREADS;  // the slot (entries are shifted)
                    const int4 t = s.tab[e];
                    const int dst = place(p, s, t, pos, sh);
                    if (dst >= 0 && dst < p.P && pos < t.w) {
                        p.src_of_row[dst] = (int)(clo + ql);
                        s.stash[ql] = dst;
                    } else {
                        s.stash[ql] = -1;  // never expected: report, do not write
                        internal = 1;
                    }
                }
            }
        }
        __syncthreads();
        for (int i0 = tid; i0 < len; i0 += WU * THREADS) {
            int d[WU];
#pragma unroll
            for (int u = 0; u < WU; ++u) {
                const int i = i0 + u * THREADS;
                d[u] = i < len ? s.stash[i] : -1;
            }
#pragma unroll
            for (int u = 0; u < WU; ++u)
                if (d[u] >= 0) p.dst_row[clo + i0 + u * THREADS] = d[u];
        }
    } else {
        // picks not kept: read them again and rank each row against the
        // warp's running offsets.  Phase A checked every index; one that has
        // changed since is reported, not placed.
        for (unsigned base = wlo; base < whi; base += 32 * UNR) {
            const int nu = (int)min((unsigned)UNR, (whi - base + 31) / 32);  // warp-uniform
            int ev[UNR], pos[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const unsigned q = base + u * 32 + lane;
                const int v = q < whi ? __ldg(p.idx + q) : -1;
                ev[u] = v < E ? v : -1;
                if (q < whi && (v < 0 || v >= E)) internal = 1;
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u)
                if (u < nu) pos[u] = rank_row<MASK>(wh, wm, ev[u], lane, lt_mask, cand);
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int e = ev[u];
                if (u < nu && e >= 0) {
                    const unsigned q = base + u * 32 + lane;
                    const int4 t = s.tab[e];
                    const int dst = place(p, s, t, pos[u], sh);
                    if (dst >= 0 && dst < p.P && pos[u] < t.w) {
                        p.dst_row[q] = dst;
                        p.src_of_row[dst] = (int)q;
                    } else {
                        internal = 1;  // never expected: report, do not write
                    }
                }
            }
        }
    }
    if (internal) atomicMax(p.status + ST_STATUS, MOONEP_STATUS_INTERNAL);
}

struct DevInfo {
    int sms = 0;
    int max_smem_optin = 0;
    size_t smem_set[2] = {0, 0};  // largest dynamic smem each form has been configured for
};

DevInfo& dev_info() {
    static thread_local int cached_dev = -1;
    static thread_local DevInfo info;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != cached_dev) {
        info = DevInfo();
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
    DevInfo& info = dev_info();
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
    p.hist = static_cast<int32_t*>(a.plan.workspace);
    p.wait_ns = a.wait_ns;
    p.barrier_extra = a.barrier_extra;

    // Shared memory, the first layout that fits: ranking by mask words (else
    // by match.any) and keeping the block's picks (the stash and the
    // expert-major order: no second read and ranking of the picks, and the
    // walk writes its rows in runs), then either alone, then neither.
    const size_t limit = (size_t)info.max_smem_optin - 1024;
    const long long chunk = ((long long)p.P + G - 1) / G;
    bool mask = false, keep = false;
    const bool forms[4][2] = {{true, true}, {false, true}, {true, false}, {false, false}};
    for (int f = 0; f < 4; ++f) {
        mask = forms[f][0];
        keep = forms[f][1];
        if (smem_ints(a.E, a.R, mask, keep, chunk) * 4 <= limit) break;
    }
    p.chunk = (int)chunk;
    p.stash = keep;
    const size_t smem = smem_ints(a.E, a.R, mask, keep, chunk) * 4;
    if (smem > (size_t)info.max_smem_optin) {
        *why = "planner shared memory exceeds the device limit (E or R too large)";
        return cudaErrorInvalidValue;
    }
    const void* kern = mask ? (const void*)plan_kernel<true> : (const void*)plan_kernel<false>;
    cudaError_t err;
    if (smem > info.smem_set[mask]) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        int per_sm = 0;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem);
        if (err != cudaSuccess) return err;
        if (per_sm < 1) {
            *why = "planner block does not fit on an SM";
            return cudaErrorInvalidConfiguration;
        }
        info.smem_set[mask] = smem;
    }
    // status block: status, fail info, the wait counter and the bad-index flag
    err = cudaMemsetAsync(a.plan.status, 0, MOONEP_STATUS_WORDS * sizeof(int32_t), stream);
    if (err != cudaSuccess) return err;
    void* args[] = {&p};
    return cudaLaunchCooperativeKernel(kern, dim3(G), dim3(THREADS), args, smem, stream);
}

}  // namespace moonep
