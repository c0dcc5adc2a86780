// expert_gemm.cu -- the grouped expert GEMM that consumes a plan: for every
// rank r and every group g of its [E+B] groups, the rows [cu[r][g-1],
// cu[r][g]) of rank r's dispatched block are multiplied by row g of rank r's
// [E+B, H, H'] weight view.
//
// This is the consumer the pages put after dispatch: the framework's grouped
// GEMM reads the contiguous [E+B, H, H'] weight tensor and selects the active
// rows through cu_seqlens[E+B] ("Moonshot AI Open-Sources MoonEP ..." on
// ainovat.com, the framework-contract paragraph; "MoonEP" on moses-y.github.io,
// "What This Does").  The pages give no kernel for it; this one is written
// for sm_100a:
//
//  - one persistent CTA per SM: warp 0 issues TMA loads, one thread of warp 1
//    issues tcgen05.mma, 8 warps drain the accumulator (two per TMEM lane
//    quarter, each taking half of the columns): warps 2-9 for bf16 rows (320
//    threads), warps 2-5 and 15-18 for fp8 rows (608 threads);
//  - bf16 payload: tile 256 rows x 256 columns when H' % 256 == 0 (else 128
//    x BN, BN = 256 or 128), k-block 64: A = two 128 x 64 bf16 blocks of the
//    dispatched rows (K-major), B = 64 x 256 of the weight row (H'
//    contiguous, MN-major), both 128-byte swizzled in shared memory; each B
//    block feeds one MMA per 128-row half, so B crosses into shared memory
//    once per 256 rows (the shared-memory traffic per MMA, TMA writes plus
//    tensor-core reads, is what bounds a one-CTA tile);
//  - fp8 payload: A never exists in bf16 outside the SM.  Warp 6 streams the
//    e4m3 tiles into a ring of 4 slots, 8 converter warps widen them
//    (a = bf16(float(q) * scale)) straight into tensor memory with
//    tcgen05.st, and the MMA reads A from there; shared memory then holds
//    only B.  A tile is 128 x 384: each widened A block feeds two MMAs of
//    N = 192, so A is widened once per 384 output columns (4 times per row
//    block at H' = 1536, not 8).  One 384-column accumulator and 3 A stages
//    (32 columns each) fit the 512 columns; the last n-tile may be partial;
//  - the fp32 accumulator lives in tensor memory; with 128-row tiles there
//    are two buffers, so the epilogue of one tile overlaps the main loop of
//    the next.  The 256 x 256 tile fills the 512 columns with one buffer of
//    two 128-row halves, which the epilogue frees one at a time: the next
//    tile's first-half MMAs start once the first half is drained, while its
//    second-half MMAs wait (holding their stages, at most all of them) for
//    the second.  The fp8 tile's one buffer is not overlapped;
//  - the epilogue reads 32 lanes x 32 columns per tcgen05.ld, rounds once to
//    bf16 (round-to-nearest-even) and stores only the rows of the group;
//    each warp passes its 32 rows x 64 B through shared memory, so that one
//    store covers 64 contiguous bytes of 8 rows.
//
// The tile list is built in each CTA from the plan: only the groups a plan
// can fill are visited (rank r's E/R home experts and its B slots; every
// other group of rank r is empty by construction of the plan), their m-tile
// counts are scanned in shared memory and a tile index is mapped back to
// (rank, group, m-tile, n-tile) by binary search.  Tiles go to CTAs
// round-robin in (m-tile, n-tile) order, so the CTAs running at one time read
// the same A rows and the same expert's weights from L2.
//
// Every wait is bounded by the library's wait limit (globaltimer).  A wait
// that runs out raises a CTA-wide abort flag; each role then stops, the TMA
// warps wait (bounded) for the loads they still have in flight, the MMA thread
// waits (bounded) for its issued MMAs to finish, TMEM is released, and the
// plan's status becomes MOONEP_STATUS_TIMEOUT.
#include <cuda.h>

#include <mutex>

#include "internal.cuh"

namespace moonep {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;   // 16 KiB of bf16 A per stage
constexpr int A8_BYTES = BM * BK;      // 8 KiB of e4m3 A per k-block (fp8 payload)
// fp8 payload: one more warp loads the e4m3 tiles and CW warps widen them
// 8 epilogue warps: two per TMEM lane quarter, each taking half of a tile's
// columns.  bf16 payload: warps 2-9; fp8 payload: warps 2-5 and, after the
// e4m3 producer (warp 6) and the CW converter warps, the last 4
constexpr int EPI_WARPS = 8;
template <bool FP8A, int CW>
__host__ __device__ constexpr int threads_for() { return FP8A ? (7 + CW + 4) * 32 : (2 + EPI_WARPS) * 32; }
// dynamic shared memory a CTA may ask for: the 227 KiB opt-in limit less
// room for the kernel's static shared variables
constexpr int SMEM_LIMIT = 227 * 1024 - 256;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* b, int count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
        "selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return done != 0;
}

// Whether the phase of `parity` has completed, without suspending the thread.
__device__ __forceinline__ bool mbar_peek(uint64_t* b, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; "
        "selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase of `parity` to complete.  Gives up (returns false) when
// another role has raised the abort flag or after `limit` ns, raising it.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, unsigned long long limit,
                                          volatile int* abort) {
    const unsigned long long t0 = globaltimer_ns();
    for (int it = 1;; ++it) {
        if (mbar_test(b, parity)) return true;
        if ((it & 63) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit) {
                *abort = 1;
                return false;
            }
        }
    }
}

// The same wait without the abort check: used to drain in-flight work.
__device__ __forceinline__ bool mbar_drain(uint64_t* b, uint32_t parity, unsigned long long limit) {
    const unsigned long long t0 = globaltimer_ns();
    for (int it = 1;; ++it) {
        if (mbar_test(b, parity)) return true;
        if ((it & 63) == 0 && globaltimer_ns() - t0 > limit) return false;
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// Shared-memory matrix descriptor for tcgen05.mma: start, leading and stride
// byte offsets (>> 4), descriptor version 1 (bits 46-47) and the 128-byte
// swizzle mode (2 in bits 61-63).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((addr >> 4) & 0x3fff);
    d |= (uint64_t)((lbo >> 4) & 0x3fff) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fff) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// The same MMA with A read from tensor memory: `tmem_a` addresses lane 0 of
// the 8 columns that hold the 128 x 16 bf16 A block (row i in lane i, two
// elements per 32-bit column, the lower k in the low half).
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Store NW 32-bit words per lane into NW consecutive tensor-memory columns of
// the warp's 32 lanes, and wait until the stores are done.
template <int NW>
__device__ __forceinline__ void tmem_store(uint32_t taddr, const uint32_t* v) {
    static_assert(NW == 8 || NW == 16 || NW == 32, "8, 16 or 32 columns");
    if constexpr (NW == 8) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                         taddr),
                     "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                     "r"(v[7])
                     : "memory");
    } else if constexpr (NW == 16) {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
            "%13,%14,%15,%16};" ::"r"(taddr),
            "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
            "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
            "r"(v[15])
            : "memory");
    } else {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
            "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
                taddr),
            "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
            "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
            "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
            "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
            "r"(v[29]), "r"(v[30]), "r"(v[31])
            : "memory");
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    unsigned short a, b;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(a) : "f"(lo));
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(b) : "f"(hi));
    return (uint32_t)a | ((uint32_t)b << 16);
}

// Two e4m3 codes (low byte first) -> bf16x2 of float(code) * scale: the
// codes widen exactly to f16 and then to f32, one binary32 product each, one
// round to nearest even to bf16.
__device__ __forceinline__ uint32_t widen_e4m3x2(uint32_t two_codes, float scale) {
    uint32_t h2, r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)two_codes));
    float lo, hi;
    asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"((unsigned short)(h2 & 0xffffu)));
    asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"((unsigned short)(h2 >> 16)));
    // both products at once (two binary32 multiplies, round to nearest even)
    asm("{ .reg .b64 v, s2, pr; .reg .f32 plo, phi;\n\t"
        "mov.b64 v, {%1, %2};\n\t"
        "mov.b64 s2, {%3, %3};\n\t"
        "mul.rn.f32x2 pr, v, s2;\n\t"
        "mov.b64 {plo, phi}, pr;\n\t"
        "cvt.rn.bf16x2.f32 %0, phi, plo; }"
        : "=r"(r)
        : "f"(lo), "f"(hi), "f"(scale));
    return r;
}

struct GemmArgs {
    int R, C, E, B, Er, H, Hp;
    const int32_t* cu;  // [R][E+B] inclusive row ends
    int32_t* status;
    uint16_t* y;  // [R*C, Hp] bf16
    const float* scale;  // fp8 payload: [R*C, H/128] per-block scales
    unsigned long long wait_ns;
    int debug_stall;  // epilogue waits on a barrier nothing completes
};

template <int BN, int STAGES, bool FP8A, int CW, int A8_SLOTS, int NSUB, int MT, bool STG>
__global__ void __launch_bounds__(threads_for<FP8A, CW>(), 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW, GemmArgs p) {
    constexpr int THREADS = threads_for<FP8A, CW>();
    // a tile is BM rows x TN = NSUB * BN columns: NSUB MMAs of N = BN per
    // k-step share one A block (fp8 payload: A is widened once per TN columns)
    constexpr int TN = NSUB * BN;
    constexpr int B_BYTES = BK * TN * 2;
    // bf16 payload: a tile may also be MT m-tiles high (TM = MT * BM rows):
    // every B block loaded then feeds MT MMAs, one per 128-row half, so the
    // B operand crosses into shared memory once per TM rows
    constexpr int TM = MT * BM;
    static_assert(MT == 1 || !FP8A, "fp8 payload: one m-tile per tile");
    // a stage of the MMA ring: bf16 A (SW128, K-major) | B.  fp8 payload: A
    // lives in tensor memory, so a stage holds only B, and the e4m3 tiles
    // land in their own ring of A8_SLOTS after the stages.
    constexpr int STAGE_A = FP8A ? 0 : MT * A_BYTES;
    constexpr int STAGE_BYTES = STAGE_A + B_BYTES;
    constexpr int A8S = FP8A ? A8_SLOTS : 0;
    // NACC accumulators of TN columns (two, so that the epilogue of one tile
    // overlaps the next tile's main loop, when they fit); fp8 payload: then A
    // stage s at columns ACOL + 32 s (128 rows x 64 bf16, two per column)
    constexpr int NACC = (FP8A ? 2 * TN + 32 * STAGES : 2 * MT * TN) <= 512 ? 2 : 1;
    constexpr int ACOL = NACC * TN;
    constexpr int ACC_COLS = MT * TN;  // one accumulator: the MT halves side by side
    // one accumulator of two halves: the epilogue frees each half on its own
    // (tempty[h]), so the next tile's first half starts while the second
    // drains.  (Splitting the fp8 tile's two column sub-tiles the same way was
    // slower: the deferred MMAs hold the widened A stages, and the converter
    // warps wait for them.)
    constexpr bool SPLIT = !FP8A && MT == 2 && NACC == 1;
    constexpr int TMEM_COLS = FP8A ? 512 : NACC * ACC_COLS;
    static_assert(NACC * ACC_COLS + (FP8A ? 32 * STAGES : 0) <= 512 && ACC_COLS <= 512,
                  "accumulators (and fp8 A stages) in the 512 tensor-memory columns");
    static_assert(!FP8A || (CW % 4 == 0 && CW <= 16), "whole converter warps per lane quarter");
    // k-block of A: 128 rows x 128 B; one k-step (16 elements) = 32 B along a row.
    // k-block of B: BN/64 column chunks of 64 k-rows x 128 B (8 KiB each); one
    // k-step = 16 k-rows = 2 KiB; the next 64-column chunk is 8 KiB further.
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* a8ring = smem + STAGES * STAGE_BYTES;  // [A8S][A8_BYTES]
    uint64_t* full = (uint64_t*)(a8ring + A8S * A8_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* conv = empty + STAGES;    // fp8 payload: the stage's A is widened
    uint64_t* a8full = conv + STAGES;   // fp8 payload: e4m3 tile landed [A8_SLOTS]
    uint64_t* a8empty = a8full + A8_SLOTS;  // fp8 payload: e4m3 tile read [A8_SLOTS]
    uint64_t* tfull = a8empty + A8_SLOTS;
    uint64_t* tempty = tfull + 2;  // [NACC] (two slots kept either way)
    uint64_t* drain = tempty + 2;
    uint64_t* never = drain + 1;
    uint32_t* tmem_slot = (uint32_t*)(never + 1);
    int* wsum = (int*)(tmem_slot + 2);  // [THREADS / 32]
    int* pre = wsum + 32;               // [npairs + 1] m-tile prefix
    static_assert(THREADS / 32 <= 32, "one per-warp sum slot per warp");
    __shared__ volatile int abort_flag;
    __shared__ int plan_status;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // one read per CTA: another CTA of this launch may raise TIMEOUT meanwhile
    if (tid == 0) plan_status = load_status(p.status);
    __syncthreads();
    if (plan_status != MOONEP_STATUS_OK) return;

    const int G = p.E + p.B;      // groups per rank
    const int per = p.Er + p.B;   // groups a plan can fill per rank
    const int npairs = p.R * per;
    // the epilogue's row staging, [epilogue warps][32 rows][80 B]
    uint8_t* estage = (uint8_t*)(((uintptr_t)(pre + npairs + 1) + 15) & ~(uintptr_t)15);
    const int ntn = (p.Hp + TN - 1) / TN;  // the last n-tile may be partial
    const int kblocks = p.H / BK;

    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&conv[s], CW);
        }
        for (int j = 0; j < A8_SLOTS; ++j) {
            mbar_init(&a8full[j], 1);
            mbar_init(&a8empty[j], CW);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], EPI_WARPS);
        }
        mbar_init(drain, 1);
        mbar_init(never, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // (rank, group) of pair i: home groups of the rank first, then its slots
    auto pair_rg = [&](int i, int& r, int& g) {
        r = i / per;
        const int j = i - r * per;
        g = j < p.Er ? r * p.Er + j : p.E + (j - p.Er);
    };
    // m-tile count of every pair, then an exclusive scan over the block
    const int chunk = (npairs + THREADS - 1) / THREADS;
    const int lo_i = min(npairs, tid * chunk), hi_i = min(npairs, lo_i + chunk);
    int sum = 0;
    for (int i = lo_i; i < hi_i; ++i) {
        int r, g;
        pair_rg(i, r, g);
        const int hi = __ldg(p.cu + r * G + g);
        const int lo = g ? __ldg(p.cu + r * G + g - 1) : 0;
        const int c = (hi - lo + TM - 1) / TM;
        pre[i] = c;
        sum += c;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    if (warp == 1) {  // TMEM: both accumulators (one warp allocates)
        asm volatile(
            "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                smem_u32(tmem_slot)),
            "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    __syncthreads();
    int run = incl - sum;
    for (int w = 0; w < warp; ++w) run += wsum[w];
    for (int i = lo_i; i < hi_i; ++i) {
        const int c = pre[i];
        pre[i] = run;
        run += c;
    }
    if (tid == THREADS - 1) pre[npairs] = run;
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const uint32_t tmem = *tmem_slot;
    const int total = pre[npairs] * ntn;

    // tile -> pair, m-tile within the pair's group, n-tile
    auto locate = [&](int tile, int& pair, int& mt, int& nt) {
        const int mtile = tile / ntn;
        nt = tile - mtile * ntn;
        int lo = 0, hi = npairs;  // pre[lo] <= mtile < pre[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= mtile)
                lo = mid;
            else
                hi = mid;
        }
        pair = lo;
        mt = mtile - pre[lo];
    };

    if (warp == 0) {
        if (lane == 0) {  // TMA producer
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
                int pair, mt, nt, r, g;
                locate(tile, pair, mt, nt);
                pair_rg(pair, r, g);
                const int row0 = r * p.C + (g ? __ldg(p.cu + r * G + g - 1) : 0) + mt * TM;
                const int wrow0 = (r * G + g) * p.H;
                // 64-column boxes of B inside H' (all of them unless the
                // last n-tile is partial; the rest of the stage is not read
                // into any stored column)
                const int nbox = min(TN / 64, (p.Hp - nt * TN) / 64);
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1, p.wait_ns, &abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a = smem + s * STAGE_BYTES;
                    uint8_t* b = a + STAGE_A;
                    if constexpr (FP8A) {  // A comes from the e4m3 producer and the converters
                        mbar_expect_tx(&full[s], nbox * 8192);
                    } else {
                        mbar_expect_tx(&full[s], MT * A_BYTES + nbox * 8192);
#pragma unroll
                        for (int h = 0; h < MT; ++h)  // rows past the buffer are zero-filled
                            tma_load_2d(a + h * A_BYTES, &tmX, &full[s], kb * BK, row0 + h * BM);
                    }
#pragma unroll
                    for (int j = 0; j < TN / 64; ++j)
                        if (j < nbox)
                            tma_load_2d(b + j * 8192, &tmW, &full[s], nt * TN + 64 * j,
                                        wrow0 + kb * BK);
                    ++issued;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) break;
            }
            if (abort_flag) {
                // load n went to stage n % STAGES in phase (n / STAGES) & 1;
                // wait for the last STAGES of them to land before leaving
                for (long long n = issued > STAGES ? issued - STAGES : 0; n < issued; ++n)
                    mbar_drain(&full[n % STAGES], (uint32_t)((n / STAGES) & 1), p.wait_ns);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // MMA issuer
            // kind::f16 instruction descriptor: D f32 (bit 4), A bf16 (bit 7),
            // B bf16 (bit 10), A K-major (bit 15 = 0), B MN-major (bit 16),
            // N >> 3 at bit 17, M >> 4 at bit 24
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                   ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            bool any = false;
            // the MMAs of stage st (k-block kb) into the halves [h0, h1)
            auto issue = [&](int st, int kb, int h0, int h1, int nsub, uint32_t d) {
                const uint32_t a = smem_u32(smem + st * STAGE_BYTES);
                const uint32_t b = a + STAGE_A;
#pragma unroll
                for (int ks = 0; ks < BK / 16; ++ks) {
#pragma unroll
                    for (int h = 0; h < MT; ++h) {
                        if (h < h0) continue;
                        if (h >= h1) break;
#pragma unroll
                        for (int sub = 0; sub < NSUB; ++sub) {
                            if (sub >= nsub) break;
                            // half h, sub-tile sub: columns h*TN + sub*BN.. of the
                            // accumulator, A rows of half h, B chunks sub*BN/64..
                            const uint32_t bsub = b + sub * (BN / 64) * 8192;
                            if constexpr (FP8A)
                                mma_bf16_tmem_a(d + sub * BN, tmem + ACOL + st * 32 + ks * 8,
                                                sdesc(bsub + ks * 2048, 8192, 1024), idesc,
                                                (kb | ks) ? 1u : 0u);
                            else
                                mma_bf16(d + h * TN + sub * BN,
                                         sdesc(a + h * A_BYTES + ks * 32, 16, 1024),
                                         sdesc(bsub + ks * 2048, 8192, 1024), idesc,
                                         (kb | ks) ? 1u : 0u);
                        }
                    }
                }
            };
            for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
                // SPLIT: only half 0 needs to be drained to start the tile
                if (!mbar_wait(&tempty[SPLIT ? 0 : acc], acc_ph ^ 1, p.wait_ns, &abort_flag)) break;
                asm volatile("tcgen05.fence::after_thread_sync;");
                const uint32_t d = tmem + acc * ACC_COLS;
                // sub-tiles wholly past H' (a partial last n-tile), and halves
                // wholly past the group's rows, are skipped
                int nt_, pair_, mt_, r_, g_;
                locate(tile, pair_, mt_, nt_);
                pair_rg(pair_, r_, g_);
                const int nsub = min(NSUB, (p.Hp - nt_ * TN + BN - 1) / BN);
                const int grows = __ldg(p.cu + r_ * G + g_) - (g_ ? __ldg(p.cu + r_ * G + g_ - 1) : 0);
                const int nhalf = min(MT, (grows - mt_ * TM + BM - 1) / BM);
                bool ok = true;
                // SPLIT: while the epilogue still drains half 1 of the last
                // tile, this tile's half-1 MMAs wait and their stages stay
                // held (at most all STAGES of them); then they are issued in
                // k order and each stage is released
                bool h1_free = !SPLIT;
                int npend = 0, pend_s = 0, pend_kb = 0;
                auto flush = [&]() {
                    int ss = pend_s;
                    for (int j = 0; j < npend; ++j) {
                        issue(ss, pend_kb + j, 1, 2, nsub, d);
                        mma_commit(&empty[ss]);
                        if (++ss == STAGES) ss = 0;
                    }
                    npend = 0;
                };
                for (int kb = 0; kb < kblocks; ++kb) {
                    // the TMA loads landed; fp8: and the converter warps have
                    // widened A into the stage
                    if (!mbar_wait(&full[s], ph, p.wait_ns, &abort_flag) ||
                        (FP8A && !mbar_wait(&conv[s], ph, p.wait_ns, &abort_flag))) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;");
                    const bool defer = SPLIT && !h1_free && nhalf > 1;
                    issue(s, kb, 0, defer ? 1 : nhalf, nsub, d);
                    any = true;
                    if (defer) {
                        if (npend == 0) {
                            pend_s = s;
                            pend_kb = kb;
                        }
                        ++npend;
                        bool freed = mbar_peek(&tempty[1], acc_ph ^ 1);
                        if (!freed && npend == STAGES) {  // out of stages: wait for the drain
                            if (!mbar_wait(&tempty[1], acc_ph ^ 1, p.wait_ns, &abort_flag)) {
                                ok = false;
                                break;
                            }
                            freed = true;
                        }
                        if (freed) {
                            h1_free = true;
                            asm volatile("tcgen05.fence::after_thread_sync;");
                            flush();
                        }
                    } else {
                        mma_commit(&empty[s]);
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) break;
                if (!h1_free) {  // SPLIT: take the drain's phase; issue what still waits
                    if (!mbar_wait(&tempty[1], acc_ph ^ 1, p.wait_ns, &abort_flag)) break;
                    asm volatile("tcgen05.fence::after_thread_sync;");
                    flush();
                }
                mma_commit(&tfull[acc]);
                if (++acc == NACC) {
                    acc = 0;
                    acc_ph ^= 1;
                }
            }
            if (abort_flag && any) {  // let every issued MMA finish before TMEM goes
                mma_commit(drain);
                mbar_drain(drain, 0, p.wait_ns);
            }
        }
    } else if ((warp >= 2 && warp < (FP8A ? 6 : 2 + EPI_WARPS)) || (FP8A && warp >= 7 + CW)) {
        // epilogue: warp w reads TMEM lanes 32*(w % 4) .. +31, and half of the
        // tile's columns
        const int q = warp & 3;
        const int eord = (FP8A && warp >= 7 + CW) ? 4 + (warp - 7 - CW) : warp - 2;  // 0..7
        const int cpart = eord >> 2;
        const int c_lo = cpart * (TN / 2), c_hi = c_lo + TN / 2;
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
            int pair, mt, nt, r, g;
            locate(tile, pair, mt, nt);
            pair_rg(pair, r, g);
            const int glo = g ? __ldg(p.cu + r * G + g - 1) : 0;
            const int ghi = __ldg(p.cu + r * G + g);
            uint64_t* bar = p.debug_stall ? never : &tfull[acc];
            if (!mbar_wait(bar, acc_ph, p.wait_ns, &abort_flag)) break;
            asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll 1
            for (int h = 0; h < MT; ++h) {
                if (mt * TM + h * BM >= ghi - glo) {  // half past the group (warp-uniform)
                    if constexpr (SPLIT) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty[h]);
                        continue;
                    } else {
                        break;
                    }
                }
                uint8_t* wst = estage + eord * (32 * 80);  // this warp's row staging (STG)
                const int row_in = mt * TM + h * BM + q * 32 + lane;  // this lane's row (!STG)
                const uint32_t tbase = tmem + acc * ACC_COLS + h * TN + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
                for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
                    if (nt * TN + c0 >= p.Hp) break;  // partial last n-tile (warp-uniform)
                    uint32_t v[32];
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,"
                        "%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,"
                        "%31}, [%32];"
                        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                          "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                          "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
                          "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                          "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]),
                          "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                        : "r"(tbase + c0));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    if constexpr (!STG) {  // each lane stores its own row's 64 B
                        if (glo + row_in < ghi) {
                            uint16_t* yrow =
                                p.y + (size_t)(r * p.C + glo + row_in) * p.Hp + nt * TN + c0;
#pragma unroll
                            for (int j = 0; j < 32; j += 8) {
                                uint4 o;
                                o.x = pack_bf16x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
                                o.y = pack_bf16x2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
                                o.z = pack_bf16x2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5]));
                                o.w = pack_bf16x2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7]));
                                *reinterpret_cast<uint4*>(yrow + j) = o;
                            }
                        }
                    } else {
                        // the warp's 32 rows x 64 B go through shared memory (80-byte
                        // row pitch: no bank conflicts either way), so that each
                        // store writes 64 contiguous bytes of 8 rows instead of 16
                        // bytes of 32 rows; only rows of the group are stored
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            uint4 o;
                            o.x = pack_bf16x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
                            o.y = pack_bf16x2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
                            o.z = pack_bf16x2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5]));
                            o.w = pack_bf16x2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7]));
                            *reinterpret_cast<uint4*>(wst + lane * 80 + (j / 8) * 16) = o;
                        }
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int rr = 8 * i + (lane >> 2), k = lane & 3;  // row, 16-B piece
                            const uint4 o = *reinterpret_cast<const uint4*>(wst + rr * 80 + k * 16);
                            const int ri = mt * TM + h * BM + q * 32 + rr;
                            if (glo + ri < ghi)
                                *reinterpret_cast<uint4*>(p.y + (size_t)(r * p.C + glo + ri) * p.Hp +
                                                          nt * TN + c0 + k * 8) = o;
                        }
                        __syncwarp();
                    }
                }
                if constexpr (SPLIT) {  // this half is drained: the next tile may use it
                    asm volatile("tcgen05.fence::before_thread_sync;");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[h]);
                }
            }
            if constexpr (!SPLIT) {
                asm volatile("tcgen05.fence::before_thread_sync;");
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
            }
            if (++acc == NACC) {
                acc = 0;
                acc_ph ^= 1;
            }
        }
    } else if constexpr (FP8A) {
        if (warp == 6) {
            if (lane == 0) {  // e4m3 producer: runs up to A8S k-blocks ahead of the converters
                long long issued = 0;
                for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
                    int pair, mt, nt, r, g;
                    locate(tile, pair, mt, nt);
                    pair_rg(pair, r, g);
                    const int row0 = r * p.C + (g ? __ldg(p.cu + r * G + g - 1) : 0) + mt * TM;
                    bool ok = true;
                    for (int kb = 0; kb < kblocks; ++kb) {
                        const int j8 = (int)(issued % A8S);
                        const uint32_t p8 = (uint32_t)((issued / A8S) & 1);
                        if (!mbar_wait(&a8empty[j8], p8 ^ 1, p.wait_ns, &abort_flag)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(&a8full[j8], A8_BYTES);
                        tma_load_2d(a8ring + j8 * A8_BYTES, &tmX, &a8full[j8], kb * BK, row0);
                        ++issued;
                    }
                    if (!ok) break;
                }
                if (abort_flag)  // wait for the last e4m3 tiles to land before leaving
                    for (long long n = issued > A8S ? issued - A8S : 0; n < issued; ++n)
                        mbar_drain(&a8full[n % A8S], (uint32_t)((n / A8S) & 1), p.wait_ns);
            }
        } else {
            // converters, A in tensor memory: a thread owns one row of the tile
            // (TMEM lane q*32 + lane, q = warp % 4, the lanes this warp may
            // address) and CPT of its 64 codes per k-block.  It reads them from
            // the e4m3 tile (64-byte swizzle: chunk c of row i sits at chunk
            // c ^ ((i >> 1) & 3), so the 8 rows of a shared-memory phase hit 8
            // distinct bank groups), widens them to bf16 = bf16(float(q) * scale)
            // and stores them into the stage's A columns with tcgen05.st.
            constexpr int PER_Q = CW / 4;      // converter warps per lane quarter
            constexpr int CPT = 64 / PER_Q;    // codes per thread and k-block
            constexpr int NCH = CPT / 16;      // 16-byte chunks per thread
            constexpr int NW = CPT / 2;        // bf16x2 words = TMEM columns
            const int q = warp & 3;
            const int h = (warp - 7) >> 2;     // which CPT codes of the row
            const int row = q * 32 + lane;
            const int xr = (row >> 1) & 3;
            const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16) + ACOL + h * NW;
            const int nsc = p.H / 128;  // scales per row; one k-block uses scale kb / 2
            const long long nrows = (long long)p.R * p.C;
            int s = 0;
            long long n = 0;  // k-blocks converted: tile n % A8S of the e4m3 ring
            for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
                int pair, mt, nt, r, g;
                locate(tile, pair, mt, nt);
                pair_rg(pair, r, g);
                const long long grow =
                    (long long)r * p.C + (g ? __ldg(p.cu + r * G + g - 1) : 0) + mt * TM + row;
                const bool live = grow < nrows;  // rows past the block are zero-filled
                const float* srow = p.scale + (live ? grow * nsc : 0);
                // the scale of the next 128 columns is loaded one group ahead
                float sc = live ? __ldg(srow) : 0.0f;
                float sc_next = live && nsc > 1 ? __ldg(srow + 1) : 0.0f;
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (kb > 0 && (kb & 1) == 0) {
                        sc = sc_next;
                        const int gi = (kb >> 1) + 1;
                        sc_next = live && gi < nsc ? __ldg(srow + gi) : 0.0f;
                    }
                    // the e4m3 tile landed
                    const int j8 = (int)(n % A8S);
                    if (!mbar_wait(&a8full[j8], (uint32_t)((n / A8S) & 1), p.wait_ns, &abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint8_t* a8 = a8ring + j8 * A8_BYTES + row * 64;
                    uint32_t o[NW];
#pragma unroll
                    for (int i = 0; i < NCH; ++i) {
                        const int c = h * NCH + i;
                        const uint4 v = *reinterpret_cast<const uint4*>(a8 + ((c ^ xr) << 4));
                        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            o[8 * i + 2 * k] = widen_e4m3x2(w4[k] & 0xffffu, sc);
                            o[8 * i + 2 * k + 1] = widen_e4m3x2(w4[k] >> 16, sc);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&a8empty[j8]);  // the e4m3 tile is read
                    // widened in registers first; now wait until the MMAs that
                    // read this stage's A columns last (k-block n - STAGES) are
                    // done, and order their reads before the stores
                    if (!mbar_wait(&empty[s], (uint32_t)(((n / STAGES) & 1) ^ 1), p.wait_ns,
                                   &abort_flag)) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;");
                    tmem_store<NW>(tlane + s * 32, o);
                    // the tensor-memory stores complete before the MMA reads them
                    asm volatile("tcgen05.fence::before_thread_sync;");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&conv[s]);
                    ++n;
                    if (++s == STAGES) s = 0;
                }
                if (!ok) break;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS));
    }
    if (tid == 0 && abort_flag) atomicMax(p.status + ST_STATUS, MOONEP_STATUS_TIMEOUT);
}

using PFN_encodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled encoder() {
    static PFN_encodeTiled fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (PFN_encodeTiled) nullptr;
        return reinterpret_cast<PFN_encodeTiled>(f);
    }();
    return fn;
}

bool encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType type, uint64_t elem_bytes,
               uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle) {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * elem_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t es[2] = {1, 1};
    return encoder()(m, type, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// alignment slack + stages + e4m3 ring + barriers (3 per stage, 2 per e4m3
// slot, 2 + 2 accumulator, drain, never) + TMEM address + per-warp sums +
// the m-tile prefix + the epilogue's row staging
size_t smem_bytes(int bn, int stages, int npairs, bool fp8a, int a8_slots = 2, int mt = 1,
                  bool stg = true) {
    return 1024 + (size_t)stages * ((fp8a ? 0 : mt * A_BYTES) + BK * bn * 2) +
           (fp8a ? a8_slots * A8_BYTES : 0) +
           (size_t)(3 * stages + 2 * a8_slots + 6) * 8 + 8 + 32 * 4 + (size_t)(npairs + 1) * 4 +
           (stg ? 16 + EPI_WARPS * 32 * 80 : 0);
}

template <int BN, int STAGES, bool FP8A, int CW = 8, int A8_SLOTS = 2, int NSUB = 1, int MT = 1,
          bool STG = true>
cudaError_t launch_variant(const CUtensorMap& x, const CUtensorMap& w, const GemmArgs& a,
                           size_t smem, int grid, cudaStream_t s) {
    static std::mutex mu;
    static size_t set[64] = {};  // attribute value set so far, per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64 || set[dev] < smem) {
            e = cudaFuncSetAttribute(expert_gemm_kernel<BN, STAGES, FP8A, CW, A8_SLOTS, NSUB, MT, STG>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) set[dev] = smem;
        }
    }
    expert_gemm_kernel<BN, STAGES, FP8A, CW, A8_SLOTS, NSUB, MT, STG>
        <<<grid, threads_for<FP8A, CW>(), smem, s>>>(x, w, a);
    return cudaGetLastError();
}

}  // namespace

int expert_gemm_npairs(const moonep_config& c) { return c.R * (c.E / c.R + c.B); }

// fp8 payload: tile columns, MMA-ring stages and e4m3 slots
constexpr int FP8_TN = 384;
constexpr int FP8_STAGES = 3;
constexpr int FP8_A8 = 4;

// the fp8 kernel's configuration, or the smallest bf16 one
bool expert_gemm_fits(const moonep_config& c) {
    const int np = expert_gemm_npairs(c);
    // the smallest layout of each payload: fp8 without the epilogue's row
    // staging (E + R*B up to 9216 pairs fits either way)
    return (c.payload == MOONEP_PAYLOAD_FP8
                ? smem_bytes(FP8_TN, FP8_STAGES, np, true, FP8_A8, 1, false)
                : smem_bytes(128, 3, np, false)) <= (size_t)SMEM_LIMIT;
}

cudaError_t launch_expert_gemm(const moonep_config& c, const moonep_plan_t& p, const void* x,
                               const float* x_scale, const void* w, void* y, cudaStream_t s,
                               const char** why) {
    if (!encoder()) {
        *why = "cuTensorMapEncodeTiled is unavailable";
        return cudaErrorNotSupported;
    }
    const bool fp8 = c.payload == MOONEP_PAYLOAD_FP8;
    const int C = c.S * c.K;
    const int np = expert_gemm_npairs(c);
    CUtensorMap tx, tw;
    const bool ok_x =
        fp8 ? encode_2d(&tx, x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)c.H, (uint64_t)c.R * C,
                        BK, BM, CU_TENSOR_MAP_SWIZZLE_64B)
            : encode_2d(&tx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)c.H,
                        (uint64_t)c.R * C, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok_x || !encode_2d(&tw, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)c.Hp,
                            (uint64_t)c.R * (c.E + c.B) * c.H, 64, BK,
                            CU_TENSOR_MAP_SWIZZLE_128B)) {
        *why = "cuTensorMapEncodeTiled rejected the recv or weight layout";
        return cudaErrorInvalidValue;
    }
    GemmArgs a;
    a.R = c.R; a.C = C; a.E = c.E; a.B = c.B; a.Er = c.E / c.R; a.H = c.H; a.Hp = c.Hp;
    a.cu = p.cu_seqlens;
    a.status = p.status;
    a.y = static_cast<uint16_t*>(y);
    a.scale = x_scale;
    a.wait_ns = current_wait_limit_ns();
    a.debug_stall = current_barrier_extra() != 0;
    const int grid = device_sm_count();
    if (fp8) {  // 128 x 384 tiles (two MMAs of N = 192 per widened A block): one
                // accumulator and 3 A stages in the 512 TMEM columns; the
                // epilogue's row staging when it fits beside the m-tile prefix
        const size_t s1 = smem_bytes(FP8_TN, FP8_STAGES, np, true, FP8_A8, 1, true);
        if (s1 <= (size_t)SMEM_LIMIT)
            return launch_variant<192, FP8_STAGES, true, 8, FP8_A8, FP8_TN / 192, 1, true>(
                tx, tw, a, s1, grid, s);
        return launch_variant<192, FP8_STAGES, true, 8, FP8_A8, FP8_TN / 192, 1, false>(
            tx, tw, a, smem_bytes(FP8_TN, FP8_STAGES, np, true, FP8_A8, 1, false), grid, s);
    }
    if (c.Hp % 256 == 0) {
#ifndef GEMM_MT1
        // 256 x 256 tiles (two m-tiles per B block), one accumulator
        if (smem_bytes(256, 3, np, false, 2, 2) <= (size_t)SMEM_LIMIT)
            return launch_variant<256, 3, false, 8, 2, 1, 2>(tx, tw, a,
                                                            smem_bytes(256, 3, np, false, 2, 2),
                                                            grid, s);
#endif
        if (smem_bytes(256, 4, np, false) <= (size_t)SMEM_LIMIT)
            return launch_variant<256, 4, false>(tx, tw, a, smem_bytes(256, 4, np, false), grid, s);
        if (smem_bytes(256, 3, np, false) <= (size_t)SMEM_LIMIT)
            return launch_variant<256, 3, false>(tx, tw, a, smem_bytes(256, 3, np, false), grid, s);
    }
    if (smem_bytes(128, 6, np, false) <= (size_t)SMEM_LIMIT)
        return launch_variant<128, 6, false>(tx, tw, a, smem_bytes(128, 6, np, false), grid, s);
    return launch_variant<128, 3, false>(tx, tw, a, smem_bytes(128, 3, np, false), grid, s);
}

}  // namespace moonep
