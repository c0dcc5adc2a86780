/*
 * moonep.h -- C ABI of libmoonep.so: the MoonEP perfectly balanced
 * expert-parallel path (plan -> zero-copy dispatch -> combine) and its side
 * steps (replica weight prefetch, replica gradient reduction) for R logical
 * expert-parallel ranks held as partitions of one GPU's memory.
 *
 * Sources (web pages describing MoonEP):
 *   [ainovat]  "Moonshot AI Open-Sources MoonEP: A Perfectly Balanced Expert
 *              Parallelism Library for MoE Training" (ainovat.com)
 *   [findrepo] "MoonEP" repository card (findrepo.work), "Strengths"
 *   [blog]     "MoonEP" (moses-y.github.io), sections "What This Does",
 *              "How It Is Wired", "How To Use It", "Real-World Use"
 *
 * Notation: R ranks, S tokens per rank, E routed experts, K picks per
 * token, B redundant-expert (prefetch) slots per rank, H hidden size, Hp the
 * expert FFN intermediate size (H' on the pages).  T = R*S tokens; global
 * token id t = r_src*S + s; pick id p = t*K + k; P = T*K; C = S*K rows per
 * rank; Er = E/R home experts per rank, expert e's home rank is e / Er.
 *
 * Conventions shared by every call:
 *  - All buffers are caller-allocated device memory unless a parameter says
 *    "host".  The library allocates device memory only inside
 *    moonep_weights_create().  The caller keeps ownership of everything it
 *    passes in.
 *  - Every compute call only enqueues work on `stream` (a cudaStream_t,
 *    passed as void*; NULL = the legacy default stream) and returns without
 *    waiting for the GPU.  Shapes never depend on the routing, so no call
 *    needs a device-to-host read ([ainovat], the paragraph on dynamic shapes
 *    forcing per-layer host synchronisation; [findrepo] "Strengths").
 *    moonep_plan_status() is the only call that waits.
 *  - Return value: MOONEP_OK, MOONEP_ERR_INVALID_ARG (a size or pointer was
 *    rejected before anything was enqueued) or MOONEP_ERR_CUDA (a CUDA call
 *    failed).  moonep_last_error() gives a one-line reason for the calling
 *    thread's last failure.
 *  - Results that depend on the data (a slot budget overrun, an expert index
 *    out of range, a device wait that gave up) are written by the planner to
 *    the plan's device status block.  Dispatch, combine, prefetch, grad-reduce
 *    and the expert stand-in read it first and do nothing when it is not
 *    MOONEP_STATUS_OK, so a failed plan never moves data.  A kernel that
 *    finds a plan index outside its buffers (dst_row outside [0, P), a slot
 *    expert >= E: a corrupted or overwritten plan) skips or clamps that
 *    access, so nothing outside the buffers is touched, and sets
 *    MOONEP_STATUS_INTERNAL.
 *  - Layouts are row-major and contiguous.  Row pointers must be 16-byte
 *    aligned (every cudaMalloc / torch allocation is).
 */
#ifndef MOONEP_H
#define MOONEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---------------------------------------------------- */
#define MOONEP_OK 0
#define MOONEP_ERR_INVALID_ARG 1
#define MOONEP_ERR_CUDA 2

/* ---- device status word values (status block word 0) ----------------- */
#define MOONEP_STATUS_OK 0
#define MOONEP_STATUS_SLOT_BUDGET 3 /* some rank needs more than B slots */
#define MOONEP_STATUS_BAD_INDEX 4   /* a top-K index outside [0, E) */
#define MOONEP_STATUS_TIMEOUT 5     /* a bounded device wait gave up */
#define MOONEP_STATUS_INTERNAL 6    /* a kernel's own range check failed (a library bug) */

/* ---- payload and rule selectors ------------------------------------- */
#define MOONEP_PAYLOAD_BF16 0 /* dispatch copies bf16 rows */
#define MOONEP_PAYLOAD_FP8 1  /* e4m3 rows + one fp32 scale per 128 elements */

#define MOONEP_RULE_INDEX_ORDER 0   /* keep home rows in expert index order */
#define MOONEP_RULE_KEEP_LIGHTEST 1 /* keep the lightest home experts whole */
#define MOONEP_RULE_LARGEST_FIRST 2 /* keep as rule 1; hand the largest overflows to the
                                       ranks with the largest deficits first */

#define MOONEP_EXPERT_IDENTITY 0 /* stand-in expert: out = payload (fp8: dequantised) */
#define MOONEP_EXPERT_SCALE 1    /* stand-in expert: out = bf16(v * (1 + e/E)) */

/* ---- limits ----------------------------------------------------------- */
#define MOONEP_MAX_E 1024
#define MOONEP_MAX_R 128
#define MOONEP_MAX_B 64
#define MOONEP_MAX_K 32
#define MOONEP_STATUS_WORDS 8

typedef void* moonep_stream_t; /* a cudaStream_t */

/* One MoE layer's sizes and choices. */
typedef struct moonep_config {
    int32_t R, S, E, K, B; /* ranks, tokens/rank, experts, picks/token, slots/rank */
    int32_t H;             /* hidden size; a multiple of 8 (of 128 for fp8) */
    int32_t Hp;            /* expert intermediate size H' (weights only; 0 if unused) */
    int32_t payload;       /* MOONEP_PAYLOAD_* */
    int32_t rule;          /* MOONEP_RULE_* (0, 1 or 2) */
} moonep_config;

/* Byte sizes of every buffer a layer needs: the "buffer and prefetch-pool
 * sizes" the pages compute from a config ([ainovat], the paragraph on the
 * size explainer; [findrepo] "Considerations", the B prefetch slots' extra
 * memory). */
typedef struct moonep_sizes_t {
    int64_t tokens;                 /* T = R*S */
    int64_t picks;                  /* P = T*K */
    int64_t rows_per_rank;          /* C = S*K, the static per-rank row count */
    size_t topk_idx_bytes;          /* int32 [T, K] */
    size_t topk_w_bytes;            /* fp32 [T, K] */
    size_t x_bytes;                 /* bf16 [T, H] */
    size_t recv_bytes;              /* payload [R*C, H]: bf16 or e4m3 */
    size_t recv_scale_bytes;        /* fp32 [R*C, H/128] for fp8, else 0 */
    size_t dispatch_buffer_bytes_per_rank; /* C*H payload + scales of one rank */
    size_t expert_out_bytes;        /* bf16 [R*C, H] */
    size_t y_bytes;                 /* bf16 [T, H] */
    size_t expert_count_bytes;      /* int32 [E] */
    size_t rank_load_bytes;         /* int32 [R] */
    size_t slot_expert_bytes;       /* int32 [R*B] */
    size_t cu_seqlens_bytes;        /* int32 [R*(E+B)] */
    size_t dst_row_bytes;           /* int32 [P] */
    size_t src_of_row_bytes;        /* int32 [P] */
    size_t status_bytes;            /* int32 [MOONEP_STATUS_WORDS] */
    size_t maxvio_bytes;            /* double [1] */
    size_t workspace_bytes;         /* planner scratch */
    size_t weight_row_bytes;        /* H*Hp bf16: one expert's projection */
    size_t prefetch_pool_bytes_per_rank; /* B * weight_row_bytes */
    size_t weights_view_bytes;      /* (E+B) * weight_row_bytes: one rank's [E+B,H,Hp] view */
} moonep_sizes_t;

/* The plan of one layer: all device pointers, sized by moonep_sizes(). */
typedef struct moonep_plan_t {
    int32_t* expert_count; /* [E]     picks routed to each expert (the T_e of maxvio) */
    int32_t* rank_load;    /* [R]     home rows of each rank before balancing */
    int32_t* slot_expert;  /* [R*B]   expert hosted in slot j of rank r, -1 if unused */
    int32_t* cu_seqlens;   /* [R*(E+B)] per rank, inclusive end row of each group */
    int32_t* dst_row;      /* [T*K]   destination row r*C+i of pick p = t*K+k */
    int32_t* src_of_row;   /* [R*C]   pick p that fills each row (inverse of dst_row) */
    int32_t* status;       /* [MOONEP_STATUS_WORDS]: [0] status, [1] failing rank,
                              [2] slots it needs, [3] max_e T_e; [4..7] planner-internal */
    double* maxvio;        /* [1]     max_e(T_e / Tbar) - 1, Tbar = P/E */
    void* workspace;       /* planner scratch of workspace_bytes, 16-byte aligned; read by
                              moonep_plan only, so the other calls accept NULL here */
    size_t workspace_bytes;
} moonep_plan_t;

/* Per-rank [E+B, H, Hp] weight views made by moonep_weights_create(). */
typedef struct moonep_weights_t {
    void* rank_view[MOONEP_MAX_R]; /* device address of rank r's view */
    size_t row_bytes;              /* bytes of one expert row (H*Hp*elem_bytes) */
    size_t view_bytes;             /* (E+B) * row_bytes */
    int32_t R, E, B, elem_bytes;
    void* impl;                    /* library-owned bookkeeping */
} moonep_weights_t;

/* Library version (major*10000 + minor*100 + patch). */
int moonep_version(void);

/* One-line reason for the calling thread's last non-OK return. */
const char* moonep_last_error(void);

/* Fill *out with the byte sizes for `cfg`.  Validates cfg: R, S, E, K, H > 0,
 * B >= 0, E % R == 0, E <= MOONEP_MAX_E, R <= MOONEP_MAX_R, B <= MOONEP_MAX_B,
 * K <= MOONEP_MAX_K, K <= E * S (fits), H % 8 == 0 (H % 128 == 0 for fp8),
 * R*S*K < 2^31.  Returns MOONEP_ERR_INVALID_ARG otherwise. */
int moonep_sizes(const moonep_config* cfg, moonep_sizes_t* out);

/* Plan one layer ([ainovat], the paragraphs on the hard invariant and on
 * planning redundant experts online from the current router outputs; [blog]
 * "What This Does", the planning kernel).
 *
 * topk_idx: int32 [T, K] router picks, row-major, token-major (device).
 * Computes expert_count, rank_load, max count and maxvio; then, rule by rule:
 * each rank keeps its home rows (experts in index order, rows in (t, k)
 * order) up to C -- rules MOONEP_RULE_KEEP_LIGHTEST and _LARGEST_FIRST keep
 * the lightest experts whole instead -- the rows not kept form one stream,
 * expert by expert (index order; for _LARGEST_FIRST by decreasing overflow,
 * ties to the lower index), each expert's rows in (t, k) order, that fills
 * the under-full ranks (in rank order; for _LARGEST_FIRST by decreasing
 * deficit, ties to the lower rank) to exactly C rows each;
 * every distinct expert a rank receives takes one slot, in order of first
 * appearance; the kept rows come first in a rank's buffer, in expert order,
 * then the slot groups in slot order.  cu_seqlens[r][g] is the end row of
 * group g (experts 0..E-1, then slots E..E+B-1) in rank r's buffer; its last
 * entry is C.
 * A rank needing more than B slots sets status SLOT_BUDGET with the lowest
 * failing rank and its slot count; an index outside [0, E) sets BAD_INDEX.
 * Then only expert_count, rank_load, max count and maxvio are defined.
 * One memset of the status block plus one kernel; no host synchronisation. */
int moonep_plan(const moonep_config* cfg, const int32_t* topk_idx, const moonep_plan_t* plan,
                moonep_stream_t stream);

/* Zero-copy dispatch ([blog] "What This Does": tokens go straight to their
 * final expert-grouped position, no permute step and no copy out of a
 * communication buffer; [findrepo] "Strengths").
 *
 * x: bf16 [T, H] (device).  recv: [R*C, H], rank r's buffer is rows
 * r*C .. r*C+C-1.  Row dst_row[t*K+k] receives token t:
 *  - payload BF16: a bit copy of x[t].  recv_scale must be NULL.
 *  - payload FP8: per block of 128 elements, amax = max |x|; scale = amax/448
 *    and q = e4m3(x * (448/amax)), round to nearest even, saturating; a zero
 *    block gets scale 1 and zero codes.  recv is uint8 e4m3 [R*C, H] and
 *    recv_scale fp32 [R*C, H/128].  Each token is quantised once and its K
 *    copies are identical. */
int moonep_dispatch(const moonep_config* cfg, const moonep_plan_t* plan, const void* x,
                    void* recv, float* recv_scale, moonep_stream_t stream);

/* Combine ([blog] "What This Does" and "Real-World Use": gather the expert
 * outputs back and reduce them per token with the router weights).
 *
 * expert_out: bf16 [R*C, H] (may be the bf16 recv buffer itself).
 * topk_w: fp32 [T, K].  y: bf16 [T, H].
 * y[t] = bf16(acc), acc = 0; for k = 0..K-1: acc = fma(w[t,k],
 * float(expert_out[dst_row[t,k]]), acc) in binary32; bf16 rounding is to
 * nearest even. */
int moonep_combine(const moonep_config* cfg, const moonep_plan_t* plan, const void* expert_out,
                   const float* topk_w, void* y, moonep_stream_t stream);

/* Backward of combine, for the layer's backward pass ([blog] "Real-World
 * Use": the backward pass runs after combine; by the chain rule through
 * y[t] = sum_k w[t,k] * expert_out[dst_row[t,k]]).
 *
 * dy: bf16 [T, H]; expert_out: bf16 [R*C, H] (the forward's expert outputs);
 * topk_w: fp32 [T, K].  Writes
 *   d_expert_out bf16 [R*C, H]: row dst_row[t,k] = bf16(w[t,k] * float(dy[t])),
 *     one binary32 product rounded to nearest even;
 *   d_topk_w fp32 [T, K]: sum_h float(dy[t,h]) * float(expert_out[row,h]) in
 *     binary32.  Each of 32 lanes sums its own elements with an fma chain,
 *     then a fixed shuffle tree adds the lanes, so the result is deterministic
 *     and within the recursive-summation bound gamma(L+5) * sum|terms| of the
 *     exact value, L = 8 * ceil(H / 256).
 * Every row of d_expert_out is written (the rows are a permutation of the
 * picks). */
int moonep_combine_backward(const moonep_config* cfg, const moonep_plan_t* plan, const void* dy,
                            const void* expert_out, const float* topk_w, void* d_expert_out,
                            float* d_topk_w, moonep_stream_t stream);

/* Backward of dispatch (recv[dst_row[t,k]] = x[t]):
 * dx[t] = bf16(acc), acc = 0; acc = acc + float(d_recv[dst_row[t,k]]) for
 * k = 0..K-1, binary32 additions in k order, rounded once to bf16.
 * d_recv: bf16 [R*C, H] (for the fp8 payload, the gradient with respect to
 * the dequantised rows); dx: bf16 [T, H]. */
int moonep_dispatch_backward(const moonep_config* cfg, const moonep_plan_t* plan,
                             const void* d_recv, void* dx, moonep_stream_t stream);

/* Replica weight prefetch ([ainovat], the paragraph on fetching duplicated
 * experts before expert computation, and the [E+B, H, H'] contract).
 *
 * rank_weights: host array of R device pointers, rank r's [E+B, H, Hp] view
 * of one projection with elements of elem_bytes (2 for bf16).  Rows 0..E-1
 * hold the home experts (row e is read from rank e/Er's view); for every used
 * slot j of rank r, row E+j of rank r's view receives a bit copy of row e =
 * slot_expert[r][j].  Unused slots are untouched.  H*Hp*elem_bytes must be a
 * multiple of 16. */
int moonep_prefetch(const moonep_config* cfg, const moonep_plan_t* plan,
                    void* const* rank_weights, int32_t elem_bytes, moonep_stream_t stream);

/* Replica gradient reduction ([ainovat], the paragraph on reducing the
 * duplicated experts' gradients back to their home ranks in the backward).
 *
 * rank_grads: host array of R device pointers to fp32 [E+B, H, Hp] views.
 * For every expert e with replicas, in place on its home row (rank e/Er's
 * view, row e): dW[e] = ((dW[e] + g_1) + g_2) + ... over its replicas
 * (r, j) in increasing r then j, g = row E+j of rank r's view; each addition
 * is one binary32 operation, so the result is deterministic. */
int moonep_grad_reduce(const moonep_config* cfg, const moonep_plan_t* plan,
                       float* const* rank_grads, moonep_stream_t stream);

/* Stand-in for the expert computation (the grouped GEMM that consumes the
 * [E+B, H, Hp] weights and cu_seqlens, [ainovat]), used to check combine:
 * MOONEP_EXPERT_IDENTITY: out = recv (fp8: bf16(float(q) * scale));
 * MOONEP_EXPERT_SCALE: out = bf16(float(v) * (1 + e/E)), e the expert of the
 * row's group (a slot group's expert from slot_expert).
 * recv / recv_scale as written by moonep_dispatch; out bf16 [R*C, H]. */
int moonep_expert_standin(const moonep_config* cfg, const moonep_plan_t* plan, const void* recv,
                          const float* recv_scale, int32_t mode, void* out,
                          moonep_stream_t stream);

/* Grouped expert GEMM over the dispatched rows: the consumer that the pages
 * place after dispatch, a grouped GEMM that reads the contiguous [E+B, H, H']
 * weight tensor and selects each group's rows through cu_seqlens[E+B]
 * ([ainovat], the framework-contract paragraph; [blog] "What This Does").
 *
 * recv:    the dispatched rows [R*C, H], rank r's rows at r*C
 *          (moonep_dispatch output): bf16, or for the fp8 payload e4m3 codes
 *          with recv_scale fp32 [R*C, H/128] (NULL for bf16).  fp8 rows are
 *          widened on the SM, into tensor memory, to a = bf16(float(q) *
 *          scale), one binary32 product, round to nearest even -- the same
 *          values the identity stand-in expert produces -- and then
 *          multiplied as bf16; no bf16 copy of them is written to memory.
 * weights: bf16, R consecutive [E+B, H, Hp] views; view r starts at element
 *          r*(E+B)*H*Hp.  Row e < E of a view is home expert e, row E+j is
 *          the replica in rank r's slot j.  The views of
 *          moonep_weights_create(cfg, 2, &w) are laid out this way: pass
 *          w.rank_view[0].
 * out:     bf16 [R*C, Hp].
 * For every rank r and group g, each row i of [cu[r][g-1], cu[r][g]) gets
 *   out[r*C+i][:] = bf16( sum_h recv[r*C+i][h] * weights[r][g][h][:] ),
 * products and sums in fp32 on the tensor cores (summation order not
 * specified), then one round-to-nearest-even to bf16.  Rows of no group do
 * not exist (every rank holds exactly C rows); only the groups a plan can
 * fill are read: rank r's E/R home experts and its B slots.
 * Requires H % 64 == 0, Hp % 128 == 0, R*(E+B)*H < 2^31, recv_scale for
 * the fp8 payload and 16-byte aligned pointers (else INVALID_ARG).  The
 * kernel keeps one entry per (rank, group) pair, E + R*B of them, in shared
 * memory; every configuration within the MOONEP_MAX_* bounds fits.  Does
 * nothing when the plan's status is not OK; a device wait that runs out sets
 * MOONEP_STATUS_TIMEOUT (out is then partly written). */
int moonep_expert_gemm(const moonep_config* cfg, const moonep_plan_t* plan, const void* recv,
                       const float* recv_scale, const void* weights, void* out,
                       moonep_stream_t stream);

/* Wait for `stream`, then copy the first four status words to the host array
 * out[4]: status, failing rank, slots it needs, max_e T_e. */
int moonep_plan_status(const moonep_plan_t* plan, moonep_stream_t stream, int32_t* out);

/* Build R contiguous [E+B, H, Hp] views of one projection with CUDA virtual
 * memory on the current device: rows 0..E-1 of every view map the same
 * physical home block (so a home expert has one copy), rows E..E+B-1 map a
 * private slot block per rank.  The views are consecutive in one address
 * range: rank_view[r] = rank_view[0] + r*view_bytes.  This is the one-GPU form of the pages'
 * symmetric-memory weight tensor ([ainovat], the contract paragraph).
 * Requires H*Hp*elem_bytes to be a multiple of the allocation granularity
 * (2 MiB on current GPUs).  Contents are undefined until written.
 * moonep_weights_destroy() unmaps and frees everything create() made. */
int moonep_weights_create(const moonep_config* cfg, int32_t elem_bytes, moonep_weights_t* out);
int moonep_weights_destroy(moonep_weights_t* w);

/* Allocation-free planner.  The web pages have no counterpart to this call:
 * it is a convenience of this library for callers that cannot give the
 * planner a workspace buffer -- a plugin whose host framework owns all device
 * memory through its own allocator and hands out no scratch, or a serving
 * loop that reserves every buffer at start-up and must not allocate once it
 * runs.
 *
 * Same inputs, outputs and results as moonep_plan(); the workspace fields of
 * *plan are ignored.  The planner's scratch is instead a static device array
 * inside this library, sized for E <= MOONEP_NOALLOC_MAX_E (4 MiB + 2 KiB);
 * every GPU that loads the library holds it until the process exits.  A
 * larger E returns MOONEP_ERR_INVALID_ARG.  The call itself allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *  - Every call made outside a stream capture looks up the array's device
 *    address (cudaGetSymbolAddress, with the calling device current) and
 *    caches it per device with the current driver context.  A call inside a
 *    capture uses that cache and returns MOONEP_ERR_CUDA if it holds no
 *    address for the current context, so make the first call on a device --
 *    and the first after a device reset or a change of driver context --
 *    outside any capture.
 *  - All calls share the one array, which keeps the last call's contents.
 *    Nothing in it needs clearing between calls (each call rewrites every
 *    word it reads; the wait counters live in the plan's status block, which
 *    each call zeroes), but two calls whose kernels overlap on the GPU (other
 *    streams, other host threads) race on it and produce wrong plans: order
 *    them on one stream or synchronise between them. */
#define MOONEP_NOALLOC_MAX_E 512
int moonep_plan_noalloc(const moonep_config* cfg, const int32_t* topk_idx,
                        const moonep_plan_t* plan, moonep_stream_t stream);

/* Bound on every device-side wait, in nanoseconds (default 1e9).  A wait
 * that runs out sets MOONEP_STATUS_TIMEOUT and the kernel returns. */
int moonep_set_wait_limit_ns(uint64_t ns);

/* Test hook: the planner's first grid-wide wait expects `extra` more
 * arrivals than there are blocks, so it runs out after the wait limit and
 * the plan reports MOONEP_STATUS_TIMEOUT; moonep_expert_gemm's epilogue
 * waits on a barrier that nothing completes, with the same outcome.  0 (the
 * default) disables it. */
int moonep_debug_set_barrier_extra(int32_t extra);

#ifdef __cplusplus
}
#endif
#endif /* MOONEP_H */
