/*
 * moonep_oracle.c -- plain, slow, single-threaded CPU oracle for the MoonEP
 * plan -> dispatch -> combine path and its two side steps (replica prefetch,
 * replica gradient reduction).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA library; the two meet only through
 * the seeded input arrays that a test hands to both.
 *
 * Sources (web pages describing MoonEP; no code was published with them):
 *   [ainovat]  "Moonshot AI Open-Sources MoonEP: A Perfectly Balanced Expert
 *              Parallelism Library for MoE Training" (ainovat.com)
 *   [findrepo] "MoonEP" repository card (findrepo.work), sections
 *              "Why it is worth attention" and "Strengths"
 *   [blog]     "MoonEP" (moses-y.github.io), sections "What This Does",
 *              "How It Is Wired", "How To Use It", "Real-World Use"
 *
 * The pages define the quantities but not a planning rule, a row order or
 * number formats.  The readings this file implements (the rule, the slot
 * order, the cu_seqlens convention, the fp8 recipe, the combine rounding
 * order) are stated function by function below.
 *
 * Notation: R ranks, S tokens per rank, E routed experts, K picks per token,
 * B redundant slots per rank, H hidden size.  T = R*S tokens, global token
 * id t = r_src*S + s, pick id p = t*K + k, P = T*K picks, C = S*K rows per
 * rank, Er = E/R home experts per rank; expert e lives on home rank e / Er.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * -ffp-contract=off keeps every float multiply and add a separately rounded
 * IEEE binary32 operation; the one fused step (combine) calls fmaf itself.
 *
 * Parity pins live in the tests: a brute-force planner that sorts
 * (expert, token, k) triples, exhaustive enumeration of tiny routings,
 * hand-worked golden cases, closed forms for maxvio and for round-robin
 * routing, and library cross-checks of the bf16 / e4m3 encoders.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_INVALID 1
#define ORACLE_SLOT_BUDGET 3
#define ORACLE_BAD_INDEX 4

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* bfloat16 -> float: a bf16 value is the upper half of a binary32. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* float -> bfloat16, round to nearest, ties to even.  Keep the upper 16
 * bits; the lower 16 bits are the part that is rounded away.  Above half
 * an ulp round up, at exactly half round to the even neighbour.  A carry
 * out of the mantissa moves into the exponent, which is the correct next
 * representable value (up to infinity).  NaN stays NaN (quiet). */
uint16_t oracle_bf16_from_f32(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u)))
        kept += 1u;
    return (uint16_t)kept;
}

/* Round a non-negative double that holds an exact value to the nearest
 * integer, ties to even. */
static double round_half_even(double q)
{
    double fl = floor(q);
    double diff = q - fl;
    if (diff > 0.5)
        return fl + 1.0;
    if (diff < 0.5)
        return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* FP8 E4M3 (OCP 8-bit floating point specification, "E4M3" encoding):
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinity,
 * NaN = S.1111.111, largest finite magnitude 1.75 * 2^8 = 448, smallest
 * normal 2^-6, subnormals m * 2^-9 for m = 1..7.
 *
 * Conversion from binary32: round to nearest, ties to even, and saturate
 * to +-448 on overflow ("satfinite").  NaN maps to NaN. */
uint8_t oracle_e4m3_from_f32(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v))
        return (uint8_t)(sign | 0x7f);
    double a = fabs((double)v);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7e); /* 0.1111.110 = 448 */
    if (a < 0.015625) {
        /* below the smallest normal 2^-6: a multiple of the subnormal
         * spacing 2^-9.  n = 8 is exactly the smallest normal, whose code
         * is also 8 (exponent field 1, mantissa 0). */
        double n = round_half_even(a * 512.0);
        return (uint8_t)(sign | (uint8_t)n);
    }
    int e2;
    (void)frexp(a, &e2); /* a = m * 2^e2, m in [0.5, 1) */
    int e = e2 - 1;      /* a in [2^e, 2^(e+1)), e in [-6, 8] */
    double spacing = ldexp(1.0, e - 3);
    double n = round_half_even(a / spacing); /* in [8, 16] */
    int code = ((e + 7) << 3) + (int)n - 8;  /* n = 16 carries into the exponent */
    if (code > 0x7e)
        code = 0x7e;
    return (uint8_t)(sign | code);
}

/* FP8 E4M3 -> float (exact). */
float oracle_e4m3_to_f32(uint8_t c)
{
    int s = c >> 7, ex = (c >> 3) & 15, m = c & 7;
    double mag;
    if (ex == 15 && m == 7)
        return s ? -NAN : NAN;
    if (ex == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + m / 8.0, ex - 7);
    return (float)(s ? -mag : mag);
}

void oracle_bf16_from_f32_array(const float* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_from_f32(in[i]);
}

void oracle_e4m3_from_f32_array(const float* in, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_from_f32(in[i]);
}

/* ------------------------------------------------------------------ */
/* Plan                                                                */
/* ------------------------------------------------------------------ */

/*
 * oracle_plan -- the online plan for one MoE layer.
 *
 * What the plan must achieve: every rank receives exactly C = S*K
 * (token, k) rows however skewed the routing ([ainovat], the paragraph on
 * the hard invariant; [findrepo] "Strengths", perfect token balance), by
 * hosting a few redundant experts chosen from the current router outputs
 * ([ainovat], the paragraph on planning redundant experts online).  Rows
 * land directly in their final expert-grouped position ([blog] "What This
 * Does").  Each rank's group layout is described by cu_seqlens over E+B
 * groups ([ainovat], the paragraph on the [E+B, H, H'] contract).
 *
 * The pages leave the rule open; this library fixes it as follows.
 *  O1  histogram cnt[e] over all picks; maxvio = max_e(cnt[e] / Tbar) - 1
 *      with Tbar = P / E, in binary64 ([ainovat], the maxvio definition).
 *  O2  rank r's home rows are the picks of its experts, experts in index
 *      order, rows of one expert in (t, k) order.  rule 0 keeps the first
 *      min(load[r], C) of them.  rule 1 keeps, per expert, as many rows as
 *      fit when the experts are filled lightest first (ascending
 *      (cnt, index)); the kept rows of an expert are its first ones in
 *      (t, k) order, and the kept rows are laid out in expert index order.
 *  O3  the overflow stream is every rank's rows that were not kept, expert
 *      by expert (rank by rank for rules 0 and 1, i.e. expert index order;
 *      by decreasing overflow count, ties to the lower index, for rule 2),
 *      each expert's rows in (t, k) order.
 *  O4  walking the ranks in order (rules 0 and 1: index order; rule 2:
 *      decreasing deficit, ties to the lower index), each rank with a
 *      deficit C - kept[r] takes the next deficit rows of the stream, placed
 *      after its kept rows in stream order.  Rule 2 keeps rows as rule 1
 *      does.
 *  O5  on a receiving rank, each distinct expert of its segment takes one
 *      slot, in order of first appearance.  A rank that needs more than B
 *      slots fails the plan (status ORACLE_SLOT_BUDGET; *fail_rank is the
 *      lowest such rank, *fail_slots the slots it needs); then only O1's
 *      outputs and rank_load are defined.
 *  O6  cu_seqlens[r][g] is the inclusive prefix sum of the row counts of
 *      groups g = 0..E+B-1: group g < E holds rank r's kept rows of expert
 *      g, group E+j holds the rows of slot j.  Its last entry is C.
 *  O7  dst_row[p] = rank * C + row, src_of_row[rank * C + row] = p.
 *
 * Arrays (all int32 unless noted, caller-allocated):
 *   idx[P] in; expert_count[E], rank_load[R], max_count[1], maxvio[1]
 *   (double), slot_expert[R*B] (-1 = unused), cu_seqlens[R*(E+B)],
 *   dst_row[P], src_of_row[P], fail_rank[1], fail_slots[1] out.
 * Returns ORACLE_OK, ORACLE_INVALID, ORACLE_SLOT_BUDGET or
 * ORACLE_BAD_INDEX (an index outside [0, E); nothing else is defined).
 */
int oracle_plan(int R, int S, int E, int K, int B, int rule,
                const int32_t* idx,
                int32_t* expert_count, int32_t* rank_load, int32_t* max_count,
                double* maxvio, int32_t* slot_expert, int32_t* cu_seqlens,
                int32_t* dst_row, int32_t* src_of_row,
                int32_t* fail_rank, int32_t* fail_slots)
{
    if (R <= 0 || S <= 0 || E <= 0 || K <= 0 || B < 0 || E % R != 0 ||
        rule < 0 || rule > 2)
        return ORACLE_INVALID;
    const int64_t T = (int64_t)R * S, P = T * K, C = (int64_t)S * K;
    const int Er = E / R;
    *fail_rank = -1;
    *fail_slots = 0;

    /* O1: histogram and maxvio. */
    for (int e = 0; e < E; ++e)
        expert_count[e] = 0;
    for (int64_t p = 0; p < P; ++p) {
        if (idx[p] < 0 || idx[p] >= E)
            return ORACLE_BAD_INDEX;
        expert_count[idx[p]] += 1;
    }
    int32_t mx = 0;
    for (int e = 0; e < E; ++e)
        if (expert_count[e] > mx)
            mx = expert_count[e];
    *max_count = mx;
    double Tbar = (double)P / (double)E;
    *maxvio = (double)mx / Tbar - 1.0;

    for (int r = 0; r < R; ++r) {
        int64_t load = 0;
        for (int e = r * Er; e < (r + 1) * Er; ++e)
            load += expert_count[e];
        rank_load[r] = (int32_t)load;
    }

    /* Each expert's picks in (t, k) order: a counting sort by expert,
     * filled by scanning the picks in increasing p. */
    int64_t* first = (int64_t*)malloc(sizeof(int64_t) * (size_t)(E + 1));
    int64_t* fillpos = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
    int32_t* rows_of = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
    int64_t* kept_n = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
    int* order = (int*)malloc(sizeof(int) * (size_t)Er);
    int64_t* next_row = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    int32_t* stream = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
    int32_t* stream_e = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
    int32_t* row_group = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
    int64_t* gcount = (int64_t*)malloc(sizeof(int64_t) * (size_t)(E + B));
    int* xorder = (int*)malloc(sizeof(int) * (size_t)E);
    int* rorder = (int*)malloc(sizeof(int) * (size_t)R);
    int* rslots = (int*)malloc(sizeof(int) * (size_t)R);
    if (!first || !fillpos || !rows_of || !kept_n || !order || !next_row ||
        !stream || !stream_e || !row_group || !gcount || !xorder || !rorder || !rslots) {
        free(first); free(fillpos); free(rows_of); free(kept_n); free(order);
        free(next_row); free(stream); free(stream_e); free(row_group); free(gcount);
        free(xorder); free(rorder); free(rslots);
        return ORACLE_INVALID;
    }
    first[0] = 0;
    for (int e = 0; e < E; ++e)
        first[e + 1] = first[e] + expert_count[e];
    for (int e = 0; e < E; ++e)
        fillpos[e] = first[e];
    for (int64_t p = 0; p < P; ++p)
        rows_of[fillpos[idx[p]]++] = (int32_t)p;

    /* O2: how many rows of each home expert its home rank keeps. */
    for (int r = 0; r < R; ++r) {
        for (int i = 0; i < Er; ++i)
            order[i] = r * Er + i; /* rule 0: index order */
        if (rule >= 1) {
            /* lightest first: insertion sort by (cnt, index) */
            for (int i = 1; i < Er; ++i) {
                int cur = order[i], j = i - 1;
                while (j >= 0 &&
                       (expert_count[order[j]] > expert_count[cur] ||
                        (expert_count[order[j]] == expert_count[cur] && order[j] > cur))) {
                    order[j + 1] = order[j];
                    --j;
                }
                order[j + 1] = cur;
            }
        }
        int64_t remaining = C;
        for (int i = 0; i < Er; ++i) {
            int e = order[i];
            int64_t take = expert_count[e] < remaining ? expert_count[e] : remaining;
            kept_n[e] = take;
            remaining -= take;
        }
    }

    /* Kept rows, laid out expert by expert in index order. */
    for (int r = 0; r < R; ++r) {
        next_row[r] = 0;
        for (int e = r * Er; e < (r + 1) * Er; ++e) {
            for (int64_t i = 0; i < kept_n[e]; ++i) {
                int32_t p = rows_of[first[e] + i];
                int64_t row = next_row[r]++;
                dst_row[p] = (int32_t)(r * C + row);
                src_of_row[r * C + row] = p;
                row_group[r * C + row] = e;
            }
        }
    }

    /* O3: the overflow stream: each expert's rows that were not kept, in
     * (t, k) order.  Rules 0 and 1 take the experts in index order (which is
     * rank order, since ranks own contiguous experts); rule 2 takes them in
     * order of decreasing overflow count, ties to the lower index. */
    for (int e = 0; e < E; ++e)
        xorder[e] = e;
    if (rule == 2) {
        for (int i = 1; i < E; ++i) {
            int cur = xorder[i], j = i - 1;
            int64_t oc = expert_count[cur] - kept_n[cur];
            while (j >= 0 && (expert_count[xorder[j]] - kept_n[xorder[j]] < oc ||
                              (expert_count[xorder[j]] - kept_n[xorder[j]] == oc && xorder[j] > cur))) {
                xorder[j + 1] = xorder[j];
                --j;
            }
            xorder[j + 1] = cur;
        }
    }
    int64_t nstream = 0;
    for (int i = 0; i < E; ++i) {
        int e = xorder[i];
        for (int64_t k = kept_n[e]; k < expert_count[e]; ++k) {
            stream[nstream] = rows_of[first[e] + k];
            stream_e[nstream] = e;
            ++nstream;
        }
    }

    /* O4: the receiving order.  Rules 0 and 1 walk the ranks in index
     * order; rule 2 in order of decreasing deficit C - kept, ties to the
     * lower index.  Ranks without a deficit take nothing. */
    for (int r = 0; r < R; ++r)
        rorder[r] = r;
    if (rule == 2) {
        for (int i = 1; i < R; ++i) {
            int cur = rorder[i], j = i - 1;
            int64_t dc = C - next_row[cur];
            while (j >= 0 && (C - next_row[rorder[j]] < dc ||
                              (C - next_row[rorder[j]] == dc && rorder[j] > cur))) {
                rorder[j + 1] = rorder[j];
                --j;
            }
            rorder[j + 1] = cur;
        }
    }

    /* O4 + O5: cut the stream in the receiving order, assign slots, place
     * the segment rows. */
    for (int64_t i = 0; i < (int64_t)R * B; ++i)
        slot_expert[i] = -1;
    int64_t pos = 0;
    for (int i = 0; i < R; ++i) {
        int r = rorder[i];
        int64_t deficit = C - next_row[r];
        int nslots = 0;
        int last_e = -1;
        /* the stream is grouped by expert, so a new expert shows up as a
         * change of expert id */
        for (int64_t q = 0; q < deficit; ++q) {
            int e = stream_e[pos + q];
            if (e != last_e) {
                ++nslots;
                last_e = e;
            }
        }
        rslots[r] = nslots;
        if (nslots <= B) {
            int j = -1;
            last_e = -1;
            for (int64_t q = 0; q < deficit; ++q) {
                int e = stream_e[pos + q];
                if (e != last_e) {
                    ++j;
                    slot_expert[(int64_t)r * B + j] = e;
                    last_e = e;
                }
                int32_t p = stream[pos + q];
                int64_t row = next_row[r]++;
                dst_row[p] = (int32_t)(r * C + row);
                src_of_row[r * C + row] = p;
                row_group[r * C + row] = E + j;
            }
        }
        pos += deficit;
    }
    /* a rank that needs more than B slots fails the plan: report the lowest
     * such rank and the slots it needs */
    int status = ORACLE_OK;
    for (int r = 0; r < R; ++r)
        if (rslots[r] > B) {
            status = ORACLE_SLOT_BUDGET;
            *fail_rank = r;
            *fail_slots = rslots[r];
            break;
        }

    /* O6: cu_seqlens from the rows actually placed. */
    if (status == ORACLE_OK) {
        for (int r = 0; r < R; ++r) {
            for (int g = 0; g < E + B; ++g)
                gcount[g] = 0;
            for (int64_t i = 0; i < C; ++i)
                gcount[row_group[r * C + i]] += 1;
            int64_t acc = 0;
            for (int g = 0; g < E + B; ++g) {
                acc += gcount[g];
                cu_seqlens[(int64_t)r * (E + B) + g] = (int32_t)acc;
            }
        }
    }

    free(first); free(fillpos); free(rows_of); free(kept_n); free(order);
    free(next_row); free(stream); free(stream_e); free(row_group); free(gcount);
    free(xorder); free(rorder); free(rslots);
    return status;
}

/* ------------------------------------------------------------------ */
/* Dispatch                                                            */
/* ------------------------------------------------------------------ */

/* O8, bf16 payload: recv[row][:] = x[src_of_row[row] / K][:], a bit copy
 * ([blog] "What This Does": tokens move straight to their final
 * expert-grouped position).  Computes the n requested rows only; out is
 * [n][H] bf16 bits. */
void oracle_dispatch_rows(int K, int H, const uint16_t* x, const int32_t* src_of_row,
                          const int64_t* rows, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = src_of_row[rows[i]] / K;
        memcpy(out + i * (int64_t)H, x + t * (int64_t)H, sizeof(uint16_t) * (size_t)H);
    }
}

/* O8, fp8 payload, one token row: for each block of 128 elements,
 * amax = max |x|; amax = 0 gives scale 1 and all-zero codes; otherwise
 * scale = amax / 448 and q = e4m3(x * (448 / amax)), each division and the
 * product one binary32 operation rounded to nearest. */
void oracle_quant_row_e4m3(int H, const uint16_t* xrow, uint8_t* q, float* scale)
{
    for (int b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) {
            float a = fabsf(oracle_bf16_to_f32(xrow[b * 128 + i]));
            if (a > amax)
                amax = a;
        }
        if (amax == 0.0f) {
            scale[b] = 1.0f;
            for (int i = 0; i < 128; ++i)
                q[b * 128 + i] = 0;
            continue;
        }
        float s = amax / 448.0f;
        float inv = 448.0f / amax;
        scale[b] = s;
        for (int i = 0; i < 128; ++i) {
            float v = oracle_bf16_to_f32(xrow[b * 128 + i]) * inv;
            q[b * 128 + i] = oracle_e4m3_from_f32(v);
        }
    }
}

/* fp8 dispatch of the n requested rows: each row is the quantised copy of
 * its source token.  q_out [n][H] codes, s_out [n][H/128] scales. */
void oracle_dispatch_rows_fp8(int K, int H, const uint16_t* x, const int32_t* src_of_row,
                              const int64_t* rows, int64_t n, uint8_t* q_out, float* s_out)
{
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = src_of_row[rows[i]] / K;
        oracle_quant_row_e4m3(H, x + t * (int64_t)H, q_out + i * (int64_t)H,
                              s_out + i * (int64_t)(H / 128));
    }
}

/* ------------------------------------------------------------------ */
/* Expert stand-ins (test only; they take the place of the group GEMM) */
/* ------------------------------------------------------------------ */

/* Which expert a row of rank r belongs to: the group g whose
 * [cu_seqlens[g-1], cu_seqlens[g]) holds the row, mapped through the slot
 * map for slot groups. */
int oracle_row_expert(int E, int B, const int32_t* cu_r, const int32_t* slot_r, int64_t row)
{
    for (int g = 0; g < E + B; ++g) {
        if (row < cu_r[g])
            return g < E ? g : slot_r[g - E];
    }
    return -1;
}

/* Scale expert: out = bf16(float(v) * (1 + e / E)), e the row's expert.
 * in/out are [n][H] bf16 rows; rows[i] is the global row index rank*C+i. */
void oracle_expert_scale_rows(int E, int B, int64_t C, int H, const int32_t* cu_seqlens,
                              const int32_t* slot_expert, const int64_t* rows, int64_t n,
                              const uint16_t* in, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) {
        int64_t r = rows[i] / C, row = rows[i] % C;
        int e = oracle_row_expert(E, B, cu_seqlens + r * (E + B), slot_expert + r * B, row);
        float s = 1.0f + (float)e / (float)E;
        for (int h = 0; h < H; ++h) {
            float v = oracle_bf16_to_f32(in[i * H + h]) * s;
            out[i * H + h] = oracle_bf16_from_f32(v);
        }
    }
}

/* Identity expert on the fp8 payload: out = bf16(float(q) * scale). */
void oracle_dequant_rows(int H, int64_t n, const uint8_t* q, const float* s, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        for (int h = 0; h < H; ++h) {
            float v = oracle_e4m3_to_f32(q[i * H + h]) * s[i * (H / 128) + h / 128];
            out[i * H + h] = oracle_bf16_from_f32(v);
        }
}

/* ------------------------------------------------------------------ */
/* Combine                                                             */
/* ------------------------------------------------------------------ */

/* Combine gathers a token's K expert outputs and reduces them with the
 * router weights ([blog] "What This Does" and "Real-World Use").  The sum
 * is accumulated in binary32, one fused multiply-add per pick in k order
 * from zero, then rounded once to bf16:
 *   acc = 0; for k: acc = fmaf(w[k], float(eo[k][h]), acc); y[h] = bf16(acc).
 * eo is [n][K][H] bf16 (the K rows of each requested token, already
 * gathered by dst_row), w is [n][K], y is [n][H]. */
void oracle_combine_tokens(int K, int H, int64_t n, const float* w, const uint16_t* eo,
                           uint16_t* y)
{
    for (int64_t i = 0; i < n; ++i)
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k)
                acc = fmaf(w[i * K + k], oracle_bf16_to_f32(eo[(i * K + k) * H + h]), acc);
            y[i * H + h] = oracle_bf16_from_f32(acc);
        }
}

/* The same sum in binary64 without the final rounding: used by the tests
 * to bound the binary32 chain's rounding error. */
void oracle_combine_tokens_f64(int K, int H, int64_t n, const float* w, const uint16_t* eo,
                               double* y)
{
    for (int64_t i = 0; i < n; ++i)
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += (double)w[i * K + k] * (double)oracle_bf16_to_f32(eo[(i * K + k) * H + h]);
            y[i * H + h] = acc;
        }
}

/* ------------------------------------------------------------------ */
/* Side steps                                                          */
/* ------------------------------------------------------------------ */

/* Replica prefetch ([ainovat], the paragraph on duplicated experts being
 * fetched before expert computation; [blog] "How It Is Wired"): slot j of
 * rank r receives a bit copy of the home weights of expert
 * slot_expert[r][j].  home is [E][elems] of elem_bytes each; slots is
 * [R][B][elems]; unused slots are left untouched. */
void oracle_prefetch(int R, int B, int64_t elems, int elem_bytes, const int32_t* slot_expert,
                     const uint8_t* home, uint8_t* slots)
{
    int64_t row = elems * elem_bytes;
    for (int r = 0; r < R; ++r)
        for (int j = 0; j < B; ++j) {
            int e = slot_expert[r * B + j];
            if (e >= 0)
                memcpy(slots + ((int64_t)r * B + j) * row, home + (int64_t)e * row, (size_t)row);
        }
}

/* Replica gradient reduction ([ainovat], the paragraph on reducing the
 * duplicated experts' gradients back to their home ranks): for every
 * expert e that has replicas, dW[e] = (((dW[e] + g1) + g2) + ...) over its
 * replicas (r, j) in increasing r, then j, each addition one binary32
 * operation.  home is [E][elems] fp32, updated in place; slots is
 * [R][B][elems]. */
void oracle_grad_reduce(int R, int B, int E, int64_t elems, const int32_t* slot_expert,
                        float* home, const float* slots)
{
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < R; ++r)
            for (int j = 0; j < B; ++j)
                if (slot_expert[r * B + j] == e) {
                    const float* g = slots + ((int64_t)r * B + j) * elems;
                    float* d = home + (int64_t)e * elems;
                    for (int64_t i = 0; i < elems; ++i)
                        d[i] = d[i] + g[i];
                }
}

/* ------------------------------------------------------------------ */
/* Backward of combine and dispatch                                    */
/* ------------------------------------------------------------------ */

/* The layer's backward pass ([blog] "Real-World Use": the backward reduces
 * gradients; the chain rule through the two data movements):
 *  combine  y[t] = sum_k w[t,k] * eo[row(t,k)]  gives
 *    d_eo[row(t,k)] = bf16(w[t,k] * float(dy[t]))   (one binary32 product,
 *                                                     rounded once to bf16)
 *    d_w[t,k]       = sum_h float(dy[t,h]) * float(eo[row(t,k),h])
 *                     (here in binary64, the exact value up to the final
 *                      rounding; the GPU's binary32 sum is checked against
 *                      it within the recursive-summation bound)
 *  dispatch recv[row(t,k)] = x[t]  gives
 *    dx[t] = bf16(acc), acc = 0; acc = acc + float(d_recv[row(t,k)]) for
 *    k = 0..K-1, binary32 additions in k order.
 * dy, eo rows gathered per requested token: dy [n][H], eo [n][K][H]
 * (bf16 bits), w [n][K]; outputs d_eo [n][K][H] bf16 bits, d_w [n][K]
 * (double). */
void oracle_combine_backward_tokens(int K, int H, int64_t n, const float* w, const uint16_t* dy,
                                    const uint16_t* eo, uint16_t* d_eo, double* d_w)
{
    for (int64_t i = 0; i < n; ++i)
        for (int k = 0; k < K; ++k) {
            double dot = 0.0;
            for (int h = 0; h < H; ++h) {
                float g = oracle_bf16_to_f32(dy[i * H + h]);
                float v = oracle_bf16_to_f32(eo[(i * K + k) * H + h]);
                d_eo[(i * K + k) * H + h] = oracle_bf16_from_f32(w[i * K + k] * g);
                dot += (double)g * (double)v;
            }
            d_w[i * K + k] = dot;
        }
}

/* d_recv rows gathered per requested token: [n][K][H] bf16 bits -> dx [n][H]. */
void oracle_dispatch_backward_tokens(int K, int H, int64_t n, const uint16_t* d_recv, uint16_t* dx)
{
    for (int64_t i = 0; i < n; ++i)
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k)
                acc = acc + oracle_bf16_to_f32(d_recv[(i * K + k) * H + h]);
            dx[i * H + h] = oracle_bf16_from_f32(acc);
        }
}

/* ------------------------------------------------------------------ */
/* Grouped expert GEMM (the consumer of a plan)                        */
/* ------------------------------------------------------------------ */

/* double -> bfloat16 with one rounding, to nearest, ties to even, taken on
 * the double itself (no intermediate binary32).  bf16 keeps 8 significant
 * bits for exponents down to -126 and a fixed spacing of 2^-133 below.  A
 * magnitude a in [2^(e-1), 2^e) (frexp's e) lies on the grid of spacing
 * 2^(max(e, -125) - 8); a / spacing is rounded to an integer, ties to even,
 * and scaled back.  A result of 2^128 or more is infinity; NaN stays NaN. */
uint16_t oracle_bf16_from_f64(double v)
{
    if (isnan(v))
        return 0x7fc0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isinf(a))
        return sign | 0x7f80;
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);
    int q = (e > -125 ? e : -125) - 8;
    double r = ldexp(round_half_even(ldexp(a, -q)), q);
    if (r >= ldexp(1.0, 128))
        return sign | 0x7f80;
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)((u >> 16) & 0x7fffu);
}

void oracle_bf16_from_f64_array(const double* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_from_f64(in[i]);
}

/* The group of rank r that holds row `row` of the rank: the g with
 * cu_r[g-1] <= row < cu_r[g] (cu_seqlens are inclusive end offsets), or -1. */
int oracle_row_group(int E, int B, const int32_t* cu_r, int64_t row)
{
    for (int g = 0; g < E + B; ++g)
        if (row < cu_r[g])
            return g;
    return -1;
}

/* The framework's grouped GEMM over a plan ([ainovat], the framework-contract
 * paragraph: it reads the contiguous [E+B, H, H'] weight tensor and picks
 * each group's rows through cu_seqlens[E+B]).  A row of rank r in group g is
 * multiplied by row g of rank r's weight view: g < E is home expert g, g >= E
 * the replica in slot g - E.  For row i (the caller has resolved its matrix
 * to mat[i] in w, [nmat][H][Hp]):
 *   s[i][j] = sum_h x[i][h] * w[mat[i]][h][j]   in binary64, h ascending,
 *   y[i][j] = bf16(s[i][j])                     one rounding, ties to even.
 * A product of two bf16 values is exact in binary64, so s differs from the
 * exact sum by binary64 rounding only (at most H * 2^-53 * sum_h |x w|).
 * s and sabs (sum_h |x w|, for error bounds) are written when not NULL. */
void oracle_expert_gemm_rows(int H, int Hp, int64_t n, const uint16_t* x, const int32_t* mat,
                             const uint16_t* w, uint16_t* y, double* s, double* sabs)
{
    double* acc = (double*)malloc(sizeof(double) * (size_t)Hp * 2);
    if (!acc)
        return;
    double* aab = acc + Hp;
    for (int64_t i = 0; i < n; ++i) {
        const uint16_t* wm = w + (int64_t)mat[i] * H * Hp;
        for (int j = 0; j < Hp; ++j) {
            acc[j] = 0.0;
            aab[j] = 0.0;
        }
        for (int h = 0; h < H; ++h) {
            double xv = (double)oracle_bf16_to_f32(x[i * H + h]);
            const uint16_t* wr = wm + (int64_t)h * Hp;
            for (int j = 0; j < Hp; ++j) {
                double p = xv * (double)oracle_bf16_to_f32(wr[j]);
                acc[j] += p;
                aab[j] += fabs(p);
            }
        }
        for (int j = 0; j < Hp; ++j) {
            y[i * Hp + j] = oracle_bf16_from_f64(acc[j]);
            if (s)
                s[i * Hp + j] = acc[j];
            if (sabs)
                sabs[i * Hp + j] = aab[j];
        }
    }
    free(acc);
}
