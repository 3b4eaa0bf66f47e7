/*
 * moe_oracle.c -- plain fp64 CPU oracle for the quantized MoE expert step.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The CUDA library
 * shares no code with it: no header, helper, table or constant generator.
 *
 * What it computes (the pages describe the step in words only; the formulas
 * below are the plain definitions, in the order of the flow the Strata
 * article gives in section 2 item 2: routing first, then the selected
 * experts -- those in VRAM at once, the others after they are moved in):
 *
 *   dequant   w = d * (q - 2^(b-1)), blocks of 32 codes with one fp16 scale
 *             (27B dense report: Q4_0 costs 0.5625 B per value; Strata
 *             article, summary table: the Q2_0 size)
 *   logits    l[t,e] = sum_h x[t,h] * Wr[e,h] (+ bias[e])
 *   top-k     the k experts that come first when sorted by (l desc, id asc)
 *             (Strata article, summary: 10 of 24,576 experts per token)
 *   gate      softmax over the k selected logits
 *   permute   stable counting sort of the (t, j) pairs by expert id
 *   expert    y = Wd (silu(Wg x) * (Wu x)), silu(g) = g / (1 + e^-g)
 *   combine   y[t] = sum_j w[t,j] * y_e(t,j)(x[t]) + y_shared(x[t])
 *   cache     frequency-driven residency with halving decay (Strata article,
 *             section 2 item 2; Janas-LLM page: repeated experts stay in RAM)
 *
 * Everything is evaluated in double precision in natural index order.
 * Readings where the pages are silent are listed in the design notes of the
 * repository; each is marked "reading" below.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BLOCK 32

enum { OR_F32 = 0, OR_BF16 = 1 };

/* ------------------------------------------------------------- threading */

/* OpenMP threads for the parallel loops that follow (n > 0); the arithmetic
 * of every function is the same at any thread count. */
void oracle_set_threads(int n)
{
    if (n > 0)
        omp_set_num_threads(n);
}

int oracle_max_threads(void)
{
    return omp_get_max_threads();
}

/* ---------------------------------------------------------------- formats */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_fp16_to_double(uint16_t h)
{
    int sign = h >> 15;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + frac), expo - 25);  /* (1 + frac/1024) * 2^(expo-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double load_value(const void *base, int dtype, size_t i)
{
    if (dtype == OR_BF16) {
        uint16_t b;
        memcpy(&b, (const uint8_t *)base + 2 * i, 2);
        return oracle_bf16_to_double(b);
    } else {
        float f;
        memcpy(&f, (const uint8_t *)base + 4 * i, 4);
        return (double)f;
    }
}

/* ------------------------------------------------------------- dequant */

/* Code q of element i (0..31) of one block of `bits`-bit codes. */
static int block_code(int bits, const uint8_t *blk, int i)
{
    if (bits == 4) {
        uint8_t byte = blk[i % 16];
        return i < 16 ? (byte & 0x0f) : (byte >> 4);
    } else {
        uint8_t byte = blk[i % 8];
        return (byte >> (2 * (i / 8))) & 0x3;
    }
}

/* Dequantise one block: out[i] = d * (q_i - 2^(b-1)). */
void oracle_dequant_block(int bits, const uint8_t *codes, uint16_t scale, double *out)
{
    double d = oracle_fp16_to_double(scale);
    int half = 1 << (bits - 1);
    for (int i = 0; i < ORACLE_BLOCK; ++i)
        out[i] = d * (double)(block_code(bits, codes, i) - half);
}

/* One packed matrix [rows][cols]: codes row-major by block, scales [rows][cols/32]. */
typedef struct {
    int bits, rows, cols;
    const uint8_t *codes;
    const uint8_t *scales;   /* fp16 bit patterns, little endian */
} qmat;

static double qmat_at(const qmat *m, int r, int c)
{
    int nb = m->cols / ORACLE_BLOCK;
    int blk = c / ORACLE_BLOCK;
    size_t bi = (size_t)r * nb + blk;
    const uint8_t *codes = m->codes + bi * (size_t)(4 * m->bits);
    uint16_t s;
    memcpy(&s, m->scales + 2 * bi, 2);
    int half = 1 << (m->bits - 1);
    return oracle_fp16_to_double(s) * (double)(block_code(m->bits, codes, c % ORACLE_BLOCK) - half);
}

/* Expert blob: codes Wg [I,H], Wu [I,H], Wd [H,I], then scales in the same order. */
typedef struct { qmat g, u, d; } expert_view;

static expert_view parse_blob(int bits, int H, int I, const uint8_t *blob)
{
    size_t cbytes = (size_t)I * H * bits / 8;       /* code bytes of one matrix */
    size_t sbytes = (size_t)I * H / ORACLE_BLOCK * 2; /* scale bytes of one matrix */
    const uint8_t *sc = blob + 3 * cbytes;
    expert_view v;
    v.g = (qmat){bits, I, H, blob, sc};
    v.u = (qmat){bits, I, H, blob + cbytes, sc + sbytes};
    v.d = (qmat){bits, H, I, blob + 2 * cbytes, sc + 2 * sbytes};
    return v;
}

size_t oracle_blob_bytes(int bits, int H, int I)
{
    return 3 * (size_t)I * H * bits / 8 + 3 * (size_t)I * H / ORACLE_BLOCK * 2;
}

/* Dense copies of the three dequantised matrices (Wg, Wu: [I][H]; Wd: [H][I]). */
void oracle_expert_weights(int bits, int H, int I, const uint8_t *blob,
                           double *Wg, double *Wu, double *Wd)
{
    expert_view v = parse_blob(bits, H, I, blob);
    for (int i = 0; i < I; ++i)
        for (int h = 0; h < H; ++h) {
            Wg[(size_t)i * H + h] = qmat_at(&v.g, i, h);
            Wu[(size_t)i * H + h] = qmat_at(&v.u, i, h);
        }
    for (int h = 0; h < H; ++h)
        for (int i = 0; i < I; ++i)
            Wd[(size_t)h * I + i] = qmat_at(&v.d, h, i);
}

/* -------------------------------------------------------------- expert */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* y = Wd (silu(Wg x) * (Wu x)) for one token; x [H], y [H].  h_out [I] optional. */
void oracle_expert_ffn(int bits, int H, int I, const uint8_t *blob,
                       const double *x, double *y, double *h_out)
{
    expert_view v = parse_blob(bits, H, I, blob);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            g += qmat_at(&v.g, i, c) * x[c];
            u += qmat_at(&v.u, i, c) * x[c];
        }
        h[i] = silu(g) * u;
    }
    for (int r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i)
            acc += qmat_at(&v.d, r, i) * h[i];
        y[r] = acc;
    }
    if (h_out)
        memcpy(h_out, h, sizeof(double) * (size_t)I);
    free(h);
}

/* n independent (expert, token) pairs: y[i] = FFN of blobs[i] applied to
 * x[i] (both [H] rows), one call of oracle_expert_ffn each, rows in
 * parallel.  Used to check chosen rows of a large step without running the
 * whole step. */
void oracle_expert_ffn_rows(int bits, int H, int I, int n, const uint8_t *const *blobs,
                            const double *x, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < (long)n; ++i)
        oracle_expert_ffn(bits, H, I, blobs[i], x + (size_t)i * H, y + (size_t)i * H, NULL);
}

/* -------------------------------------------------------------- router */

void oracle_router_logits(int T, int H, int E, const void *x, int x_dtype,
                          const void *w_router, int w_dtype, const float *bias,
                          double *logits)
{
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += load_value(x, x_dtype, (size_t)t * H + h) *
                     load_value(w_router, w_dtype, (size_t)e * H + h);
            if (bias)
                s += (double)bias[e];
            logits[(size_t)t * E + e] = s;
        }
}

/* Total order used for selection: larger logit first, equal logits by lower
 * id (reading: the tie rule of the benchmark spec), NaN below everything. */
typedef struct { double v; int32_t id; } scored;

static int rank_cmp(const void *pa, const void *pb)
{
    const scored *a = (const scored *)pa, *b = (const scored *)pb;
    int na = isnan(a->v), nb = isnan(b->v);
    if (na != nb)
        return na ? 1 : -1;
    if (!na) {
        if (a->v > b->v) return -1;
        if (a->v < b->v) return 1;
    }
    return (a->id < b->id) ? -1 : (a->id > b->id);
}

/* ids[t,j], w[t,j]: the first k experts of the sorted order and their gates
 * w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the k selected
 * (reading: softmax restricted to the selected experts, so gates sum to 1).
 * Returns 0, or -1 if a selected logit is NaN or +inf for some token. */
int oracle_topk(int T, int E, int k, const double *logits, int32_t *ids, double *w)
{
    int status = 0;
    scored *buf = (scored *)malloc(sizeof(scored) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            buf[e].v = logits[(size_t)t * E + e];
            buf[e].id = e;
        }
        qsort(buf, (size_t)E, sizeof(scored), rank_cmp);
        double lmax = buf[0].v, sum = 0.0;
        for (int j = 0; j < k; ++j) {
            ids[(size_t)t * k + j] = buf[j].id;
            if (isnan(buf[j].v) || (isinf(buf[j].v) && buf[j].v > 0))
                status = -1;
        }
        for (int j = 0; j < k; ++j)
            sum += exp(buf[j].v - lmax);
        for (int j = 0; j < k; ++j)
            w[(size_t)t * k + j] = exp(buf[j].v - lmax) / sum;
    }
    free(buf);
    return status;
}

/* Same selection on single-precision logits (widened exactly). */
int oracle_topk_f32(int T, int E, int k, const float *logits, int32_t *ids, double *w)
{
    double *l = (double *)malloc(sizeof(double) * (size_t)T * E);
    for (size_t i = 0; i < (size_t)T * E; ++i)
        l[i] = (double)logits[i];
    int st = oracle_topk(T, E, k, l, ids, w);
    free(l);
    return st;
}

/* ------------------------------------------------------------- permute */

/* Stable counting sort of the T*k (token, slot) pairs by expert id.
 * offsets [E+1]: exclusive prefix sum of per-expert counts.
 * perm_src [T*k]: row -> token.  perm_dst [T*k]: (t, j) -> row.
 * active [1 + E] (optional): count, then the experts with rows, ascending.
 * Returns 0, or -1 if an id is outside [0, E). */
int oracle_permute(int T, int k, int E, const int32_t *ids, int32_t *offsets,
                   int32_t *perm_src, int32_t *perm_dst, int32_t *active)
{
    int32_t *count = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    size_t n = (size_t)T * k;
    for (size_t p = 0; p < n; ++p) {
        if (ids[p] < 0 || ids[p] >= E) {
            free(count);
            free(cursor);
            return -1;
        }
        count[ids[p]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + count[e];
    for (int e = 0; e < E; ++e)
        cursor[e] = offsets[e];
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = ids[(size_t)t * k + j];
            int r = cursor[e]++;
            perm_src[r] = t;
            perm_dst[(size_t)t * k + j] = r;
        }
    if (active) {
        int na = 0;
        for (int e = 0; e < E; ++e)
            if (count[e] > 0)
                active[1 + na++] = e;
        active[0] = na;
    }
    free(count);
    free(cursor);
    return 0;
}

/* --------------------------------------------------------------- layer */

/* The whole step.  Either (w_router, w_dtype, bias) or logits_in [T,E] gives
 * the router logits.  blobs[e] points at expert e's blob; shared_blob may be
 * NULL.  Outputs: ids/w [T,k], offsets [E+1], perm_src/perm_dst [T*k],
 * y [T,H]; optional logits_out [T,E], y_perm [T*k,H], y_shared [T,H].
 * Returns 0, -1 for a non-finite selected logit, -2 for a bad id. */
int oracle_moe_layer(int bits, int T, int H, int I, int E, int k,
                     const void *x, int x_dtype,
                     const void *w_router, int w_dtype, const float *bias,
                     const float *logits_in,
                     const uint8_t *const *blobs, const uint8_t *shared_blob,
                     double *logits_out, int32_t *ids, double *w,
                     int32_t *offsets, int32_t *perm_src, int32_t *perm_dst,
                     double *y_perm, double *y_shared, double *y)
{
    size_t TE = (size_t)T * E, TK = (size_t)T * k, TH = (size_t)T * H;
    double *logits = (double *)malloc(sizeof(double) * (TE ? TE : 1));
    if (logits_in) {
        for (size_t i = 0; i < TE; ++i)
            logits[i] = (double)logits_in[i];
    } else {
        oracle_router_logits(T, H, E, x, x_dtype, w_router, w_dtype, bias, logits);
    }
    if (logits_out)
        memcpy(logits_out, logits, sizeof(double) * TE);
    int status = oracle_topk(T, E, k, logits, ids, w);
    free(logits);
    if (oracle_permute(T, k, E, ids, offsets, perm_src, perm_dst, NULL) != 0)
        return -2;

    double *xd = (double *)malloc(sizeof(double) * (TH ? TH : 1));
    for (size_t i = 0; i < TH; ++i)
        xd[i] = load_value(x, x_dtype, i);

    double *yp = y_perm ? y_perm : (double *)malloc(sizeof(double) * (TK * H > 0 ? TK * H : 1));
    /* row r belongs to the expert e with offsets[e] <= r < offsets[e+1] */
    int32_t *row_expert = (int32_t *)malloc(sizeof(int32_t) * (TK ? TK : 1));
    for (int e = 0; e < E; ++e)
        for (int r = offsets[e]; r < offsets[e + 1]; ++r)
            row_expert[r] = e;

#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < (long)TK; ++r)
        oracle_expert_ffn(bits, H, I, blobs[row_expert[r]], xd + (size_t)perm_src[r] * H,
                          yp + (size_t)r * H, NULL);

    double *ys = NULL;
    if (shared_blob) {
        ys = y_shared ? y_shared : (double *)malloc(sizeof(double) * TH);
#pragma omp parallel for schedule(dynamic, 1)
        for (long t = 0; t < (long)T; ++t)
            oracle_expert_ffn(bits, H, I, shared_blob, xd + (size_t)t * H, ys + (size_t)t * H, NULL);
    }

    /* combine, in slot order j = 0..k-1, then the shared expert (reading:
     * the shared expert enters with weight 1) */
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[(size_t)t * k + j] * yp[(size_t)perm_dst[(size_t)t * k + j] * H + h];
            if (ys)
                acc += ys[(size_t)t * H + h];
            y[(size_t)t * H + h] = acc;
        }

    if (ys && ys != y_shared)
        free(ys);
    if (yp != y_perm)
        free(yp);
    free(row_expert);
    free(xd);
    return status;
}

/* Combine alone: y[t] = sum_j w[t,j] y_perm[perm_dst[t,j]] (+ y_shared[t]). */
void oracle_combine(int T, int k, int H, const double *y_perm, const int32_t *perm_dst,
                    const double *w, const double *y_shared, double *y)
{
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[(size_t)t * k + j] * y_perm[(size_t)perm_dst[(size_t)t * k + j] * H + h];
            if (y_shared)
                acc += y_shared[(size_t)t * H + h];
            y[(size_t)t * H + h] = acc;
        }
}

/* --------------------------------------------------------- expert cache */

/* Replays a trace of per-step expert ids through the residency policy.
 *
 * Policy (Strata article, section 2 item 2: the most-called experts stay
 * resident, the rest are fetched on demand; reading for the details):
 *  - at the start of step s (s > 0, s % decay_period == 0) every counter is
 *    halved (integer floor);
 *  - for each id of the step, in the given order: counter += 1, last use = s;
 *    resident -> hit; otherwise a miss, which always enters the cache:
 *    the lowest free slot if any, else the slot of the resident expert that
 *    is not among this step's ids and is smallest in (counter, last use, id).
 *
 * With admit_min > 1 (reading: the zero-copy form of "only the others move
 * in" for experts that are rarely used), a miss whose counter after this use
 * is below admit_min does not enter: it is computed in place from host
 * memory (hit 3, slot -1, no victim) and nothing else changes beyond its
 * counter and last use.  admit_min 0 or 1 is the policy above;
 * oracle_cache_sim is that case.
 *
 * ids [steps][n].  Outputs per (step, j): slot, hit (1/0/3), victim (-1 none).
 * counts_out [n_experts] (optional): the counters after the last step.
 * Returns the number of misses (admitted or not), or -1 on invalid input (id
 * out of range, repeated id within a step, n > capacity). */
long oracle_cache_sim_admit(int n_experts, int capacity, int decay_period, int admit_min, int steps,
                            int n, const int32_t *ids, int32_t *slot_out, int8_t *hit_out,
                            int32_t *victim_out, int64_t *counts_out)
{
    if (n > capacity || capacity <= 0)
        return -1;
    int32_t *slot_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_experts);
    int32_t *expert_in = (int32_t *)malloc(sizeof(int32_t) * (size_t)capacity);
    int64_t *cnt = (int64_t *)calloc((size_t)n_experts, sizeof(int64_t));
    int64_t *last = (int64_t *)malloc(sizeof(int64_t) * (size_t)n_experts);
    for (int e = 0; e < n_experts; ++e) {
        slot_of[e] = -1;
        last[e] = -1;
    }
    for (int s = 0; s < capacity; ++s)
        expert_in[s] = -1;
    long misses = 0;
    for (int s = 0; s < steps; ++s) {
        const int32_t *step_ids = ids + (size_t)s * n;
        for (int j = 0; j < n; ++j) {
            if (step_ids[j] < 0 || step_ids[j] >= n_experts)
                goto bad;
            for (int i = 0; i < j; ++i)
                if (step_ids[i] == step_ids[j])
                    goto bad;
        }
        if (decay_period > 0 && s > 0 && s % decay_period == 0)
            for (int e = 0; e < n_experts; ++e)
                cnt[e] /= 2;
        for (int j = 0; j < n; ++j) {
            int e = step_ids[j];
            size_t o = (size_t)s * n + j;
            cnt[e] += 1;
            last[e] = s;
            victim_out[o] = -1;
            if (slot_of[e] >= 0) {
                hit_out[o] = 1;
                slot_out[o] = slot_of[e];
                continue;
            }
            misses++;
            if (admit_min > 1 && cnt[e] < admit_min) {
                hit_out[o] = 3;                      /* computed in place, not admitted */
                slot_out[o] = -1;
                continue;
            }
            hit_out[o] = 0;
            int slot = -1;
            for (int sl = 0; sl < capacity; ++sl)
                if (expert_in[sl] < 0) {
                    slot = sl;
                    break;
                }
            if (slot < 0) {
                int best = -1;
                for (int sl = 0; sl < capacity; ++sl) {
                    int c = expert_in[sl];
                    int in_step = 0;
                    for (int i = 0; i < n; ++i)
                        if (step_ids[i] == c)
                            in_step = 1;
                    if (in_step)
                        continue;
                    if (best < 0 || cnt[c] < cnt[best] ||
                        (cnt[c] == cnt[best] && (last[c] < last[best] ||
                                                 (last[c] == last[best] && c < best))))
                        best = c;
                }
                slot = slot_of[best];
                slot_of[best] = -1;
                victim_out[o] = best;
            }
            expert_in[slot] = e;
            slot_of[e] = slot;
            slot_out[o] = slot;
        }
    }
    if (counts_out)
        memcpy(counts_out, cnt, sizeof(int64_t) * (size_t)n_experts);
    free(slot_of);
    free(expert_in);
    free(cnt);
    free(last);
    return misses;
bad:
    free(slot_of);
    free(expert_in);
    free(cnt);
    free(last);
    return -1;
}

long oracle_cache_sim(int n_experts, int capacity, int decay_period, int steps, int n,
                      const int32_t *ids, int32_t *slot_out, int8_t *hit_out,
                      int32_t *victim_out, int64_t *counts_out)
{
    return oracle_cache_sim_admit(n_experts, capacity, decay_period, 0, steps, n, ids, slot_out, hit_out,
                                  victim_out, counts_out);
}

/* The same policy with prefetch (reading: the pages keep hot experts resident
 * and move the rest in; loading the next layer's likely experts ahead of
 * their use is the cross-layer form of that).  After the stage of step s, the
 * ids pf_ids[s][0..npf) (-1 = none) are prefetched in order:
 *  - a resident id (or -1): nothing happens (pf_slot = pf_victim = -1);
 *  - otherwise the id enters the lowest free slot, else the slot of the
 *    resident expert smallest in (counter, last use, id) that is neither one
 *    of step s's ids nor on the prefetch list (the list names the experts
 *    expected next: none of them is evicted for another); if no such expert
 *    exists the id is skipped (pf_slot = -1);
 *  - a prefetch is not a use: counters and last uses do not change.
 * Stage outputs as oracle_cache_sim; pf_slot_out / pf_victim_out [steps][npf].
 * *pf_admitted_out (optional) = the number of ids prefetched into a slot.
 * Returns the stage misses, or -1 on invalid input. */
long oracle_cache_sim_prefetch(int n_experts, int capacity, int decay_period, int steps, int n,
                               const int32_t *ids, int npf, const int32_t *pf_ids,
                               int32_t *slot_out, int8_t *hit_out, int32_t *victim_out,
                               int32_t *pf_slot_out, int32_t *pf_victim_out,
                               int64_t *counts_out, long *pf_admitted_out)
{
    if (n > capacity || capacity <= 0 || npf < 0)
        return -1;
    int32_t *slot_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_experts);
    int32_t *expert_in = (int32_t *)malloc(sizeof(int32_t) * (size_t)capacity);
    int64_t *cnt = (int64_t *)calloc((size_t)n_experts, sizeof(int64_t));
    int64_t *last = (int64_t *)malloc(sizeof(int64_t) * (size_t)n_experts);
    int8_t *guard = (int8_t *)calloc((size_t)n_experts, 1);   /* protected from eviction */
    for (int e = 0; e < n_experts; ++e) {
        slot_of[e] = -1;
        last[e] = -1;
    }
    for (int s = 0; s < capacity; ++s)
        expert_in[s] = -1;
    long misses = 0, admitted = 0;
    for (int s = 0; s < steps; ++s) {
        const int32_t *step_ids = ids + (size_t)s * n;
        for (int j = 0; j < n; ++j) {
            if (step_ids[j] < 0 || step_ids[j] >= n_experts)
                goto bad;
            for (int i = 0; i < j; ++i)
                if (step_ids[i] == step_ids[j])
                    goto bad;
        }
        if (decay_period > 0 && s > 0 && s % decay_period == 0)
            for (int e = 0; e < n_experts; ++e)
                cnt[e] /= 2;
        for (int j = 0; j < n; ++j)
            guard[step_ids[j]] = 1;
        /* stage: the policy of oracle_cache_sim */
        for (int j = 0; j < n; ++j) {
            int e = step_ids[j];
            size_t o = (size_t)s * n + j;
            cnt[e] += 1;
            last[e] = s;
            victim_out[o] = -1;
            if (slot_of[e] >= 0) {
                hit_out[o] = 1;
                slot_out[o] = slot_of[e];
                continue;
            }
            hit_out[o] = 0;
            misses++;
            int slot = -1;
            for (int sl = 0; sl < capacity; ++sl)
                if (expert_in[sl] < 0) {
                    slot = sl;
                    break;
                }
            if (slot < 0) {
                int best = -1;
                for (int sl = 0; sl < capacity; ++sl) {
                    int c = expert_in[sl];
                    if (guard[c])
                        continue;
                    if (best < 0 || cnt[c] < cnt[best] ||
                        (cnt[c] == cnt[best] && (last[c] < last[best] ||
                                                 (last[c] == last[best] && c < best))))
                        best = c;
                }
                slot = slot_of[best];
                slot_of[best] = -1;
                victim_out[o] = best;
            }
            expert_in[slot] = e;
            slot_of[e] = slot;
            slot_out[o] = slot;
        }
        /* prefetch after the stage: the whole list is protected */
        for (int j = 0; j < npf; ++j) {
            int e = pf_ids[(size_t)s * npf + j];
            if (e < -1 || e >= n_experts)
                goto bad;
            if (e >= 0)
                guard[e] = 1;
        }
        for (int j = 0; j < npf; ++j) {
            size_t o = (size_t)s * npf + j;
            int e = pf_ids[o];
            pf_slot_out[o] = -1;
            pf_victim_out[o] = -1;
            if (e < -1 || e >= n_experts)
                goto bad;
            if (e < 0 || slot_of[e] >= 0)
                continue;
            int slot = -1;
            for (int sl = 0; sl < capacity; ++sl)
                if (expert_in[sl] < 0) {
                    slot = sl;
                    break;
                }
            if (slot < 0) {
                int best = -1;
                for (int sl = 0; sl < capacity; ++sl) {
                    int c = expert_in[sl];
                    if (guard[c])
                        continue;
                    if (best < 0 || cnt[c] < cnt[best] ||
                        (cnt[c] == cnt[best] && (last[c] < last[best] ||
                                                 (last[c] == last[best] && c < best))))
                        best = c;
                }
                if (best < 0)
                    continue;                        /* everything resident is protected */
                slot = slot_of[best];
                slot_of[best] = -1;
                pf_victim_out[o] = best;
            }
            expert_in[slot] = e;
            slot_of[e] = slot;
            pf_slot_out[o] = slot;
            admitted++;
        }
        for (int j = 0; j < n; ++j)
            guard[step_ids[j]] = 0;
        for (int j = 0; j < npf; ++j)
            if (pf_ids[(size_t)s * npf + j] >= 0)
                guard[pf_ids[(size_t)s * npf + j]] = 0;
    }
    if (counts_out)
        memcpy(counts_out, cnt, sizeof(int64_t) * (size_t)n_experts);
    if (pf_admitted_out)
        *pf_admitted_out = admitted;
    free(slot_of);
    free(expert_in);
    free(cnt);
    free(last);
    free(guard);
    return misses;
bad:
    free(slot_of);
    free(expert_in);
    free(cnt);
    free(last);
    free(guard);
    return -1;
}
