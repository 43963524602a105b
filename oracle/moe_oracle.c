/*
 * moe_oracle.c -- CPU oracle for the routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py.  The product path never links or calls it, and
 * it shares no source (no header, helper, table or constant) with the CUDA
 * library.  See moe_oracle.h for the pages each function follows.
 *
 * Build: gcc -std=c99 -O2 -ffp-contract=off -fopenmp -fPIC -shared
 * (-ffp-contract=off matters: every fp32 step below must round exactly once,
 * as written).  OpenMP only spreads independent routes / rows over threads;
 * no result depends on the thread count.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ threads */

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* --------------------------------------------------------------- bf16 / fp32 */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bf16_value(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* fp32 -> bf16, round to nearest, ties to even (NaN stays NaN). */
uint16_t oracle_bf16_rne(float f)
{
    uint32_t u = bits_from_f32(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------ expert blobs */
/*
 * Expert formats (prain README.md, "Expert formats"): bf16 as trained; int8
 * with an fp32 scale per row; int4 with a bf16 scale per 64 weights.  The blob
 * of one expert holds, in this order and with no padding,
 *   bf16: W13[2I,H] bf16 . W2[H,I] bf16
 *   int8: Q13[2I,H] i8 . S13[2I] f32 . Q2[H,I] i8 . S2[H] f32
 *   int4: Q13[2I,H/2] u8 . S13[2I,H/64] bf16 . Q2[H,I/2] u8 . S2[H,I/64] bf16
 * Rows [0,I) of W13 are the gate, rows [I,2I) the up projection (reading of
 * the name "w13" = w1 stacked on w3; the pages do not say).  At H=2816, I=704
 * the sizes are 11.34 / 5.69 / 3.01 MiB, the figures of that table.
 */
void oracle_blob_offsets(int fmt, int H, int I, size_t off[4])
{
    size_t h = (size_t)H, i = (size_t)I;
    if (fmt == ORACLE_BF16) {
        off[0] = 0;
        off[1] = 2 * i * h * 2;          /* no s13 */
        off[2] = 2 * i * h * 2;
        off[3] = off[2] + h * i * 2;     /* no s2 */
    } else if (fmt == ORACLE_INT8) {
        off[0] = 0;
        off[1] = 2 * i * h;
        off[2] = off[1] + 2 * i * 4;
        off[3] = off[2] + h * i;
    } else {
        off[0] = 0;
        off[1] = 2 * i * (h / 2);
        off[2] = off[1] + 2 * i * (h / 64) * 2;
        off[3] = off[2] + h * (i / 2);
    }
}

size_t oracle_expert_bytes(int fmt, int H, int I)
{
    size_t off[4];
    size_t h = (size_t)H, i = (size_t)I;
    oracle_blob_offsets(fmt, H, I, off);
    if (fmt == ORACLE_BF16) return off[3];
    if (fmt == ORACLE_INT8) return off[3] + h * 4;
    return off[3] + h * (i / 64) * 2;
}

void oracle_pack_expert(int fmt, const void *w13, const void *s13, const void *w2, const void *s2,
                        int H, int I, uint8_t *blob)
{
    size_t off[4];
    size_t h = (size_t)H, i = (size_t)I;
    oracle_blob_offsets(fmt, H, I, off);
    if (fmt == ORACLE_BF16) {
        memcpy(blob + off[0], w13, 2 * i * h * 2);
        memcpy(blob + off[2], w2, h * i * 2);
    } else if (fmt == ORACLE_INT8) {
        memcpy(blob + off[0], w13, 2 * i * h);
        memcpy(blob + off[1], s13, 2 * i * 4);
        memcpy(blob + off[2], w2, h * i);
        memcpy(blob + off[3], s2, h * 4);
    } else {
        memcpy(blob + off[0], w13, 2 * i * (h / 2));
        memcpy(blob + off[1], s13, 2 * i * (h / 64) * 2);
        memcpy(blob + off[2], w2, h * (i / 2));
        memcpy(blob + off[3], s2, h * (i / 64) * 2);
    }
}

/* Dequantised weight, exact in fp64: bf16 value; q * s (int8); (nibble-8) * s (int4).
 * q points at the codes of the matrix (K = its row length), s at its scales. */
static double dequant(int fmt, const uint8_t *q, const uint8_t *s, int K, int row, int col)
{
    if (fmt == ORACLE_BF16) {
        uint16_t b;
        memcpy(&b, q + ((size_t)row * K + col) * 2, 2);
        return (double)bf16_value(b);
    }
    if (fmt == ORACLE_INT8) {
        float sc;
        memcpy(&sc, s + (size_t)row * 4, 4);
        return (double)((const int8_t *)q)[(size_t)row * K + col] * (double)sc;
    }
    {
        uint16_t sb;
        uint8_t byte = q[(size_t)row * (K / 2) + col / 2];
        int nib = (col & 1) ? (byte >> 4) : (byte & 15);
        memcpy(&sb, s + ((size_t)row * (K / 64) + col / 64) * 2, 2);
        return (double)(nib - 8) * (double)bf16_value(sb);
    }
}

double oracle_weight(int fmt, const uint8_t *blob, int H, int I, int which, int row, int col)
{
    size_t off[4];
    oracle_blob_offsets(fmt, H, I, off);
    if (which == 13) return dequant(fmt, blob + off[0], blob + off[1], H, row, col);
    return dequant(fmt, blob + off[2], blob + off[3], I, row, col);
}

/* ------------------------------------------------------------------ routing */
/*
 * exp_p: the fp32 exponential both sides of the parity test compute, written
 * from the mathematics (Cody & Waite argument reduction, Taylor series):
 *   n = rint(x * LOG2E)                     (fp32 multiply, ties to even)
 *   r = fma(-n, LN2_HI, x); r = fma(-n, LN2_LO, r)
 *   p = 1 + r(1 + r(1/2! + r(1/3! + ... + r/7!)))   Horner, one fma per step
 *   result = p * 2^n  (two power-of-two multiplies when 2^n is subnormal)
 * LOG2E is log2(e) rounded to fp32; LN2_HI is ln 2 rounded to fp32 with its
 * low 8 mantissa bits cleared (so n * LN2_HI is exact for |n| < 256);
 * LN2_LO = ln 2 - LN2_HI rounded to fp32; c_k = 1/k! rounded to fp32.
 * |r| <= ln2/2, so the series error r^8/8! < 6e-9 relative: under 1 ulp.
 */
static const float LOG2E  = 0x1.715476p+0f;
static const float LN2_HI = 0x1.62e400p-1f;
static const float LN2_LO = 0x1.7f7d1cp-20f;

static float pow2i(int m) /* 2^m for -126 <= m <= 127 */
{
    return f32_from_bits((uint32_t)(m + 127) << 23);
}

float oracle_exp_p(float x)
{
    if (x != x) return x;
    if (x > 88.8f) return INFINITY;
    if (x < -104.0f) return 0.0f;
    float t = x * LOG2E;
    float n = rintf(t);
    float r = fmaf(-n, LN2_HI, x);
    r = fmaf(-n, LN2_LO, r);
    float p = 1.0f / 5040.0f;           /* 1/7! */
    p = fmaf(p, r, 1.0f / 720.0f);      /* 1/6! */
    p = fmaf(p, r, 1.0f / 120.0f);      /* 1/5! */
    p = fmaf(p, r, 1.0f / 24.0f);       /* 1/4! */
    p = fmaf(p, r, 1.0f / 6.0f);        /* 1/3! */
    p = fmaf(p, r, 0.5f);               /* 1/2! */
    p = fmaf(p, r, 1.0f);               /* 1/1! */
    p = fmaf(p, r, 1.0f);               /* 1/0! */
    int ni = (int)n;
    if (ni < -126) return (p * pow2i(ni + 100)) * pow2i(-100);
    if (ni > 127) return (p * pow2i(ni - 1)) * 2.0f;
    return p * pow2i(ni);
}

/* Ranking of experts for one token: larger logit first; equal logits go to
 * the lower expert id (the only tie rule on the pages: expert_pool.rs ranks
 * equal hit counts by the lower expert id in target_gpu_from_counts and its
 * test); a NaN logit ranks below every number. */
static int ranks_before(float la, int a, float lb, int b)
{
    int na = (la != la), nb = (lb != lb);
    if (na != nb) return nb;
    if (!na && la != lb) return la > lb;
    return a < b;
}

/*
 * Top-k routing, softmax then top-k renormalisation.  Renormalising the full
 * softmax over the k kept experts equals a softmax over the k kept logits
 * (the full denominator cancels), so the weights are computed in fp32 as
 *   m = l_0 (the top logit); e_j = exp_p(l_j - m), j in rank order;
 *   S = e_0 + e_1 + ... + e_{k-1} (in that order); w_j = e_j / S.
 */
void oracle_route_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w)
{
    int *order = (int *)malloc((size_t)E * sizeof(int));
    float *e = (float *)malloc((size_t)(k > 0 ? k : 1) * sizeof(float));
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (size_t)t * E;
        /* insertion sort of all E experts by rank */
        for (int i = 0; i < E; ++i) {
            int j = i;
            while (j > 0 && ranks_before(l[i], i, l[order[j - 1]], order[j - 1])) {
                order[j] = order[j - 1];
                --j;
            }
            order[j] = i;
        }
        float m = l[order[0]];
        float S = 0.0f;
        for (int j = 0; j < k; ++j) {
            ids[(size_t)t * k + j] = order[j];
            e[j] = oracle_exp_p(l[order[j]] - m);
        }
        for (int j = 0; j < k; ++j) S = S + e[j];
        for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = e[j] / S;
    }
    free(order);
    free(e);
}

/*
 * [miss] min_weight (prain README.md, "Trading quality for speed"): a
 * per-token threshold on the fraction of the router weight whose experts are
 * actually evaluated.  With the threshold below 1, light routes to experts held
 * outside VRAM may be left out once enough weight is covered, and the weights
 * that remain are enlarged so they again add up to the token's total.  Reading,
 * per token, in fp32:
 *   walk the routes in rank order (heaviest first) keeping a running sum `kept`
 *   of the weights kept so far; a route whose expert has no cache slot
 *   (slot_table[e] < 0, or no table) is dropped when kept >= min_weight,
 *   otherwise kept (kept = kept + w_j).  min_weight >= 1 changes nothing.
 *   Then total = sum of all k weights (in order) and every kept weight becomes
 *   w_j * (total / kept); a dropped route gets id -1 and weight 0.  If nothing is
 *   kept (min_weight <= 0 and no resident expert) every route is dropped.
 */
void oracle_route_min_weight(int32_t *ids, float *w, const int32_t *slot_table, int T, int k, int E,
                             float min_weight)
{
    if (!(min_weight < 1.0f)) return;
    for (int t = 0; t < T; ++t) {
        int32_t *id = ids + (size_t)t * k;
        float *wt = w + (size_t)t * k;
        float kept = 0.0f, total = 0.0f;
        char drop[64];
        for (int j = 0; j < k; ++j) {
            int e = id[j];
            int resident = slot_table != NULL && e >= 0 && e < E && slot_table[e] >= 0;
            drop[j] = (!resident && kept >= min_weight);
            if (!drop[j]) kept = kept + wt[j];
        }
        for (int j = 0; j < k; ++j) total = total + wt[j];
        float r = kept > 0.0f ? total / kept : 0.0f;
        for (int j = 0; j < k; ++j) {
            if (drop[j] || kept <= 0.0f) {
                id[j] = -1;
                wt[j] = 0.0f;
            } else {
                wt[j] = wt[j] * r;
            }
        }
    }
}

/*
 * The step before the path: the router projection (prain README.md,
 * "Experiments": the router is an fp32 GEMV over the hidden state).  Reading:
 * a plain linear map with no bias, logits[t][e] = sum_h x[t][h] * w_router[e][h],
 * x the layer's bf16 input row, w_router fp32 [E][H]; here every product and
 * the sum over h (in h order) are taken in fp64.  Top-k routing then runs on
 * the logits as oracle_route_topk states.
 */
void oracle_router_logits(const uint16_t *x, const float *w_router, int T, int H, int E, double *logits)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const uint16_t *xr = x + (size_t)t * H;
        for (int e = 0; e < E; ++e) {
            const float *wr = w_router + (size_t)e * H;
            double acc = 0.0;
            for (int h = 0; h < H; ++h) acc += (double)bf16_value(xr[h]) * (double)wr[h];
            logits[(size_t)t * E + e] = acc;
        }
    }
}

/* ------------------------------------------------------------------ permute */
/*
 * Group the R = T*k routes by expert (Winery-Strata remote_experts.cpp,
 * RemoteExperts::begin): a route r = t*k + j belongs to token r / k; inside a
 * group the rows keep ascending route order.  Groups are laid out in
 * ascending expert id (the page orders them by first appearance; id order
 * gives the same groups, relabelled, and is a plain exclusive scan).
 * Routes whose id is outside [0,E) join no group (the page skips them too):
 * route_pos = -1, and sorted_route is -1 past offsets[E].
 */
void oracle_permute(const int32_t *ids, int T, int k, int E, int32_t *counts, int32_t *offsets,
                    int32_t *sorted_route, int32_t *route_pos)
{
    long R = (long)T * k;
    int32_t *cursor = (int32_t *)calloc((size_t)E + 1, sizeof(int32_t));
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (long r = 0; r < R; ++r)
        if (ids[r] >= 0 && ids[r] < E) counts[ids[r]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (long r = 0; r < R; ++r) sorted_route[r] = -1;
    for (long r = 0; r < R; ++r) {
        int e = ids[r];
        if (e < 0 || e >= E) {
            route_pos[r] = -1;
            continue;
        }
        int pos = offsets[e] + cursor[e];
        cursor[e] += 1;
        sorted_route[pos] = (int32_t)r;
        route_pos[r] = pos;
    }
    free(cursor);
}

/* Expert-hit histogram (expert_pool.rs, count_hits): a bincount that ignores
 * ids outside [0,E); accumulated into hits. */
void oracle_hits(const int32_t *ids, long n, int E, uint32_t *hits)
{
    for (long i = 0; i < n; ++i)
        if (ids[i] >= 0 && ids[i] < E) hits[ids[i]] += 1u;
}

/*
 * Windowed hit counts, a variant of the refresh window (rlx_runtime
 * expert_pool.rs counts only the refreshing step's routes): the hits of the
 * last W steps, kept as W per-step histograms ring[W][E]; the window's count of
 * expert e is the sum of its W entries.
 */
void oracle_hits_window(const uint32_t *ring, int W, int E, uint32_t *sum)
{
    for (int e = 0; e < E; ++e) {
        uint32_t acc = 0;
        for (int s = 0; s < W; ++s) acc += ring[(size_t)s * E + e];
        sum[e] = acc;
    }
}

/* --------------------------------------------------------------- quantisers */
/*
 * int8, fp32 scale per row (prain README.md, "Expert formats").  Reading:
 * symmetric absmax, s = absmax / 127 (fp32), q = clamp(rint(w / s), -127, 127)
 * with ties to even; an all-zero row has s = 0 and q = 0.  A row is an output
 * row of the weight (K = its input width).
 */
void oracle_quantize_int8(const uint16_t *w, int rows, int K, int8_t *q, float *scale)
{
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const uint16_t *wr = w + (size_t)r * K;
        float amax = 0.0f;
        for (int c = 0; c < K; ++c) {
            float v = fabsf(bf16_value(wr[c]));
            if (v > amax) amax = v;
        }
        float s = amax / 127.0f;
        scale[r] = s;
        for (int c = 0; c < K; ++c) {
            int qi = 0;
            if (s != 0.0f) {
                float v = bf16_value(wr[c]) / s;
                qi = (int)rintf(v);
                if (qi > 127) qi = 127;
                if (qi < -127) qi = -127;
            }
            q[(size_t)r * K + c] = (int8_t)qi;
        }
    }
}

/*
 * int4, bf16 scale per 64 weights chosen by MSE clip (prain README.md,
 * "Expert formats"; the 16 ratios in [0.7, 1.0] come with the workload).
 * Reading, per group of 64 consecutive weights along K:
 *   absmax = max |w|;  r_i = fp32((70 + 2i) / 100), i = 15 down to 0;
 *   s_i = bf16_rne((r_i * absmax) / 7)          (fp32 multiply, fp32 divide)
 *   q   = clamp(rint(w / s_i), -8, 7)           (fp32 divide, ties to even)
 *   err = sum over the 64 weights, in order, of (w - q*s_i)^2 in fp64
 *   keep candidate i only if its err is strictly below the best so far
 *   (so ties keep the larger ratio, i.e. less clipping).  s_i = 0 gives q = 0.
 * Stored as nibble q+8; byte j of a row holds weight 2j in its low nibble and
 * weight 2j+1 in its high nibble.
 */
static void int4_candidate(const uint16_t *w64, float amax, int i, float *s_out, int8_t *q_out,
                           double *err_out)
{
    float r = (float)((double)(70 + 2 * i) / 100.0);
    float t = r * amax;
    t = t / 7.0f;
    float s = bf16_value(oracle_bf16_rne(t));
    double err = 0.0;
    for (int c = 0; c < 64; ++c) {
        float wv = bf16_value(w64[c]);
        int qi = 0;
        if (s != 0.0f) {
            float v = wv / s;
            qi = (int)rintf(v);
            if (qi > 7) qi = 7;
            if (qi < -8) qi = -8;
        }
        double d = (double)wv - (double)qi * (double)s;
        double d2 = d * d;
        err = err + d2;
        if (q_out) q_out[c] = (int8_t)qi;
    }
    *s_out = s;
    *err_out = err;
}

static float group_absmax(const uint16_t *w64)
{
    float amax = 0.0f;
    for (int c = 0; c < 64; ++c) {
        float v = fabsf(bf16_value(w64[c]));
        if (v > amax) amax = v;
    }
    return amax;
}

void oracle_int4_candidates(const uint16_t *w64, float *s_out, double *err_out)
{
    float amax = group_absmax(w64);
    for (int i = 0; i < 16; ++i) int4_candidate(w64, amax, i, &s_out[i], NULL, &err_out[i]);
}

void oracle_quantize_int4(const uint16_t *w, int rows, int K, uint8_t *q, uint16_t *scale)
{
    int G = K / 64;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        int8_t qc[64], qb[64];
        for (int g = 0; g < G; ++g) {
            const uint16_t *w64 = w + (size_t)r * K + (size_t)g * 64;
            float amax = group_absmax(w64);
            double best = INFINITY;
            float sbest = 0.0f;
            for (int i = 15; i >= 0; --i) {
                float s;
                double err;
                int4_candidate(w64, amax, i, &s, qc, &err);
                if (err < best) {
                    best = err;
                    sbest = s;
                    memcpy(qb, qc, 64);
                }
            }
            scale[(size_t)r * G + g] = oracle_bf16_rne(sbest);
            for (int j = 0; j < 32; ++j) {
                uint8_t lo = (uint8_t)(qb[2 * j] + 8), hi = (uint8_t)(qb[2 * j + 1] + 8);
                q[(size_t)r * (K / 2) + (size_t)g * 32 + j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* ---------------------------------------------------------------- expert FFN */

const uint8_t *oracle_resolve(const oracle_layer *L, int e)
{
    int s = L->slot_table ? L->slot_table[e] : -1;
    if (s >= 0) return L->pool + (size_t)s * L->expert_bytes;
    return L->home + (size_t)e * L->expert_bytes;
}

/* GELU with the tanh approximation:
 * gelu_tanh(v) = 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))). */
double oracle_gelu_tanh(double v)
{
    const double c = sqrt(2.0 / 3.14159265358979323846);
    return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

/*
 * One expert on one token, the plain definition, fp64 throughout from exactly
 * dequantised weights:  g = W13 x;  h_i = gelu_tanh(g_i) * g_{I+i};  y = W2 h.
 */
void oracle_expert_ffn(const oracle_layer *L, int e, const uint16_t *x_row, double *y)
{
    const int H = L->H, I = L->I, fmt = L->fmt;
    const uint8_t *blob = oracle_resolve(L, e);
    size_t off[4];
    double *x = (double *)malloc((size_t)H * sizeof(double));
    double *g = (double *)malloc((size_t)2 * I * sizeof(double));
    double *h = (double *)malloc((size_t)I * sizeof(double));
    oracle_blob_offsets(fmt, H, I, off);
    for (int c = 0; c < H; ++c) x[c] = (double)bf16_value(x_row[c]);
    for (int r = 0; r < 2 * I; ++r) {
        double acc = 0.0;
        for (int c = 0; c < H; ++c) acc += dequant(fmt, blob + off[0], blob + off[1], H, r, c) * x[c];
        g[r] = acc;
    }
    for (int i = 0; i < I; ++i) h[i] = oracle_gelu_tanh(g[i]) * g[I + i];
    for (int r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += dequant(fmt, blob + off[2], blob + off[3], I, r, i) * h[i];
        y[r] = acc;
    }
    free(x);
    free(g);
    free(h);
}

void oracle_ffn_some_routes(const oracle_layer *L, const uint16_t *x, int k, const int32_t *ids,
                            const int32_t *which, int n_which, double *rows)
{
    const int H = L->H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_which; ++n) {
        long r = which[n];
        int e = ids[r];
        double *out = rows + (size_t)n * H;
        if (e < 0 || e >= L->E) {
            for (int c = 0; c < H; ++c) out[c] = 0.0;
            continue;
        }
        oracle_expert_ffn(L, e, x + (size_t)(r / k) * H, out);
    }
}

void oracle_ffn_routes(const oracle_layer *L, const uint16_t *x, int T, int k, const int32_t *ids,
                       double *rows)
{
    long R = (long)T * k;
    int32_t *which = (int32_t *)malloc((size_t)(R > 0 ? R : 1) * sizeof(int32_t));
    for (long r = 0; r < R; ++r) which[r] = (int32_t)r;
    oracle_ffn_some_routes(L, x, k, ids, which, (int)R, rows);
    free(which);
}

/* ------------------------------------------------------------------ combine */
/*
 * Weighted combine back to token order (remote_experts.cpp, finish: each
 * row goes back to its original route position; the weighting is the
 * router's):  y[t] = sum_{j=0..k-1} w[t,j] * rows[t*k+j], in j order.
 */
void oracle_combine(const double *rows, const int32_t *ids, const float *w, int T, int k, int E, int H,
                    double *y)
{
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < H; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                long r = (long)t * k + j;
                if (ids[r] < 0 || ids[r] >= E) continue;
                acc += (double)w[r] * rows[(size_t)r * H + c];
            }
            y[(size_t)t * H + c] = acc;
        }
}

void oracle_moe_layer(const oracle_layer *L, const float *logits, const uint16_t *x, int T, int k,
                      int32_t *ids, float *w, double *rows, double *y)
{
    oracle_route_topk(logits, T, L->E, k, ids, w);
    oracle_ffn_routes(L, x, T, k, ids, rows);
    oracle_combine(rows, ids, w, T, k, L->E, L->H, y);
}

/* ---------------------------------------------------------------- placement */
/*
 * Expert residency pool (rlx_runtime expert_pool.rs).
 *
 * refresh_target (target_gpu_from_counts): experts with count > 0, ranked by
 * count descending then id ascending, the first `budget` of them.
 */
int oracle_refresh_target(const uint32_t *hits, int E, int budget, int32_t *target)
{
    int n = 0;
    char *taken = (char *)calloc((size_t)E + 1, 1);
    while (n < budget) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e] || hits[e] == 0) continue;
            if (best < 0 || hits[e] > hits[best]) best = e;
        }
        if (best < 0) break;
        taken[best] = 1;
        target[n++] = best;
    }
    free(taken);
    return n;
}

/*
 * apply_target_placement with cache slots.  promote = target experts not
 * resident, in target order; demote candidates = resident experts not in the
 * target, in ascending id (the page iterates a hash set, whose order is
 * unspecified); the first |promote| candidates are demoted, the rest stay
 * resident.  The i-th promoted expert takes the slot of the i-th demoted one,
 * else the lowest free slot.  Returns 0, or -1 if no slot is free.
 */
int oracle_apply_placement(int32_t *slot_of, int E, int n_slots, const int32_t *target, int n_target,
                           int32_t *promote, int32_t *demote, int32_t *n_promote, int32_t *n_demote)
{
    char *in_target = (char *)calloc((size_t)E + 1, 1);
    int np = 0, nd = 0, rc = 0;
    for (int i = 0; i < n_target; ++i) in_target[target[i]] = 1;
    for (int i = 0; i < n_target; ++i)
        if (slot_of[target[i]] < 0) promote[np++] = target[i];
    for (int e = 0; e < E && nd < np; ++e)
        if (slot_of[e] >= 0 && !in_target[e]) demote[nd++] = e;
    for (int i = 0; i < np; ++i) {
        int slot = -1;
        if (i < nd) {
            slot = slot_of[demote[i]];
            slot_of[demote[i]] = -1;
        } else {
            for (int s = 0; s < n_slots && slot < 0; ++s) {
                int used = 0;
                for (int e = 0; e < E; ++e)
                    if (slot_of[e] == s) used = 1;
                if (!used) slot = s;
            }
        }
        if (slot < 0) {
            rc = -1;
            break;
        }
        slot_of[promote[i]] = slot;
    }
    *n_promote = np;
    *n_demote = nd;
    free(in_target);
    return rc;
}

/* should_refresh: never without offload; always in Refresh mode or on a
 * prefill block; otherwise when step is a multiple of the interval
 * (EveryForward is interval 1). */
int oracle_should_refresh(int offload_enabled, int mode_refresh, long step, int is_prefill_block,
                          long interval)
{
    if (!offload_enabled) return 0;
    if (mode_refresh) return 1;
    if (is_prefill_block) return 1;
    if (interval < 1) interval = 1;
    return (step % interval) == 0;
}

/* gpu_expert_budget_from_vram: (free - reserve) / (expert_bytes * layers),
 * capped by the per-layer maximum and by E. */
long oracle_budget_from_vram(long free_bytes, long reserve_bytes, long expert_bytes, long layers,
                             long max_per_layer, long E)
{
    long cap = max_per_layer < E ? max_per_layer : E;
    if (expert_bytes == 0 || layers == 0) return cap;
    long usable = free_bytes > reserve_bytes ? free_bytes - reserve_bytes : 0;
    long per_layer = usable / (expert_bytes * layers);
    return per_layer < cap ? per_layer : cap;
}
