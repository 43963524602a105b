/*
 * moe_oracle.h -- CPU oracle for the routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg use it.  It shares no source with the CUDA library.
 *
 * It is a plain, slow statement of what the layer computes, written from the
 * pages the method is described on:
 *   - prain README.md ("Expert formats" table: bf16 / int8 with an fp32 scale
 *     per row / int4 with a bf16 scale per 64 weights chosen by MSE clip;
 *     "Trading quality for speed": router weight shares per token);
 *   - rlx_runtime expert_pool.rs (count_hits, target_gpu_from_counts,
 *     apply_target_placement, should_refresh, gpu_expert_budget_from_vram and
 *     the tests module);
 *   - Winery-Strata remote_experts.cpp (RemoteExperts::begin: routes grouped
 *     by expert, token of a route = route index / k, rows in ascending route
 *     order inside a group; RemoteExperts::finish: rows copied back to their
 *     original route position; expert blobs reached through a cache slot).
 * Where the pages leave a step open, the reading taken is stated beside the
 * function that takes it.
 *
 * Every floating-point step that decides an integer or must be bit-exact
 * (routing weights, quantiser scales and codes) is done in fp32 exactly as
 * stated; the expert FFN and the combine are done in fp64 from exactly
 * dequantised weights.  Compile with -ffp-contract=off.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_BF16 = 0, ORACLE_INT8 = 1, ORACLE_INT4 = 2 };

/* One MoE layer's experts in host memory (host copies of the device blobs). */
typedef struct {
    int32_t fmt, E, H, I;
    const int32_t *slot_table;  /* [E] slot id or -1; NULL means every expert at home */
    const uint8_t *pool;        /* slot blobs, stride expert_bytes */
    const uint8_t *home;        /* E blobs, stride expert_bytes */
    size_t expert_bytes;
} oracle_layer;

void   oracle_set_threads(int n);
int    oracle_get_threads(void);

/* expert blob size and the byte offsets of its four pieces (w13, s13, w2, s2) */
size_t oracle_expert_bytes(int fmt, int H, int I);
void   oracle_blob_offsets(int fmt, int H, int I, size_t off[4]);

/* helpers exposed for the pins */
float  oracle_exp_p(float x);
double oracle_gelu_tanh(double x);
uint16_t oracle_bf16_rne(float f);

/* routing: ids [T,k] (descending logit, ties to the lower id), w [T,k] */
void oracle_route_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w);

/* [miss] min_weight partial routing: drop a token's lightest non-resident routes
 * once the kept share reaches min_weight; rescale the kept weights (in place) */
void oracle_route_min_weight(int32_t *ids, float *w, const int32_t *slot_table, int T, int k, int E,
                             float min_weight);

/* the step before the path: logits[t][e] = sum_h x[t][h] * w_router[e][h] in fp64 (x bf16 bits) */
void oracle_router_logits(const uint16_t *x, const float *w_router, int T, int H, int E, double *logits);

/* stable counting sort of the T*k routes by expert id */
void oracle_permute(const int32_t *ids, int T, int k, int E, int32_t *counts, int32_t *offsets,
                    int32_t *sorted_route, int32_t *route_pos);

/* hits[e] += number of ids equal to e; ids outside [0,E) are ignored */
void oracle_hits(const int32_t *ids, long n, int E, uint32_t *hits);
/* sum[e] = sum over the W rows of ring[W][E] (hits of the last W steps) */
void oracle_hits_window(const uint32_t *ring, int W, int E, uint32_t *sum);

/* quantisers: w bf16 bits [rows,K] */
void oracle_quantize_int8(const uint16_t *w, int rows, int K, int8_t *q, float *scale);
void oracle_quantize_int4(const uint16_t *w, int rows, int K, uint8_t *q, uint16_t *scale);
/* the reconstruction error of every int4 candidate of one 64-group, for pins */
void oracle_int4_candidates(const uint16_t *w64, float *s_out, double *err_out);

/* pack the pieces of one expert into its blob */
void oracle_pack_expert(int fmt, const void *w13, const void *s13, const void *w2, const void *s2,
                        int H, int I, uint8_t *blob);

/* dequantised weight of one expert (which = 13 for w13 [2I,H], 2 for w2 [H,I]) */
double oracle_weight(int fmt, const uint8_t *blob, int H, int I, int which, int row, int col);

/* blob of expert e through the slot table */
const uint8_t *oracle_resolve(const oracle_layer *L, int e);

/* one expert applied to one bf16 activation row: y = W2 (gelu_tanh(W13[:I] x) * (W13[I:] x)) */
void oracle_expert_ffn(const oracle_layer *L, int e, const uint16_t *x_row, double *y);

/* every route independently: rows[r] = FFN_{ids[r]}(x[r / k]); rows of invalid ids are zero */
void oracle_ffn_routes(const oracle_layer *L, const uint16_t *x, int T, int k, const int32_t *ids,
                       double *rows);
/* the same for a subset of routes (full-size sampled checks) */
void oracle_ffn_some_routes(const oracle_layer *L, const uint16_t *x, int k, const int32_t *ids,
                            const int32_t *which, int n_which, double *rows);

/* y[t] = sum_j w[t,j] * rows[t*k+j], summed in j order; invalid routes contribute nothing */
void oracle_combine(const double *rows, const int32_t *ids, const float *w, int T, int k, int E, int H,
                    double *y);

/* whole layer: route, then per-route FFN, then combine */
void oracle_moe_layer(const oracle_layer *L, const float *logits, const uint16_t *x, int T, int k,
                      int32_t *ids, float *w, double *rows, double *y);

/* placement (expert residency pool) */
int  oracle_refresh_target(const uint32_t *hits, int E, int budget, int32_t *target);
int  oracle_apply_placement(int32_t *slot_of, int E, int n_slots, const int32_t *target, int n_target,
                            int32_t *promote, int32_t *demote, int32_t *n_promote, int32_t *n_demote);
int  oracle_should_refresh(int offload_enabled, int mode_refresh, long step, int is_prefill_block,
                           long interval);
long oracle_budget_from_vram(long free_bytes, long reserve_bytes, long expert_bytes, long layers,
                             long max_per_layer, long E);

#ifdef __cplusplus
}
#endif
#endif
