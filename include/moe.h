/*
 * moe.h -- C ABI of the B200 (sm_100a) routed-expert MoE layer library
 *          (libmoe_b200.so).
 *
 * The layer computed here is the routed expert FFN of a mixture-of-experts
 * layer as the pages on expert offloading describe it:
 *   route   top-k experts per token from fp32 router logits, softmax weights
 *           renormalised over the k kept experts;
 *   permute group the T*k routes by expert (Winery-Strata remote_experts.cpp,
 *           RemoteExperts::begin) and count expert hits (rlx_runtime
 *           expert_pool.rs, count_hits);
 *   ffn     per expert, gated GELU-tanh FFN: w13 (gate rows [0,I), up rows
 *           [I,2I)) then w2, over bf16 / int8 (fp32 scale per row) / int4
 *           (bf16 scale per 64 weights) experts (prain README.md, "Expert
 *           formats"), each expert reached through a cache-slot table
 *           (remote_experts.cpp, slot_of / device_slot; prain README.md
 *           places experts in VRAM either pinned or in a cache slot);
 *   combine weighted sum of each token's k expert rows back in token order
 *           (remote_experts.cpp, RemoteExperts::finish).
 *
 * Conventions (every call):
 *  - Pointers named in a call are DEVICE memory owned by the caller unless the
 *    call says "host".  bf16 data is passed as raw 16-bit words (uint16_t).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Device
 *    calls are asynchronous on it; the library never synchronises.
 *    (moe_stream_t is void * and bf16 is uint16_t so that this header needs no
 *    CUDA headers; a cudaStream_t and __nv_bfloat16 data pass unchanged.)
 *  - The library never allocates device memory.  Calls that need scratch take
 *    a caller-owned workspace whose size the matching *_workspace() query gives.
 *  - Arguments are checked on the host before any launch.  A bad argument
 *    returns MOE_ERR_INVALID_ARG and launches nothing; a failed launch returns
 *    MOE_ERR_CUDA; a bounded device wait that gave up returns MOE_ERR_TIMEOUT.
 *    moe_last_error() then holds a one-line reason (thread-local).  This
 *    follows remote_experts.cpp, whose calls return false with an error string
 *    naming the failed step.
 *  - Limits: 1 <= E <= 1024 experts; 1 <= k <= min(E, 32); H and I multiples of
 *    64 in [64, 16384]; T >= 0 (T == 0 is a no-op); T*k < 2^31.  Device
 *    pointers to bf16/fp32 matrices and expert blobs must be 16-byte aligned.
 *  - Two calls that overlap on the GPU and write the same buffers race; the
 *    library adds no locking.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef void *moe_stream_t; /* cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_CUDA = 3,
    MOE_ERR_TIMEOUT = 4
} moe_status;

/* Expert weight formats (prain README.md, "Expert formats"). */
typedef enum { MOE_W_BF16 = 0, MOE_W_INT8 = 1, MOE_W_INT4 = 2 } moe_wfmt;

/* Kernel path for the grouped FFN.  AUTO takes the tensor-core kernels from
 * T*k >= 24 / 32 / 40 routes (bf16 / int8 / int4 weights), the GEMV kernels
 * below that (measured crossovers on B200 at the Gemma shape, top-8). */
typedef enum { MOE_FFN_AUTO = 0, MOE_FFN_GEMV = 1, MOE_FFN_TC = 2 } moe_ffn_path;

/*
 * One MoE layer's experts (host struct; the pointers in it are device memory).
 * Expert e is read from   pool + slot_table[e] * expert_bytes   when
 * slot_table[e] >= 0, else from   home + e * expert_bytes
 * (remote_experts.cpp: a cached expert is found by slot_of and read from its
 * device slot).  slot_table may be NULL (every expert read from home).
 * pool_slots is the number of blobs in pool (a pool may hold more slots than
 * the layer has experts: prain's 540 cache slots are shared by all layers).  It
 * is an addition to the pages' interface: the slot table lives on the device,
 * so the kernels need the pool's extent to bound what they read.  Required
 * (>= 1) with a slot table; ignored without one.  A slot_table entry at or past
 * pool_slots is refused on the device: the kernels skip that expert's routes
 * (their output rows are not written) and record the fault for
 * moe_take_device_errors() (MOE_ERR_CUDA, info = the bad slot id).
 * Blob layout of one expert, row-major, no padding:
 *   bf16: W13[2I][H] bf16 | W2[H][I] bf16
 *   int8: Q13[2I][H] i8 | S13[2I] f32 | Q2[H][I] i8 | S2[H] f32
 *   int4: Q13[2I][H/2] u8 | S13[2I][H/64] bf16 | Q2[H][I/2] u8 | S2[H][I/64] bf16
 * int8 weight = q * s (s per output row); int4 weight = (nibble - 8) * s (s per
 * 64 consecutive weights of a row); byte j of an int4 row holds weight 2j in
 * its low nibble and weight 2j+1 in its high nibble.
 */
typedef struct {
    int32_t fmt;               /* moe_wfmt */
    int32_t E, H, I;           /* experts, hidden, expert intermediate */
    const int32_t *slot_table; /* [E] slot id or -1, device; may be NULL */
    const void *pool;          /* slot blobs, stride expert_bytes, device; may be NULL if unused */
    const void *home;          /* E blobs, stride expert_bytes, device */
    uint64_t expert_bytes;     /* blob stride: >= moe_expert_bytes(), multiple of 256 */
    int32_t pool_slots;        /* blobs in pool (>= 1 when slot_table is set) */
} moe_layer;

/* Library version string and the last error of this thread ("" if none). */
MOE_API const char *moe_version(void);
MOE_API const char *moe_last_error(void);

/* Bytes of one expert blob (11894784 / 5964288 / 3159552 at H=2816, I=704:
 * the 11.34 / 5.69 / 3.01 MiB of the prain "Expert formats" table), or 0 for
 * bad arguments.  Host only. */
MOE_API size_t moe_expert_bytes(int32_t fmt, int32_t H, int32_t I);

/* Byte offsets of the four blob pieces {w13, s13, w2, s2} (host array of 4).
 * For bf16, s13 and s2 are empty and their offsets equal the next piece's. */
MOE_API moe_status moe_blob_offsets(int32_t fmt, int32_t H, int32_t I, uint64_t *off /* host [4] */);

/*
 * Top-k routing.  logits fp32 [T][E] -> ids int32 [T][k], w fp32 [T][k].
 * ids: the k largest logits of the token in descending order; equal logits go
 * to the lower expert id (the tie rule of expert_pool.rs,
 * target_gpu_from_counts); a NaN logit ranks below every number.
 * w: softmax then renormalisation over the kept experts, computed in fp32 as
 *   m = top logit; e_j = exp_p(l_j - m) (rank order); S = e_0 + ... + e_{k-1}
 *   (sequential); w_j = e_j / S (IEEE division),
 * where exp_p is the library's own fp32 exponential (Cody-Waite reduction with
 * ln2 split into LN2_HI = 0x3F317200 and LN2_LO = 0x35BFBE8E, rint of
 * x * 0x3FB8AA3B, a degree-7 Taylor polynomial in fma Horner form with fp32
 * coefficients 1/k!, and 2^n by exponent bits).  The result is bit-exact and
 * reproducible on any conforming fp32 implementation.  Weights are meaningful
 * for finite logits.
 */
MOE_API moe_status moe_route_topk(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *ids, float *w,
                          moe_stream_t stream);

/*
 * The step before the path, fused with it: the fp32 router projection (prain
 * README.md, "Experiments": the router is an fp32 GEMV) followed by
 * moe_route_topk's recipe, in one launch.
 *   logits[t][e] = sum_h x[t][h] * w_router[e][h]   (fp32 fused multiply-adds)
 * x bf16 [T][H] row-major (8-byte aligned, H a multiple of 4); w_router fp32
 * [E][H] row-major (16-byte aligned); logits fp32 [T][E] (output, nullable: pass
 * it to see the values the routing decided on); ids int32 [T][k] and w fp32
 * [T][k] exactly as moe_route_topk produces from those logits.  The logits are
 * fp32 sums (lane-strided partial sums over h, then a butterfly), so they match
 * an exact projection to rounding; ids and w are bit-exact functions of them.
 * One cluster of 8 CTAs per group of up to 16 tokens; each CTA stages its
 * group's rows in shared memory (MOE_ERR_UNSUPPORTED when even one row, 2*H
 * bytes plus the logits, exceeds 200 KiB).
 */
MOE_API moe_status moe_router_topk(const uint16_t *x, const float *w_router, int32_t T, int32_t H, int32_t E,
                                   int32_t k, float *logits, int32_t *ids, float *w, moe_stream_t stream);

/*
 * [miss] min_weight partial routing (prain README.md, "Trading quality for
 * speed"), applied in place to the output of moe_route_topk.  Per token, routes
 * are taken heaviest first with a running sum `kept` of the weights kept so far
 * (fp32, in order); a route whose expert has no cache slot (slot_table[e] < 0,
 * or slot_table NULL) is dropped once kept >= min_weight.  Dropped routes get
 * id -1 (moe_permute then leaves them out) and weight 0; every kept weight is
 * multiplied by total / kept (fp32, IEEE), so the kept weights again sum to the
 * token's total.  min_weight >= 1 is a no-op; a token with nothing kept (only
 * possible for min_weight <= 0) has all its routes dropped and contributes 0.
 * ids int32 [T][k], w fp32 [T][k], slot_table int32 [E] (device, nullable).
 */
MOE_API moe_status moe_route_min_weight(int32_t *ids, float *w, const int32_t *slot_table, int32_t T, int32_t k,
                                        int32_t E, float min_weight, moe_stream_t stream);

/*
 * Stable counting sort of the R = T*k routes by expert (remote_experts.cpp,
 * RemoteExperts::begin: a route r belongs to token r / k; inside an expert's
 * group the routes keep ascending r).  Groups are laid out by ascending
 * expert id.  Outputs: counts int32 [E]; offsets int32 [E+1] (exclusive scan,
 * offsets[E] = routes kept); sorted_route int32 [R] (flat route index of each
 * sorted row, -1 past offsets[E]); route_pos int32 [R] (sorted row of each
 * route, -1 for a dropped route).  Routes whose id is outside [0,E) are
 * dropped.  hits (uint32 [E], nullable) is incremented by counts (the
 * per-layer expert-hit histogram, expert_pool.rs count_hits).  One CTA; uses
 * 32*E*4 + 8 KiB of shared memory.  T == 0 is the empty grouping: counts and
 * offsets, where given, are set to zero (nothing else is touched).
 */
MOE_API moe_status moe_permute(const int32_t *ids, int32_t T, int32_t k, int32_t E, int32_t *counts,
                       int32_t *offsets, int32_t *sorted_route, int32_t *route_pos, uint32_t *hits,
                       moe_stream_t stream);

/*
 * moe_route_topk followed by moe_permute, with the same arguments and the
 * same results bit for bit (ids, w, counts, offsets, sorted_route, route_pos,
 * hits), in one launch when T <= 16: one CTA routes the batch's tokens (one
 * warp each) into shared memory and groups the routes there (a small decode
 * step then launches one kernel before the FFN instead of two; up to 64 KiB of
 * shared memory).  Larger batches run the two kernels.  T == 0 behaves as moe_permute's empty
 * grouping.
 */
MOE_API moe_status moe_route_permute(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *ids, float *w,
                                     int32_t *counts, int32_t *offsets, int32_t *sorted_route, int32_t *route_pos,
                                     uint32_t *hits, moe_stream_t stream);

/* hits[e] += number of the n ids equal to e; ids outside [0,E) are ignored
 * (expert_pool.rs, count_hits). */
MOE_API moe_status moe_expert_hits(const int32_t *ids, int64_t n, int32_t E, uint32_t *hits, moe_stream_t stream);

/*
 * Grouped gated FFN over the sorted routes.
 * x bf16 [T][H]; counts/offsets/sorted_route from moe_permute.  For every
 * sorted row s < offsets[E] of expert e (offsets[e] <= s < offsets[e+1]) with
 * token t = sorted_route[s] / k:
 *   g = W13_e x_t (fp32 accumulate);  h_i = gelu_tanh(g_i) * g_{I+i}
 *   (h rounded to bf16);  rows[s] = W2_e h  (fp32 accumulate)
 * with gelu_tanh(v) = 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))).
 * rows fp32 [T*k][H] in sorted order; rows past offsets[E] are not written.
 * ws: device workspace of at least moe_grouped_ffn_workspace() bytes.  The
 * query follows the scratch-size queries of remote_experts.cpp
 * (moe_hit_grouped_scratch_bytes / native_expert_scratch_bytes: the caller asks
 * how much scratch a grouped call needs, then owns it): here the larger of the
 * GEMV kernels' need (h, T*k*I*2 bytes) and the tensor-core kernels' (h plus x
 * gathered into sorted-route order, T*k*H*2 bytes), so one workspace serves
 * either path.
 * moe_grouped_ffn_path forces a kernel path (MOE_FFN_GEMV: split-K GEMV
 * kernels; MOE_FFN_TC: tcgen05 tensor-core kernels); MOE_ERR_UNSUPPORTED if
 * the forced path does not handle the format.  Asynchronous on `stream`; the
 * kernels are launched with programmatic stream serialization (each waits for
 * the previous kernel in the stream before reading its results), which is
 * transparent to callers and to CUDA graph capture.  A tensor-core kernel that
 * finds an inconsistent route block or gives up a bounded wait records it for
 * moe_take_device_errors() and skips the affected work.
 */
MOE_API size_t moe_grouped_ffn_workspace(const moe_layer *layer, int32_t T, int32_t k);
MOE_API moe_status moe_grouped_ffn(const moe_layer *layer, const uint16_t *x, int32_t T, int32_t k,
                           const int32_t *counts, const int32_t *offsets, const int32_t *sorted_route,
                           float *rows, void *ws, size_t ws_bytes, moe_stream_t stream);
MOE_API moe_status moe_grouped_ffn_path(const moe_layer *layer, const uint16_t *x, int32_t T, int32_t k,
                                const int32_t *counts, const int32_t *offsets,
                                const int32_t *sorted_route, float *rows, void *ws, size_t ws_bytes,
                                int32_t path, moe_stream_t stream);

/*
 * moe_route_permute followed by moe_grouped_ffn (AUTO path), with the arguments
 * of both (T, k and E from the layer; ws sized by moe_grouped_ffn_workspace())
 * and the same results: ids, w, counts, offsets, sorted_route, route_pos and hits
 * bit for bit, rows bit for bit as moe_grouped_ffn's.  For one token (T == 1,
 * E <= 128) where AUTO takes the GEMV kernels (k below 24 / 32 / 40 for bf16 /
 * int8 / int4) the routing runs inside the FFN's two launches
 * instead of a launch of its own: every CTA takes the token's top-k from the
 * logits with the routing kernels' code and groups the k routes itself, and
 * CTA 0 of the first launch writes the routing outputs (one launch fewer per
 * one-token layer step).  Otherwise the two calls run as they are.  The stages
 * of the pages' layer (prain README's route -> permute -> FFN; remote_experts.cpp
 * RemoteExperts::begin) are unchanged; only where they run differs.
 */
MOE_API moe_status moe_route_ffn(const moe_layer *layer, const float *logits, const uint16_t *x, int32_t T,
                                 int32_t k, uint32_t *hits, int32_t *ids, float *w, int32_t *counts,
                                 int32_t *offsets, int32_t *sorted_route, int32_t *route_pos, float *rows,
                                 void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Grouped FFN without a caller-provided workspace, for callers that cannot
 * allocate device memory (a plugin or serving runtime that passes the library
 * only its input and output buffers, or a loop that must never call
 * cudaMalloc).  The pages have no counterpart: this is a library convenience.
 * Same arguments as moe_grouped_ffn, minus ws, and the same rows up to the FFN
 * tolerance: this entry point always runs the split-K GEMV kernels
 * (MOE_FFN_GEMV), so its rows are bit-identical to moe_grouped_ffn's where
 * that call picks the GEMV kernels and within 1e-2 (max-relative) where it
 * picks the tensor cores; prefill-sized batches run slower than there.
 * Scratch: a fixed 16 MiB device array inside the library, reserved on every
 * GPU that loads it until the process exits.  The layer and sizes are checked
 * first, as in moe_grouped_ffn; then calls with T*k*I*2 > 16 MiB (the bf16
 * intermediate) are rejected with MOE_ERR_INVALID_ARG before any launch.  The
 * first call on a device looks up the array's device address (once per
 * device, that device current); make that first call before any stream
 * capture, and do not call this entry point again after a cudaDeviceReset in
 * the same process (the address it keeps would be stale).  Every call shares
 * the array and leaves its contents behind; calls that overlap on the GPU race
 * on it.  No allocation is made by this call.
 */
MOE_API moe_status moe_grouped_ffn_noalloc(const moe_layer *layer, const uint16_t *x, int32_t T, int32_t k,
                                           const int32_t *counts, const int32_t *offsets,
                                           const int32_t *sorted_route, float *rows, moe_stream_t stream);

/*
 * Weighted combine back to token order (remote_experts.cpp,
 * RemoteExperts::finish copies each row back to its route's position; the
 * weighting is the router's):  y[t] = sum_{j<k} w[t][j] * rows[route_pos[t*k+j]]
 * in fp32, summed in j order; routes with route_pos < 0 contribute nothing.
 * A pure gather: no atomics, deterministic.  y bf16 [T][H] (RNE).
 */
MOE_API moe_status moe_combine(const float *rows, const int32_t *route_pos, const float *w, int32_t T, int32_t k,
                       int32_t H, uint16_t *y, moe_stream_t stream);

/*
 * The whole layer in one call: route -> permute (+hits) -> grouped FFN ->
 * combine (moe_route_ffn, then moe_combine).  logits fp32 [T][E], x bf16
 * [T][H] -> y bf16 [T][H].  hits
 * (uint32 [E]), ids_out (int32 [T][k]) and w_out (fp32 [T][k]) are nullable.
 * ws: at least moe_layer_forward_workspace() bytes.  y must be 16-byte
 * aligned.  For one token where moe_route_ffn routes inside the FFN's launches
 * (the GEMV path, E <= 128), the combine also runs inside the FFN's second
 * launch: each of its CTAs takes whole output rows of all k routes, keeps those
 * rows in shared memory and sums them into y in route order with the same fp32
 * fma as moe_combine, so y is bit-identical to the separate calls; the call is
 * then two launches, and the rows region of ws is left unwritten.
 */
MOE_API size_t moe_layer_forward_workspace(const moe_layer *layer, int32_t T, int32_t k);
MOE_API moe_status moe_layer_forward(const moe_layer *layer, const float *logits, const uint16_t *x, int32_t T,
                             int32_t k, uint32_t *hits, uint16_t *y, int32_t *ids_out, float *w_out,
                             void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * int8 weight-only quantiser, fp32 scale per row (prain README.md, "Expert
 * formats"; the one-time GPU quantisation of the pack).  w bf16 [rows][K] ->
 * q int8 [rows][K], scale fp32 [rows]:  s = absmax / 127 (fp32);
 * q = clamp(rint(w / s), -127, 127), ties to even; an all-zero row gives
 * s = 0, q = 0.  Bit-exact.
 */
MOE_API moe_status moe_quantize_int8(const uint16_t *w, int32_t rows, int32_t K, int8_t *q, float *scale,
                             moe_stream_t stream);

/*
 * int4 weight-only quantiser, bf16 scale per 64 weights chosen by MSE clip
 * (prain README.md, "Expert formats").  w bf16 [rows][K] (K % 64 == 0) ->
 * q u8 [rows][K/2], scale bf16 [rows][K/64].  Per group of 64: for ratios
 * r_i = fp32((70 + 2i) / 100), i = 15 down to 0: s = bf16_rne(r_i * absmax / 7)
 * (fp32 multiply, fp32 divide); q = clamp(rint(w / s), -8, 7); error = the sum
 * of (w - q s)^2 in fp64 taken in weight order; a candidate replaces the best
 * only if its error is strictly smaller.  Stored as nibble q + 8.  Bit-exact.
 */
MOE_API moe_status moe_quantize_int4(const uint16_t *w, int32_t rows, int32_t K, uint8_t *q, uint16_t *scale,
                             moe_stream_t stream);

/* Pack one expert's pieces into its blob (layout above).  For bf16, w13 and w2
 * are bf16 and s13/s2 are ignored.  Device-to-device copies on `stream`. */
MOE_API moe_status moe_pack_expert(int32_t fmt, const void *w13, const void *s13, const void *w2, const void *s2,
                           int32_t H, int32_t I, void *blob, moe_stream_t stream);

/*
 * The placement refresh on the device (rlx_runtime expert_pool.rs,
 * target_gpu_from_counts then apply_target_placement): exactly what
 * moe_refresh_target followed by moe_apply_placement compute on the host, with
 * every array in device memory, so that a refresh needs no host round trip and
 * can be captured in a CUDA graph.  hits uint32 [E]; slot_table int32 [E] (the
 * layer's table, updated in place: demoted experts get -1, promoted experts
 * their new slot); promo int32 [2 * n_slots] receives (expert, slot) pairs in
 * promotion order; status int32 [3] receives {promotions, demotions, 0}, or
 * {0, 0, 1} when slot_table was inconsistent (a slot >= n_slots or held twice:
 * nothing is changed).  budget <= n_slots <= 1024, E <= 1024.  One CTA.
 */
MOE_API moe_status moe_refresh_device(const uint32_t *hits, int32_t E, int32_t budget, int32_t *slot_table,
                                      int32_t n_slots, int32_t *promo, int32_t *status, moe_stream_t stream);

/*
 * The promotion copies of a device refresh: for j < min(status[0], max_promo),
 * blob promo[2j] of home is copied into slot promo[2j+1] of pool (one kernel
 * reading the list from device memory; expert_bytes a multiple of 16, home and
 * pool 16-byte aligned).  Issue it on a second stream to overlap it with
 * compute; the layer's next forward must be ordered after it (an event).
 */
MOE_API moe_status moe_promote_copies(const void *home, void *pool, uint64_t expert_bytes, const int32_t *promo,
                                      const int32_t *status, int32_t max_promo, moe_stream_t stream);

/* Copy blobs of experts experts[i] from home into pool slot slots[i] (the
 * promotion copies of a placement refresh).  experts and slots are HOST
 * arrays of n entries.  Device-to-device copies on `stream`. */
MOE_API moe_status moe_copy_to_slots(const void *home, void *pool, uint64_t expert_bytes, const int32_t *experts,
                             const int32_t *slots, int32_t n, moe_stream_t stream);

/* Diagnostics: synchronise the device, then read and clear the first problem
 * the FFN kernels recorded since the last call (the tensor-core kernels' record
 * first, then the GEMV kernels': a slot past the pool).  *code = 0 and MOE_OK
 * if none; MOE_ERR_TIMEOUT if a bounded wait inside a kernel gave up (the
 * kernel then drained out without finishing its work); MOE_ERR_CUDA if an
 * index check failed (the access was skipped; *info holds the value). */
MOE_API moe_status moe_take_device_errors(uint32_t *code, uint32_t *info);

/* ---------------------------------------------------------------------------
 * Expert residency pool, host only (rlx_runtime expert_pool.rs).
 * ------------------------------------------------------------------------- */

/* Target residents (target_gpu_from_counts): experts with hits > 0 ranked by
 * hits descending, then id ascending; the first `budget`.  hits and target
 * are HOST arrays ([E] and at least [budget]); *n_target receives the count. */
MOE_API moe_status moe_refresh_target(const uint32_t *hits, int32_t E, int32_t budget, int32_t *target,
                              int32_t *n_target);

/*
 * Paired promote/demote (apply_target_placement) on a slot table.  expert_pool.rs
 * keeps a resident set and reports only counts; a slot table also needs to know
 * which slot each promoted expert takes, so this call adds n_slots (the pool's
 * extent) and returns the promoted and the demoted experts separately
 * (n_promote, n_demote; the page's paired swap makes n_demote <= n_promote,
 * with equality while the pool is full).
 * slot_of: HOST [E], slot id or -1, updated in place.  promote = target
 * experts not resident, in target order; demote = resident experts not in the
 * target, in ascending id, at most |promote| of them (the rest stay
 * resident).  The i-th promoted expert takes the i-th demoted expert's slot,
 * else the lowest free slot in [0, n_slots).  promote/demote: HOST, at least
 * [E].  Errors: MOE_ERR_INVALID_ARG if n_target > n_slots or no slot is free.
 */
MOE_API moe_status moe_apply_placement(int32_t *slot_of, int32_t E, int32_t n_slots, const int32_t *target,
                               int32_t n_target, int32_t *promote, int32_t *demote, int32_t *n_promote,
                               int32_t *n_demote);

/*
 * Windowed hit counts (host, pure CPU): sum[e] = sum over s < W of
 * ring[s][e], the hits of the last W steps kept as one histogram per step (a
 * variant of expert_pool.rs, which counts only the refreshing step's routes).
 * ring uint32 [W][E] and sum uint32 [E] are host memory.
 */
MOE_API moe_status moe_hits_window(const uint32_t *ring, int32_t W, int32_t E, uint32_t *sum);

/* should_refresh: 0 without offload; 1 in refresh mode or on a prefill block;
 * else 1 when step is a multiple of interval (interval < 1 counts as 1). */
MOE_API int32_t moe_should_refresh(int32_t offload_enabled, int32_t mode_refresh, int64_t step,
                           int32_t is_prefill_block, int64_t interval);

/* gpu_expert_budget_from_vram: (free - reserve) / (expert_bytes * layers),
 * capped by max_per_layer and E (max_per_layer capped by E if expert_bytes or
 * layers is 0). */
MOE_API int64_t moe_budget_from_vram(int64_t free_bytes, int64_t reserve_bytes, int64_t expert_bytes,
                             int64_t layers, int64_t max_per_layer, int64_t E);

/* ------------------------------------------------------------------------
 * Expert parallelism across GPUs.  Rank d of N holds local experts
 * [d*El, (d+1)*El) of a layer, El = E / N (E a multiple of N); one process per
 * GPU.  This is the multi-GPU form of the pages' remote-expert runtime
 * (Winery-Strata remote_experts.cpp: a secondary GPU owns a claimed subset of
 * the experts; RemoteExperts::begin stages the rows routed to it and
 * RemoteExperts::finish returns the compact result rows to their routes).
 * Per layer call, on every rank:
 *   1. moe_route_topk + moe_permute over all E experts.  The expert-sorted rows
 *      for rank d are the contiguous range [offsets[d*El], offsets[(d+1)*El]).
 *   2. moe_gather_rows(x, index = sorted_route, divisor = k) packs the routed
 *      tokens' rows in that order.
 *   3. An all-to-all of counts (El per rank pair) gives recv_counts [N][El];
 *      moe_ep_splits turns both into the row splits of the exchanges.
 *   4. An all-to-all of the packed rows (splits from step 3).
 *   5. The owner labels the received rows with moe_ep_recv_ids, groups them
 *      with moe_permute (k = 1, E = El), runs moe_grouped_ffn on its own El
 *      experts, and puts the fp32 result rows back in arrival order with
 *      moe_gather_rows(rows, index = route_pos, divisor = 1).
 *   6. The reverse all-to-all returns them; they land in the sender's sorted
 *      order, where one GPU's moe_grouped_ffn would have written them.
 *   7. moe_combine.
 * The exchanges are the caller's (NCCL all-to-all); nothing here waits on
 * another GPU.
 */

/*
 * dst row i = src row (index[i] / divisor) for i in [0, n), copied as
 * row_bytes bytes; rows whose index is negative or points at or past src_rows
 * are left untouched.  src [src_rows][row_bytes] and dst [n][row_bytes] are
 * device memory, 16-byte aligned; row_bytes a positive multiple of 16;
 * divisor >= 1.  Errors: MOE_ERR_INVALID_ARG (launches nothing).
 */
MOE_API moe_status moe_gather_rows(const void *src, int32_t src_rows, int32_t row_bytes, const int32_t *index,
                                   int32_t n, int32_t divisor, void *dst, moe_stream_t stream);

/*
 * Local expert of each received row: rows arrive grouped by source rank s and,
 * inside a source, by local expert e, recv_counts[s*El + e] rows each
 * (recv_counts int32 [N][El], device).  ids int32 [n] (device) gets e for
 * every row below the total of recv_counts, -1 for the rest.  N*El <= 1024.
 * Negative counts are read as 0.
 */
MOE_API moe_status moe_ep_recv_ids(const int32_t *recv_counts, int32_t N, int32_t El, int32_t *ids, int32_t n,
                                   moe_stream_t stream);

/*
 * Row splits of the two row exchanges (host, pure CPU).  counts: HOST [E], this
 * rank's routes per expert (moe_permute's counts); recv_counts: HOST [N][El],
 * what every source sends here per local expert.  send_rows[d] = rows this rank
 * sends to rank d = sum of counts over d's experts; recv_rows[s] = rows it
 * receives from s = sum of recv_counts[s].  The reverse exchange swaps the two.
 * Errors: MOE_ERR_INVALID_ARG if E is not a multiple of N, a count is negative
 * or a total does not fit in int32.
 */
MOE_API moe_status moe_ep_splits(const int32_t *counts, int32_t E, const int32_t *recv_counts, int32_t N,
                                 int32_t *send_rows, int32_t *recv_rows);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
