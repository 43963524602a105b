// abi.cu -- the extern "C" entry points of libmoe_b200.so (include/moe.h):
// argument checks on the host, then the kernel launches on the caller's stream.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace moe {

cudaError_t launch_route_topk(const float *, int, int, int, int32_t *, float *, cudaStream_t);
cudaError_t launch_router_topk(const uint16_t *, const float *, int, int, int, int, float *, int32_t *, float *,
                               cudaStream_t);
int router_tok(int T, int H, int E);
size_t router_smem(int tok, int H, int E);
extern const size_t kRouterMaxSmemBytes;
cudaError_t launch_refresh_placement(const uint32_t *, int, int, int32_t *, int, int32_t *, int32_t *, cudaStream_t);
cudaError_t launch_promote_copies(const void *, void *, uint64_t, const int32_t *, const int32_t *, int, cudaStream_t);
cudaError_t launch_route_min_weight(int32_t *, float *, const int32_t *, int, int, int, float, cudaStream_t);
cudaError_t launch_permute(const int32_t *, int, int, int32_t *, int32_t *, int32_t *, int32_t *, uint32_t *,
                           cudaStream_t);
cudaError_t launch_expert_hits(const int32_t *, int64_t, int, uint32_t *, cudaStream_t);
bool route_permute_fused(int T, int k);
cudaError_t launch_route_permute(const float *, int, int, int, int32_t *, float *, int32_t *, int32_t *, int32_t *,
                                 int32_t *, uint32_t *, cudaStream_t);
cudaError_t launch_combine(const float *, const int32_t *, const float *, int, int, int, uint16_t *, cudaStream_t);
cudaError_t launch_quantize_int8(const uint16_t *, int, int, int8_t *, float *, cudaStream_t);
cudaError_t launch_quantize_int4(const uint16_t *, int, int, uint8_t *, uint16_t *, cudaStream_t);
size_t ffn_gemv_workspace(int T, int k, int I);
bool ffn_gemv_can_route(const LayerView &L, int T, int k);
bool ffn_gemv_can_combine(const LayerView &L, int T, int k);
cudaError_t launch_ffn_gemv_routed(const LayerView &L, const uint16_t *x, const float *logits, int k,
                                   uint32_t *hits, int32_t *ids, float *w, int32_t *counts, int32_t *offsets,
                                   int32_t *sorted_route, int32_t *route_pos, float *rows, void *ws, uint16_t *y,
                                   cudaStream_t s);
cudaError_t launch_ffn_gemv(const LayerView &, const uint16_t *, int, int, const int32_t *, const int32_t *,
                            const int32_t *, float *, void *, cudaStream_t);
size_t ffn_tc_workspace(int T, int k, int E, int H, int I);
bool ffn_tc_supports(int fmt, int H, int I, uint64_t stride);
cudaError_t launch_ffn_tc(const LayerView &, const uint16_t *, int, int, const int32_t *, const int32_t *,
                          const int32_t *, float *, void *, cudaStream_t);
cudaError_t tc_take_error(unsigned *code, unsigned *info);
cudaError_t gemv_take_error(unsigned *code, unsigned *info);

static thread_local char g_err[512];

moe_status set_error(moe_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

static moe_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return MOE_OK;
    return set_error(MOE_ERR_CUDA, "%s: %s (CUDA error %d)", what, cudaGetErrorString(e), (int)e);
}

#define CHECK_ARG(cond, ...)                                      \
    do {                                                          \
        if (!(cond)) return set_error(MOE_ERR_INVALID_ARG, __VA_ARGS__); \
    } while (0)

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

static moe_status check_shape(int E, int k, int H, int I) {
    CHECK_ARG(E >= 1 && E <= kMaxE, "E=%d outside [1, %d]", E, kMaxE);
    CHECK_ARG(k >= 1 && k <= E && k <= kMaxK, "k=%d outside [1, min(E, %d)]", k, kMaxK);
    CHECK_ARG(H >= 64 && H <= 16384 && H % 64 == 0, "H=%d must be a multiple of 64 in [64, 16384]", H);
    CHECK_ARG(I >= 64 && I <= 16384 && I % 64 == 0, "I=%d must be a multiple of 64 in [64, 16384]", I);
    return MOE_OK;
}

static moe_status check_tk(int T, int k) {
    CHECK_ARG(T >= 0, "T=%d is negative", T);
    CHECK_ARG((int64_t)T * k < (int64_t)1 << 31, "T*k=%lld does not fit in int32", (long long)T * k);
    return MOE_OK;
}

static moe_status layer_view(const moe_layer *l, LayerView *v) {
    CHECK_ARG(l != nullptr, "layer is NULL");
    CHECK_ARG(l->fmt == MOE_W_BF16 || l->fmt == MOE_W_INT8 || l->fmt == MOE_W_INT4, "unknown weight format %d",
              l->fmt);
    moe_status st = check_shape(l->E, 1, l->H, l->I);
    if (st != MOE_OK) return st;
    BlobOffsets o = blob_offsets(l->fmt, l->H, l->I);
    CHECK_ARG(l->home != nullptr, "layer home is NULL");
    CHECK_ARG(l->expert_bytes >= o.total && l->expert_bytes % 256 == 0,
              "expert_bytes=%llu must be >= %llu and a multiple of 256", (unsigned long long)l->expert_bytes,
              (unsigned long long)o.total);
    CHECK_ARG(aligned16(l->home) && aligned16(l->pool), "home/pool must be 16-byte aligned");
    CHECK_ARG(l->slot_table == nullptr || l->pool != nullptr, "a slot table needs a pool");
    CHECK_ARG(l->slot_table == nullptr || l->pool_slots >= 1, "a slot table needs pool_slots >= 1 (got %d)",
              l->pool_slots);
    v->fmt = l->fmt;
    v->E = l->E;
    v->H = l->H;
    v->I = l->I;
    v->slot_table = l->slot_table;
    v->pool = static_cast<const uint8_t *>(l->pool);
    v->home = static_cast<const uint8_t *>(l->home);
    v->stride = l->expert_bytes;
    v->pool_slots = l->slot_table ? l->pool_slots : 0;
    v->off = o;
    return MOE_OK;
}

static size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// The grouped FFN's layer and size checks, for the entry points that share them.
moe_status check_ffn_args(const moe_layer *layer, int T, int k) {
    LayerView v;
    moe_status st = layer_view(layer, &v);
    if (st != MOE_OK) return st;
    if ((st = check_shape(v.E, k, v.H, v.I)) != MOE_OK) return st;
    return check_tk(T, k);
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_version(void) { return "moe_b200 0.1 (sm_100a)"; }
const char *moe_last_error(void) { return g_err; }

size_t moe_expert_bytes(int32_t fmt, int32_t H, int32_t I) {
    if (fmt < 0 || fmt > 2 || H < 64 || I < 64 || H % 64 || I % 64) return 0;
    return (size_t)blob_offsets(fmt, H, I).total;
}

moe_status moe_blob_offsets(int32_t fmt, int32_t H, int32_t I, uint64_t *off) {
    CHECK_ARG(off != nullptr, "off is NULL");
    CHECK_ARG(fmt >= 0 && fmt <= 2, "unknown weight format %d", fmt);
    CHECK_ARG(H >= 64 && I >= 64 && H % 64 == 0 && I % 64 == 0, "H, I must be multiples of 64");
    BlobOffsets o = blob_offsets(fmt, H, I);
    off[0] = o.q13;
    off[1] = o.s13;
    off[2] = o.q2;
    off[3] = o.s2;
    return MOE_OK;
}

moe_status moe_route_topk(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *ids, float *w,
                          moe_stream_t stream) {
    moe_status st = check_shape(E, k, 64, 64);
    if (st != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(logits && ids && w, "moe_route_topk: NULL pointer");
    return cuda_status(launch_route_topk(logits, T, E, k, ids, w, (cudaStream_t)stream), "moe_route_topk launch");
}

moe_status moe_router_topk(const uint16_t *x, const float *w_router, int32_t T, int32_t H, int32_t E, int32_t k,
                           float *logits, int32_t *ids, float *w, moe_stream_t stream) {
    moe_status st = check_shape(E, k, 64, 64);
    if (st != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    CHECK_ARG(H >= 4 && H % 4 == 0, "H=%d must be a positive multiple of 4", H);
    CHECK_ARG(T <= 0 || (T + router_tok(T, H, E) - 1) / router_tok(T, H, E) <= 65535,
              "T=%d: more than 65535 token groups", T);
    CHECK_ARG((int64_t)T * E <= INT32_MAX, "T*E=%lld does not fit int32", (long long)T * E);
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && w_router && ids && w, "moe_router_topk: NULL pointer");
    CHECK_ARG(((uintptr_t)x & 7u) == 0 && aligned16(w_router), "x must be 8-byte and w_router 16-byte aligned");
    const size_t smem = router_smem(router_tok(T, H, E), H, E);
    if (smem > kRouterMaxSmemBytes)
        return set_error(MOE_ERR_UNSUPPORTED, "moe_router_topk: H=%d needs %zu bytes of shared memory per CTA (max %zu)",
                         H, smem, kRouterMaxSmemBytes);
    return cuda_status(launch_router_topk(x, w_router, T, H, E, k, logits, ids, w, (cudaStream_t)stream),
                       "moe_router_topk launch");
}

moe_status moe_route_min_weight(int32_t *ids, float *w, const int32_t *slot_table, int32_t T, int32_t k, int32_t E,
                                float min_weight, moe_stream_t stream) {
    moe_status st = check_shape(E, k, 64, 64);
    if (st != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    CHECK_ARG(min_weight == min_weight, "min_weight is NaN");
    if (T == 0 || !(min_weight < 1.0f)) return MOE_OK;
    CHECK_ARG(ids && w, "moe_route_min_weight: NULL pointer");
    return cuda_status(launch_route_min_weight(ids, w, slot_table, T, k, E, min_weight, (cudaStream_t)stream),
                       "moe_route_min_weight launch");
}

moe_status moe_permute(const int32_t *ids, int32_t T, int32_t k, int32_t E, int32_t *counts, int32_t *offsets,
                       int32_t *sorted_route, int32_t *route_pos, uint32_t *hits, moe_stream_t stream) {
    moe_status st = check_shape(E, k, 64, 64);
    if (st != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    if (T == 0) {
        // an empty grouping: zero counts and offsets where the caller gave them
        cudaError_t e = cudaSuccess;
        if (counts) e = cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), (cudaStream_t)stream);
        if (e == cudaSuccess && offsets)
            e = cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), (cudaStream_t)stream);
        return cuda_status(e, "moe_permute: clearing counts and offsets");
    }
    CHECK_ARG(ids && counts && offsets && sorted_route && route_pos, "moe_permute: NULL pointer");
    return cuda_status(launch_permute(ids, T * k, E, counts, offsets, sorted_route, route_pos, hits,
                                      (cudaStream_t)stream),
                       "moe_permute launch");
}

moe_status moe_route_permute(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *ids, float *w,
                             int32_t *counts, int32_t *offsets, int32_t *sorted_route, int32_t *route_pos,
                             uint32_t *hits, moe_stream_t stream) {
    moe_status st = check_shape(E, k, 64, 64);
    if (st != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    if (T == 0) return moe_permute(nullptr, 0, k, E, counts, offsets, sorted_route, route_pos, hits, stream);
    CHECK_ARG(logits && ids && w && counts && offsets && sorted_route && route_pos, "moe_route_permute: NULL pointer");
    cudaStream_t s = (cudaStream_t)stream;
    if (route_permute_fused(T, k))
        return cuda_status(launch_route_permute(logits, T, E, k, ids, w, counts, offsets, sorted_route, route_pos,
                                                hits, s),
                           "moe_route_permute launch");
    if ((st = cuda_status(launch_route_topk(logits, T, E, k, ids, w, s), "moe_route_permute: route")) != MOE_OK)
        return st;
    return cuda_status(launch_permute(ids, T * k, E, counts, offsets, sorted_route, route_pos, hits, s),
                       "moe_route_permute: permute");
}

moe_status moe_expert_hits(const int32_t *ids, int64_t n, int32_t E, uint32_t *hits, moe_stream_t stream) {
    CHECK_ARG(E >= 1 && E <= kMaxE, "E=%d outside [1, %d]", E, kMaxE);
    CHECK_ARG(n >= 0, "n=%lld is negative", (long long)n);
    if (n == 0) return MOE_OK;
    CHECK_ARG(ids && hits, "moe_expert_hits: NULL pointer");
    return cuda_status(launch_expert_hits(ids, n, E, hits, (cudaStream_t)stream), "moe_expert_hits launch");
}

size_t moe_grouped_ffn_workspace(const moe_layer *layer, int32_t T, int32_t k) {
    if (!layer || T < 0 || k < 1) return 0;
    size_t a = ffn_gemv_workspace(T, k, layer->I);
    size_t b = ffn_tc_workspace(T, k, layer->E, layer->H, layer->I);
    return align256(a > b ? a : b);
}

// The kernel path MOE_FFN_AUTO takes.  Measured on B200 (Gemma-shaped layer,
// top-8, FFN alone): the tensor-core kernels win from 3 tokens for bf16 (56.9 vs
// 61.9 us; at 2 tokens the GEMV: 44.4 vs 51.0), from 4 for int8 (63.2 vs 67.5)
// and from about 5 for int4 (6 tokens: 90.8 vs 98.1); one token at top-8 stays
// on the GEMV.
static int auto_path(const LayerView &v, int T, int k) {
    const int min_routes = v.fmt == MOE_W_BF16 ? 24 : (v.fmt == MOE_W_INT8 ? 32 : 40);
    return (T * k >= min_routes && ffn_tc_supports(v.fmt, v.H, v.I, v.stride)) ? MOE_FFN_TC : MOE_FFN_GEMV;
}

moe_status moe_grouped_ffn_path(const moe_layer *layer, const uint16_t *x, int32_t T, int32_t k,
                                const int32_t *counts, const int32_t *offsets, const int32_t *sorted_route,
                                float *rows, void *ws, size_t ws_bytes, int32_t path, moe_stream_t stream) {
    LayerView v;
    moe_status st = layer_view(layer, &v);
    if (st != MOE_OK) return st;
    if ((st = check_shape(v.E, k, v.H, v.I)) != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    CHECK_ARG(path == MOE_FFN_AUTO || path == MOE_FFN_GEMV || path == MOE_FFN_TC, "unknown path %d", path);
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && counts && offsets && sorted_route && rows && ws, "moe_grouped_ffn: NULL pointer");
    CHECK_ARG(aligned16(x) && aligned16(rows) && aligned16(ws), "x, rows and ws must be 16-byte aligned");
    const int use = path == MOE_FFN_AUTO ? auto_path(v, T, k) : path;
    if (use == MOE_FFN_TC && !ffn_tc_supports(v.fmt, v.H, v.I, v.stride))
        return set_error(MOE_ERR_UNSUPPORTED, "tensor-core path does not handle format %d at H=%d I=%d stride=%llu",
                         v.fmt, v.H, v.I, (unsigned long long)v.stride);
    // the workspace the chosen path needs (moe_grouped_ffn_workspace() covers both)
    const size_t need = align256(use == MOE_FFN_TC ? ffn_tc_workspace(T, k, v.E, v.H, v.I) : ffn_gemv_workspace(T, k, v.I));
    CHECK_ARG(ws_bytes >= need, "workspace %zu bytes < %zu needed", ws_bytes, need);
    if (use == MOE_FFN_TC) {
        return cuda_status(launch_ffn_tc(v, x, T, k, counts, offsets, sorted_route, rows, ws, (cudaStream_t)stream),
                           "moe_grouped_ffn (tensor-core) launch");
    }
    return cuda_status(launch_ffn_gemv(v, x, T, k, counts, offsets, sorted_route, rows, ws, (cudaStream_t)stream),
                       "moe_grouped_ffn (gemv) launch");
}

moe_status moe_grouped_ffn(const moe_layer *layer, const uint16_t *x, int32_t T, int32_t k, const int32_t *counts,
                           const int32_t *offsets, const int32_t *sorted_route, float *rows, void *ws,
                           size_t ws_bytes, moe_stream_t stream) {
    return moe_grouped_ffn_path(layer, x, T, k, counts, offsets, sorted_route, rows, ws, ws_bytes, MOE_FFN_AUTO,
                                stream);
}

// moe_route_ffn; with y non-null (moe_layer_forward) a one-token call whose
// FFN launches route the token also writes y in its second launch (the combine
// in the same launch, bit-identical to moe_combine), says so in *combined and
// leaves rows unwritten.
static moe_status route_ffn(const moe_layer *layer, const float *logits, const uint16_t *x, int32_t T, int32_t k,
                            uint32_t *hits, int32_t *ids, float *w, int32_t *counts, int32_t *offsets,
                            int32_t *sorted_route, int32_t *route_pos, float *rows, void *ws, size_t ws_bytes,
                            uint16_t *y, bool *combined, moe_stream_t stream) {
    if (combined) *combined = false;
    LayerView v;
    moe_status st = layer_view(layer, &v);
    if (st != MOE_OK) return st;
    if ((st = check_shape(v.E, k, v.H, v.I)) != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    if (T != 1 || auto_path(v, T, k) != MOE_FFN_GEMV || !ffn_gemv_can_route(v, T, k)) {
        // the two calls (moe_route_permute checks its own arguments)
        if ((st = moe_route_permute(logits, T, v.E, k, ids, w, counts, offsets, sorted_route, route_pos, hits,
                                    stream)) != MOE_OK)
            return st;
        return moe_grouped_ffn(layer, x, T, k, counts, offsets, sorted_route, rows, ws, ws_bytes, stream);
    }
    CHECK_ARG(logits && x && ids && w && counts && offsets && sorted_route && route_pos && rows && ws,
              "moe_route_ffn: NULL pointer");
    CHECK_ARG(aligned16(x) && aligned16(rows) && aligned16(ws), "x, rows and ws must be 16-byte aligned");
    const size_t need = align256(ffn_gemv_workspace(T, k, v.I));
    CHECK_ARG(ws_bytes >= need, "workspace %zu bytes < %zu needed", ws_bytes, need);
    const bool fuse = y != nullptr && ffn_gemv_can_combine(v, T, k);
    moe_status st2 = cuda_status(launch_ffn_gemv_routed(v, x, logits, k, hits, ids, w, counts, offsets, sorted_route,
                                                        route_pos, rows, ws, fuse ? y : nullptr, (cudaStream_t)stream),
                                 "moe_route_ffn launch");
    if (st2 == MOE_OK && combined) *combined = fuse;
    return st2;
}

moe_status moe_route_ffn(const moe_layer *layer, const float *logits, const uint16_t *x, int32_t T, int32_t k,
                         uint32_t *hits, int32_t *ids, float *w, int32_t *counts, int32_t *offsets,
                         int32_t *sorted_route, int32_t *route_pos, float *rows, void *ws, size_t ws_bytes,
                         moe_stream_t stream) {
    return route_ffn(layer, logits, x, T, k, hits, ids, w, counts, offsets, sorted_route, route_pos, rows, ws,
                     ws_bytes, nullptr, nullptr, stream);
}

moe_status moe_combine(const float *rows, const int32_t *route_pos, const float *w, int32_t T, int32_t k, int32_t H,
                       uint16_t *y, moe_stream_t stream) {
    CHECK_ARG(k >= 1 && k <= kMaxK, "k=%d outside [1, %d]", k, kMaxK);
    CHECK_ARG(H >= 64 && H <= 16384 && H % 64 == 0, "H=%d must be a multiple of 64 in [64, 16384]", H);
    moe_status st = check_tk(T, k);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(rows && route_pos && w && y, "moe_combine: NULL pointer");
    CHECK_ARG(aligned16(rows) && aligned16(y), "rows and y must be 16-byte aligned");
    return cuda_status(launch_combine(rows, route_pos, w, T, k, H, y, (cudaStream_t)stream), "moe_combine launch");
}

// forward workspace: ids | w | counts | offsets | sorted_route | route_pos | rows | ffn ws
struct FwdLayout {
    size_t ids, w, counts, offsets, sorted, pos, rows, ffn, total;
};

static FwdLayout fwd_layout(const moe_layer *layer, int T, int k) {
    FwdLayout f{};
    const size_t R = (size_t)T * k;
    size_t at = 0;
    f.ids = at; at += align256(R * 4);
    f.w = at; at += align256(R * 4);
    f.counts = at; at += align256((size_t)layer->E * 4);
    f.offsets = at; at += align256((size_t)(layer->E + 1) * 4);
    f.sorted = at; at += align256(R * 4);
    f.pos = at; at += align256(R * 4);
    f.rows = at; at += align256(R * (size_t)layer->H * 4);
    f.ffn = at; at += moe_grouped_ffn_workspace(layer, T, k);
    f.total = at;
    return f;
}

size_t moe_layer_forward_workspace(const moe_layer *layer, int32_t T, int32_t k) {
    if (!layer || T < 0 || k < 1) return 0;
    return fwd_layout(layer, T, k).total;
}

moe_status moe_layer_forward(const moe_layer *layer, const float *logits, const uint16_t *x, int32_t T, int32_t k,
                             uint32_t *hits, uint16_t *y, int32_t *ids_out, float *w_out, void *ws, size_t ws_bytes,
                             moe_stream_t stream) {
    LayerView v;
    moe_status st = layer_view(layer, &v);
    if (st != MOE_OK) return st;
    if ((st = check_shape(v.E, k, v.H, v.I)) != MOE_OK) return st;
    if ((st = check_tk(T, k)) != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(logits && x && y && ws, "moe_layer_forward: NULL pointer");
    CHECK_ARG(aligned16(ws), "ws must be 16-byte aligned");
    const FwdLayout f = fwd_layout(layer, T, k);
    CHECK_ARG(ws_bytes >= f.total, "workspace %zu bytes < %zu needed", ws_bytes, f.total);
    char *base = static_cast<char *>(ws);
    int32_t *ids = ids_out ? ids_out : reinterpret_cast<int32_t *>(base + f.ids);
    float *w = w_out ? w_out : reinterpret_cast<float *>(base + f.w);
    int32_t *counts = reinterpret_cast<int32_t *>(base + f.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(base + f.offsets);
    int32_t *sorted = reinterpret_cast<int32_t *>(base + f.sorted);
    int32_t *pos = reinterpret_cast<int32_t *>(base + f.pos);
    float *rows = reinterpret_cast<float *>(base + f.rows);
    CHECK_ARG(aligned16(y), "y must be 16-byte aligned");
    bool combined = false;
    if ((st = route_ffn(layer, logits, x, T, k, hits, ids, w, counts, offsets, sorted, pos, rows, base + f.ffn,
                        ws_bytes - f.ffn, y, &combined, stream)) != MOE_OK)
        return st;
    if (combined) return MOE_OK;  // one token: the FFN's second launch wrote y
    return moe_combine(rows, pos, w, T, k, v.H, y, stream);
}

moe_status moe_quantize_int8(const uint16_t *w, int32_t rows, int32_t K, int8_t *q, float *scale, moe_stream_t stream) {
    CHECK_ARG(rows >= 0 && K >= 1, "rows=%d K=%d", rows, K);
    if (rows == 0) return MOE_OK;
    CHECK_ARG(w && q && scale, "moe_quantize_int8: NULL pointer");
    return cuda_status(launch_quantize_int8(w, rows, K, q, scale, (cudaStream_t)stream), "moe_quantize_int8 launch");
}

moe_status moe_quantize_int4(const uint16_t *w, int32_t rows, int32_t K, uint8_t *q, uint16_t *scale,
                             moe_stream_t stream) {
    CHECK_ARG(rows >= 0 && K >= 64 && K % 64 == 0, "rows=%d K=%d (K must be a positive multiple of 64)", rows, K);
    if (rows == 0) return MOE_OK;
    CHECK_ARG(w && q && scale, "moe_quantize_int4: NULL pointer");
    CHECK_ARG(aligned16(w) && aligned16(q), "w and q must be 16-byte aligned");
    return cuda_status(launch_quantize_int4(w, rows, K, q, scale, (cudaStream_t)stream), "moe_quantize_int4 launch");
}

moe_status moe_pack_expert(int32_t fmt, const void *w13, const void *s13, const void *w2, const void *s2, int32_t H,
                           int32_t I, void *blob, moe_stream_t stream) {
    CHECK_ARG(fmt >= 0 && fmt <= 2, "unknown weight format %d", fmt);
    CHECK_ARG(H >= 64 && I >= 64 && H % 64 == 0 && I % 64 == 0, "H, I must be multiples of 64");
    CHECK_ARG(w13 && w2 && blob, "moe_pack_expert: NULL pointer");
    CHECK_ARG(fmt == MOE_W_BF16 || (s13 && s2), "moe_pack_expert: NULL scale pointer");
    const BlobOffsets o = blob_offsets(fmt, H, I);
    cudaStream_t s = (cudaStream_t)stream;
    char *b = static_cast<char *>(blob);
    cudaError_t e = cudaMemcpyAsync(b + o.q13, w13, o.s13 - o.q13, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && fmt != MOE_W_BF16) e = cudaMemcpyAsync(b + o.s13, s13, o.q2 - o.s13, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(b + o.q2, w2, o.s2 - o.q2, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && fmt != MOE_W_BF16) e = cudaMemcpyAsync(b + o.s2, s2, o.total - o.s2, cudaMemcpyDeviceToDevice, s);
    return cuda_status(e, "moe_pack_expert copy");
}

moe_status moe_take_device_errors(uint32_t *code, uint32_t *info) {
    CHECK_ARG(code && info, "moe_take_device_errors: NULL pointer");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e, "moe_take_device_errors: device synchronise");
    unsigned c = 0, i = 0, cg = 0, ig = 0;
    e = tc_take_error(&c, &i);
    if (e == cudaSuccess) e = gemv_take_error(&cg, &ig);
    if (e != cudaSuccess) return cuda_status(e, "moe_take_device_errors: read");
    if (c == 0) {  // the tensor-core word first, then the GEMV kernels' word
        c = cg;
        i = ig;
    }
    *code = c;
    *info = i;
    if (c >= 0x1000u && c < 0x2000u)
        return set_error(MOE_ERR_TIMEOUT, "a tensor-core kernel gave up waiting (warp %u, barrier word %#x)",
                         c & 0xFFFu, i);
    if (c == 0x2005u || c == 0x2006u)
        return set_error(MOE_ERR_CUDA, "slot %u of the slot table is past the pool; that expert's routes were skipped",
                         i);
    if (c) return set_error(MOE_ERR_CUDA, "a kernel failed an index check (site %u, value %u)", c & 0xFFFu, i);
    return MOE_OK;
}

moe_status moe_refresh_device(const uint32_t *hits, int32_t E, int32_t budget, int32_t *slot_table,
                              int32_t n_slots, int32_t *promo, int32_t *status, moe_stream_t stream) {
    CHECK_ARG(E >= 1 && E <= kMaxE, "E=%d outside [1, %d]", E, kMaxE);
    CHECK_ARG(n_slots >= 0 && n_slots <= kMaxE, "n_slots=%d outside [0, %d]", n_slots, kMaxE);
    CHECK_ARG(budget >= 0 && budget <= n_slots, "budget=%d outside [0, n_slots=%d]", budget, n_slots);
    CHECK_ARG(hits && slot_table && promo && status, "moe_refresh_device: NULL pointer");
    return cuda_status(launch_refresh_placement(hits, E, budget, slot_table, n_slots, promo, status,
                                                (cudaStream_t)stream),
                       "moe_refresh_device launch");
}

moe_status moe_promote_copies(const void *home, void *pool, uint64_t expert_bytes, const int32_t *promo,
                              const int32_t *status, int32_t max_promo, moe_stream_t stream) {
    CHECK_ARG(max_promo >= 0, "max_promo=%d is negative", max_promo);
    if (max_promo == 0) return MOE_OK;
    CHECK_ARG(home && pool && promo && status, "moe_promote_copies: NULL pointer");
    CHECK_ARG(expert_bytes > 0 && expert_bytes % 16 == 0, "expert_bytes=%llu must be a positive multiple of 16",
              (unsigned long long)expert_bytes);
    CHECK_ARG(aligned16(home) && aligned16(pool), "home and pool must be 16-byte aligned");
    return cuda_status(launch_promote_copies(home, pool, expert_bytes, promo, status, max_promo, (cudaStream_t)stream),
                       "moe_promote_copies launch");
}

moe_status moe_copy_to_slots(const void *home, void *pool, uint64_t expert_bytes, const int32_t *experts,
                             const int32_t *slots, int32_t n, moe_stream_t stream) {
    CHECK_ARG(n >= 0, "n=%d is negative", n);
    if (n == 0) return MOE_OK;
    CHECK_ARG(home && pool && experts && slots && expert_bytes > 0, "moe_copy_to_slots: NULL pointer or size");
    for (int i = 0; i < n; ++i) CHECK_ARG(experts[i] >= 0 && slots[i] >= 0, "negative expert or slot at %d", i);
    for (int i = 0; i < n; ++i) {
        cudaError_t e = cudaMemcpyAsync(static_cast<char *>(pool) + (size_t)slots[i] * expert_bytes,
                                        static_cast<const char *>(home) + (size_t)experts[i] * expert_bytes,
                                        expert_bytes, cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_status(e, "moe_copy_to_slots copy");
    }
    return MOE_OK;
}

}  // extern "C"
