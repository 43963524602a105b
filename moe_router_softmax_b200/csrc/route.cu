// route.cu -- top-k routing of fp32 router logits (one warp per token).
//
// ids: the k largest logits in descending order, equal logits to the lower
// expert id (expert_pool.rs ranks equal counts by the lower id), NaN last.
// w: softmax renormalised over the k kept experts, which equals a softmax over
// the kept logits (the full denominator cancels).  All fp32 steps are written
// with explicit round-to-nearest intrinsics so that no multiply-add is fused
// behind our back: the result is bit-for-bit the recipe of moe_route_topk.
#include <cooperative_groups.h>

#include "common.cuh"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace moe {
using topk::exp_p;
using topk::rank_key;
using topk::route_token_warp;

// dynamic shared memory of one router CTA: TOK x EB fp32 logits and TOK x H
// bf16 activation rows; TOK = tokens per cluster: the batch itself up to 4,
// 8 for decode batches, 16 past 64 tokens (fewer re-reads of the router
// weights), halved while the rows do not fit
constexpr size_t kRouterMaxSmem = 200 * 1024;
extern const size_t kRouterMaxSmemBytes = kRouterMaxSmem;
size_t router_smem(int tok, int H, int E) {
    return (((size_t)tok * ((E + 7) / 8) * 4 + 15) & ~(size_t)15) + (size_t)tok * H * 2;
}
int router_tok(int T, int H, int E) {
    int tok = T <= 1 ? 1 : (T == 2 ? 2 : (T <= 4 ? 4 : (T <= 64 ? 8 : 16)));
    while (tok > 1 && router_smem(tok, H, E) > kRouterMaxSmem) tok >>= 1;
    return tok;
}

namespace {

template <int VPL>
__global__ void __launch_bounds__(256) k_route_topk(const float *__restrict__ logits, int T, int E, int k,
                                                    int32_t *__restrict__ ids, float *__restrict__ w) {
    // programmatic dependent launch: wait for the previous kernel before
    // touching memory, then let the next one be scheduled
    pdl_wait();
    pdl_launch_dependents();
    const int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    if (t >= T) return;
    const float *l = logits + (size_t)t * E;
    route_token_warp<VPL>([l](int e) { return __ldg(l + e); }, E, k, ids + (size_t)t * k, w + (size_t)t * k);
}

// ------------------------------------- routing and grouping in one launch
// For a decode batch of T <= 16 tokens the top-k above and the stable grouping
// of moe_permute in one CTA of 16 warps.  Warp w routes token w into shared
// memory (a token's top-k is a chain of k warp reductions, so one CTA routing
// more tokens than it has warps would be slower than the many-CTA routing
// kernel); then the grouping takes moe_permute's steps over the routes held
// there: warp w owns a contiguous segment of routes and counts them per expert
// with __match_any_sync (no atomics), a scan in (expert, warp) order gives every
// warp its base row per expert, and a second walk of the segment places each
// route at that base plus its rank among the equal ids before it.  The outputs
// are those of moe_route_topk followed by moe_permute, bit for bit, from one
// launch instead of two.
constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedMaxR = kFusedWarps * kMaxK;  // routes of 16 tokens at k <= 32

template <int VPL>
__global__ void __launch_bounds__(kFusedThreads) k_route_permute(const float *__restrict__ logits, int T, int E, int k,
                                                                 int32_t *__restrict__ ids, float *__restrict__ w,
                                                                 int32_t *__restrict__ counts,
                                                                 int32_t *__restrict__ offsets,
                                                                 int32_t *__restrict__ sorted_route,
                                                                 int32_t *__restrict__ route_pos,
                                                                 uint32_t *__restrict__ hits) {
    constexpr int NW = kFusedWarps, PER = kMaxE / kFusedThreads;
    extern __shared__ int s_cw[];  // [NW][E] per-warp counts, then bases
    __shared__ int32_t s_ids[kFusedMaxR];
    __shared__ float s_wt[kFusedMaxR];
    __shared__ int s_warp[NW];
    __shared__ int s_total;
    // programmatic dependent launch: wait for the logits, then let the next
    // kernel be scheduled
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int R = T * k;
    for (int t = warp; t < T; t += NW) {
        const float *l = logits + (size_t)t * E;
        route_token_warp<VPL>([l](int e) { return __ldg(l + e); }, E, k, s_ids + t * k, s_wt + t * k);
    }
    for (int i = tid; i < NW * E; i += kFusedThreads) s_cw[i] = 0;
    __syncthreads();
    for (int r = tid; r < R; r += kFusedThreads) {
        ids[r] = s_ids[r];
        w[r] = s_wt[r];
    }
    const int seg = (R + NW - 1) / NW;
    const int r_begin = warp * seg, r_end = min(R, r_begin + seg);
    const unsigned lt_mask = (1u << lane) - 1u;
    // pass 1: per-warp counts
    for (int base = r_begin; base < r_end; base += 32) {
        const int r = base + lane;
        int e = r < r_end ? s_ids[r] : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (peers & lt_mask) == 0) s_cw[warp * E + e] += __popc(peers);
    }
    __syncthreads();
    // totals per expert and their exclusive scan; thread tid holds experts
    // PER*tid .. PER*tid + PER-1
    int loc[PER], sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = tid * PER + i;
        int c = 0;
        if (e < E)
            for (int v = 0; v < NW; ++v) c += s_cw[v * E + e];
        loc[i] = c;
        sum += c;
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < NW ? s_warp[lane] : 0;
        int x = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += u;
        }
        if (lane < NW) s_warp[lane] = x - v;
        if (lane == 31) s_total = x;
    }
    __syncthreads();
    int run = s_warp[warp] + incl - sum;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = tid * PER + i;
        if (e < E) {
            counts[e] = loc[i];
            offsets[e] = run;
            if (hits) hits[e] += (uint32_t)loc[i];
            int b = run;
            for (int v = 0; v < NW; ++v) {  // per-warp bases, in warp (= route) order
                const int c = s_cw[v * E + e];
                s_cw[v * E + e] = b;
                b += c;
            }
        }
        run += loc[i];
    }
    if (tid == 0) offsets[E] = s_total;
    __syncthreads();
    // pass 2: stable placement
    for (int base = r_begin; base < r_end; base += 32) {
        const int r = base + lane;
        int e = r < r_end ? s_ids[r] : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (r < r_end) {
            if (e >= 0) {
                const int pos = s_cw[warp * E + e] + __popc(peers & lt_mask);
                sorted_route[pos] = r;
                route_pos[r] = pos;
            } else {
                route_pos[r] = -1;
            }
        }
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) s_cw[warp * E + e] += __popc(peers);
        __syncwarp();
    }
    for (int i = s_total + tid; i < R; i += kFusedThreads) sorted_route[i] = -1;
}

// The same outputs for one token (T = 1, so k <= 32 routes) from a single
// warp: lane r holds route r; the counts of the experts a lane owns (a
// contiguous block of VPL ids) come from one pass over the routes by shuffles,
// their exclusive scan in id order gives the offsets, and route r goes to
// offsets[e_r] + (routes before r with the same expert) -- the stable order of
// moe_permute.  No block barrier, and the hit counters are read before the
// logits arrive.
template <int VPL>
__global__ void __launch_bounds__(32) k_route_permute_warp(const float *__restrict__ logits, int T, int E, int k,
                                                           int32_t *__restrict__ ids, float *__restrict__ w,
                                                           int32_t *__restrict__ counts,
                                                           int32_t *__restrict__ offsets,
                                                           int32_t *__restrict__ sorted_route,
                                                           int32_t *__restrict__ route_pos,
                                                           uint32_t *__restrict__ hits) {
    __shared__ int32_t s_ids[32];
    __shared__ float s_wt[32];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x;
    const int R = T * k;
    const int e0 = lane * VPL;  // this lane's experts: e0 .. e0 + VPL - 1
    uint32_t hv[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) hv[i] = (hits != nullptr && e0 + i < E) ? hits[e0 + i] : 0u;
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (size_t)t * E;
        route_token_warp<VPL>([l](int e) { return __ldg(l + e); }, E, k, s_ids + t * k, s_wt + t * k);
    }
    __syncwarp();
    const int raw = lane < R ? s_ids[lane] : -1;
    const int er = (raw >= 0 && raw < E) ? raw : -1;
    if (lane < R) {
        ids[lane] = raw;
        w[lane] = s_wt[lane];
    }
    // one pass over the routes: counts of this lane's experts, and for route
    // `lane` the valid routes of lower experts and of its expert before it
    int c[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) c[i] = 0;
    int lower = 0, same_before = 0;
    for (int r = 0; r < R; ++r) {
        const int e = __shfl_sync(0xffffffffu, er, r);
        const int d = e - e0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) c[i] += (d == i);
        lower += (e >= 0 && e < er);
        same_before += (r < lane && e == er);
    }
    int sum = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) sum += c[i];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = e0 + i;
        if (e < E) {
            counts[e] = c[i];
            offsets[e] = run;
            if (hits) hits[e] = hv[i] + (uint32_t)c[i];
        }
        run += c[i];
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) offsets[E] = total;
    if (lane < R) {
        const int pos = er >= 0 ? lower + same_before : -1;
        route_pos[lane] = pos;
        if (pos >= 0) sorted_route[pos] = lane;
        if (lane >= total) sorted_route[lane] = -1;
    }
}

// ------------------------------------------------ router projection + top-k
// The step before the routing: logits[t][e] = sum_h x[t][h] * w_router[e][h]
// (x bf16, router weights fp32, fp32 fused multiply-adds), then the top-k
// recipe above on those logits, in one launch.
//
// A cluster of kRouterCluster CTAs takes TOK tokens; CTA r of the cluster
// projects experts [r*EB, (r+1)*EB) (EB = ceil(E / kRouterCluster)) for all TOK
// tokens into its shared memory, so the router weights are read once per
// cluster and every SM of the cluster streams a different slice of them (the
// group's activation rows are staged in its shared memory).  After
// a cluster barrier, CTA r routes token r of the group: its warp 0 reads the E
// logits from the eight CTAs' shared memory (distributed shared memory) and
// runs route_token_warp.  A second cluster barrier keeps every slice alive
// until all reads are done.
//
// Summation order of one logit: lane l of the warp owning expert e sums the
// products of h = 4l .. 4l+3 (mod 128) in increasing h, then the 32 lane sums
// are added by a butterfly (xor 16, 8, 4, 2, 1).
constexpr int kRouterCluster = 8;
constexpr int kRouterThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// NT threads per CTA: 256 (eight warps, two experts each), or for one token
// 512 (sixteen warps, one expert each, all of a lane's chunks of the row in
// flight at once: one DRAM round trip instead of three at H = 2816).
template <int TOK, int VPL, int NT>
__global__ void __cluster_dims__(kRouterCluster, 1, 1) __launch_bounds__(NT)
    k_router_topk(const uint16_t *__restrict__ x, const float *__restrict__ wr, int T, int H, int E, int k,
                  float *__restrict__ logits, int32_t *__restrict__ ids, float *__restrict__ w) {
    extern __shared__ __align__(16) uint8_t smem[];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int EB = (E + kRouterCluster - 1) / kRouterCluster;
    const int t0 = blockIdx.y * TOK;
    const int nt = min(TOK, T - t0);
    float *s_logit = reinterpret_cast<float *>(smem);                                  // [TOK][EB]
    uint16_t *s_x = reinterpret_cast<uint16_t *>(smem + ((TOK * EB * 4 + 15) & ~15));  // [TOK][H]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // this CTA's slice of the router weights (rows e_lo .. e_hi-1, contiguous)
    // is requested into L2 first, so its DRAM latency overlaps the staging below
    // (and, under programmatic dependent launch, the previous kernel's tail: the
    // weights do not depend on it; x does, so the staging waits for it)
    const int e_lo = rank * EB, e_hi = min(E, e_lo + EB);
    if (e_hi > e_lo) {
        const char *slice = reinterpret_cast<const char *>(wr + (size_t)e_lo * H);
        const size_t bytes = (size_t)(e_hi - e_lo) * H * 4;
        for (size_t off = (size_t)threadIdx.x * 128; off < bytes; off += (size_t)NT * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(slice + off));
    }
    pdl_wait();
    pdl_launch_dependents();

    // the group's activation rows (zero past the last token)
    const int h4 = H / 4;
    for (int i = threadIdx.x; i < TOK * h4; i += NT) {
        const int t = i / h4, c = i - t * h4;
        uint2 v = make_uint2(0u, 0u);
        if (t < nt) v = __ldg(reinterpret_cast<const uint2 *>(x + (size_t)(t0 + t) * H) + c);
        reinterpret_cast<uint2 *>(s_x + (size_t)t * H)[c] = v;
    }
    __syncthreads();

    // projection: warp w takes experts e_lo + EPW w (and the next one when EPW
    // is 2), then + EPW * NW, ...; U chunks of 128 h per lane are loaded before
    // they are used, so U loads of each operand are in flight (the sums still run
    // in increasing h)
    constexpr int NW = NT / 32, EPW = NT >= 512 ? 1 : 2;
    constexpr int U = NT >= 512 ? 22 : (TOK <= 8 ? 8 : 4);
    for (int e0 = e_lo + EPW * warp; e0 < e_hi; e0 += EPW * NW) {
        const bool two = EPW == 2 && e0 + 1 < e_hi;
        const float *w0 = wr + (size_t)e0 * H;
        const float *w1 = wr + (size_t)(two ? e0 + 1 : e0) * H;
        float a0[TOK], a1[TOK];
#pragma unroll
        for (int t = 0; t < TOK; ++t) a0[t] = a1[t] = 0.0f;
        for (int hb = lane * 4; hb < H; hb += 128 * U) {
            float4 p[U], q[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int h = hb + 128 * u;
                p[u] = q[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (h < H) {
                    p[u] = __ldg(reinterpret_cast<const float4 *>(w0 + h));
                    if (EPW == 2) q[u] = __ldg(reinterpret_cast<const float4 *>(w1 + h));
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int h = hb + 128 * u;
                if (h < H) {
#pragma unroll
                    for (int t = 0; t < TOK; ++t) {
                        const uint2 xv = *reinterpret_cast<const uint2 *>(s_x + (size_t)t * H + h);
                        const float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
                        const float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
                        a0[t] = __fmaf_rn(x0, p[u].x, a0[t]);
                        a0[t] = __fmaf_rn(x1, p[u].y, a0[t]);
                        a0[t] = __fmaf_rn(x2, p[u].z, a0[t]);
                        a0[t] = __fmaf_rn(x3, p[u].w, a0[t]);
                        if (EPW == 2) {
                            a1[t] = __fmaf_rn(x0, q[u].x, a1[t]);
                            a1[t] = __fmaf_rn(x1, q[u].y, a1[t]);
                            a1[t] = __fmaf_rn(x2, q[u].z, a1[t]);
                            a1[t] = __fmaf_rn(x3, q[u].w, a1[t]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TOK; ++t) {
            a0[t] = warp_sum(a0[t]);
            if (EPW == 2) a1[t] = warp_sum(a1[t]);
        }
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < TOK; ++t) {
                s_logit[t * EB + (e0 - e_lo)] = a0[t];
                if (two) s_logit[t * EB + (e0 + 1 - e_lo)] = a1[t];
                if (logits != nullptr && t < nt) {
                    logits[(size_t)(t0 + t) * E + e0] = a0[t];
                    if (two) logits[(size_t)(t0 + t) * E + e0 + 1] = a1[t];
                }
            }
        }
    }

    cluster.sync();
    // CTA r routes tokens r, r + 8, ... of the group, one warp each
    const int t = rank + kRouterCluster * warp;
    if (warp < (TOK + kRouterCluster - 1) / kRouterCluster && t < nt) {
        route_token_warp<VPL>(
            [&](int e) {
                const float *slice = cluster.map_shared_rank(s_logit, e / EB);
                return slice[t * EB + e % EB];
            },
            E, k, ids + (size_t)(t0 + t) * k, w + (size_t)(t0 + t) * k);
    }
    cluster.sync();
}

template <int TOK, int VPL, int NT = kRouterThreads>
cudaError_t launch_router(const uint16_t *x, const float *wr, int T, int H, int E, int k, float *logits,
                          int32_t *ids, float *w, cudaStream_t s) {
    auto kern = k_router_topk<TOK, VPL, NT>;
    static bool attr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!attr[dev]) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRouterMaxSmem);
        if (err != cudaSuccess) return err;
        attr[dev] = true;
    }
    dim3 grid(kRouterCluster, (unsigned)((T + TOK - 1) / TOK));
    // programmatic dependent launch (the cluster shape comes from the kernel's
    // __cluster_dims__)
    return launch_pdl(kern, grid, dim3(NT), router_smem(TOK, H, E), s, x, wr, T, H, E, k, logits, ids, w);
}

template <int VPL>
cudaError_t launch_router_vpl(const uint16_t *x, const float *wr, int T, int H, int E, int k, float *logits,
                              int32_t *ids, float *w, cudaStream_t s) {
    const int tok = router_tok(T, H, E);
    if (router_smem(tok, H, E) > kRouterMaxSmem) return cudaErrorInvalidValue;
    if (tok == 16) return launch_router<16, VPL>(x, wr, T, H, E, k, logits, ids, w, s);
    if (tok == 1) return launch_router<1, VPL, 512>(x, wr, T, H, E, k, logits, ids, w, s);
    if (tok == 2) return launch_router<2, VPL>(x, wr, T, H, E, k, logits, ids, w, s);
    if (tok == 4) return launch_router<4, VPL>(x, wr, T, H, E, k, logits, ids, w, s);
    return launch_router<8, VPL>(x, wr, T, H, E, k, logits, ids, w, s);
}

// [miss] min_weight partial routing, one thread per token: heaviest route
// first, a route whose expert has no cache slot is dropped once the kept weight
// has reached min_weight; the kept weights are scaled by total / kept.
__global__ void __launch_bounds__(256) k_route_min_weight(int32_t *__restrict__ ids, float *__restrict__ w,
                                                          const int32_t *__restrict__ slot_table, int T, int k,
                                                          int E, float min_weight) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    int32_t *id = ids + (size_t)t * k;
    float *wt = w + (size_t)t * k;
    uint32_t dropped = 0;
    float kept = 0.0f, total = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int e = id[j];
        const bool resident = slot_table != nullptr && e >= 0 && e < E && __ldg(slot_table + e) >= 0;
        if (!resident && kept >= min_weight) dropped |= 1u << j;
        else kept = __fadd_rn(kept, wt[j]);
    }
    for (int j = 0; j < k; ++j) total = __fadd_rn(total, wt[j]);
    const float scale = kept > 0.0f ? __fdiv_rn(total, kept) : 0.0f;
    for (int j = 0; j < k; ++j) {
        if (((dropped >> j) & 1u) || !(kept > 0.0f)) {
            id[j] = -1;
            wt[j] = 0.0f;
        } else {
            wt[j] = __fmul_rn(wt[j], scale);
        }
    }
}

}  // namespace

cudaError_t launch_route_min_weight(int32_t *ids, float *w, const int32_t *slot_table, int T, int k, int E,
                                    float min_weight, cudaStream_t s) {
    if (T == 0 || !(min_weight < 1.0f)) return cudaSuccess;
    k_route_min_weight<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(ids, w, slot_table, T, k, E, min_weight);
    return cudaGetLastError();
}

cudaError_t launch_router_topk(const uint16_t *x, const float *w_router, int T, int H, int E, int k, float *logits,
                               int32_t *ids, float *w, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    if (E <= 128) return launch_router_vpl<4>(x, w_router, T, H, E, k, logits, ids, w, s);
    return launch_router_vpl<32>(x, w_router, T, H, E, k, logits, ids, w, s);
}

cudaError_t launch_route_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w,
                              cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int vpl = (E + 31) / 32;
    dim3 block(256), grid((unsigned)((T + 7) / 8));
    if (vpl <= 1) return launch_pdl(k_route_topk<1>, grid, block, 0, s, logits, T, E, k, ids, w);
    if (vpl <= 2) return launch_pdl(k_route_topk<2>, grid, block, 0, s, logits, T, E, k, ids, w);
    if (vpl <= 4) return launch_pdl(k_route_topk<4>, grid, block, 0, s, logits, T, E, k, ids, w);
    if (vpl <= 8) return launch_pdl(k_route_topk<8>, grid, block, 0, s, logits, T, E, k, ids, w);
    if (vpl <= 16) return launch_pdl(k_route_topk<16>, grid, block, 0, s, logits, T, E, k, ids, w);
    return launch_pdl(k_route_topk<32>, grid, block, 0, s, logits, T, E, k, ids, w);
}

bool route_permute_fused(int T, int k) { return T <= kFusedWarps && k <= kMaxK; }

cudaError_t launch_route_permute(const float *logits, int T, int E, int k, int32_t *ids, float *w,
                                 int32_t *counts, int32_t *offsets, int32_t *sorted_route, int32_t *route_pos,
                                 uint32_t *hits, cudaStream_t s) {
    const int vpl = (E + 31) / 32;
    const size_t smem = (size_t)kFusedWarps * E * sizeof(int);  // <= 64 KiB (E <= 1024)
    dim3 block(kFusedThreads), grid(1);
    auto go = [&](auto kern) {
        // one-time attribute per device and instantiation (kept out of stream capture)
        static size_t cached[kMaxDevices] = {};
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
        if (cached[dev] < smem) {
            err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (err != cudaSuccess) return err;
            cached[dev] = smem;
        }
        return launch_pdl(kern, grid, block, smem, s, logits, T, E, k, ids, w, counts, offsets, sorted_route,
                          route_pos, hits);
    };
    if (T == 1) {  // one warp (no shared-memory attribute needed)
        auto one = [&](auto kern) {
            return launch_pdl(kern, dim3(1), dim3(32), 0, s, logits, T, E, k, ids, w, counts, offsets, sorted_route,
                              route_pos, hits);
        };
        if (vpl <= 1) return one(k_route_permute_warp<1>);
        if (vpl <= 2) return one(k_route_permute_warp<2>);
        if (vpl <= 4) return one(k_route_permute_warp<4>);
        if (vpl <= 8) return one(k_route_permute_warp<8>);
        if (vpl <= 16) return one(k_route_permute_warp<16>);
        return one(k_route_permute_warp<32>);
    }
    if (vpl <= 1) return go(k_route_permute<1>);
    if (vpl <= 2) return go(k_route_permute<2>);
    if (vpl <= 4) return go(k_route_permute<4>);
    if (vpl <= 8) return go(k_route_permute<8>);
    if (vpl <= 16) return go(k_route_permute<16>);
    return go(k_route_permute<32>);
}

}  // namespace moe
