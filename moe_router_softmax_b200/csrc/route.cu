// route.cu -- top-k routing of fp32 router logits (one warp per token).
//
// ids: the k largest logits in descending order, equal logits to the lower
// expert id (expert_pool.rs ranks equal counts by the lower id), NaN last.
// w: softmax renormalised over the k kept experts, which equals a softmax over
// the kept logits (the full denominator cancels).  All fp32 steps are written
// with explicit round-to-nearest intrinsics so that no multiply-add is fused
// behind our back: the result is bit-for-bit the recipe of moe_route_topk.
#include "common.cuh"

namespace moe {
namespace {

// exp_p -- the library's fp32 exponential, from the mathematics:
//   x = n ln2 + r with n = rint(x log2e), r by a two-constant Cody-Waite
//   reduction (LN2_HI has its low 8 mantissa bits clear, so n*LN2_HI is exact
//   for |n| < 256); e^r by its Taylor series to degree 7 (|r| <= ln2/2, the
//   truncation error is below 6e-9 relative) in fma Horner form; 2^n from the
//   exponent bits, in two steps when 2^n is subnormal.
// Constants: log2(e), ln2 split, and 1/k! -- each the nearest fp32.
__device__ __forceinline__ float pow2_bits(int m) { return __uint_as_float((uint32_t)(m + 127) << 23); }

__device__ float exp_p(float x) {
    const float kLog2e = 0x1.715476p+0f;   // log2(e)
    const float kLn2Hi = 0x1.62e400p-1f;   // ln 2, top 16 significant bits
    const float kLn2Lo = 0x1.7f7d1cp-20f;  // ln 2 - kLn2Hi
    if (x != x) return x;
    if (x > 88.8f) return __int_as_float(0x7f800000);
    if (x < -104.0f) return 0.0f;
    float n = rintf(__fmul_rn(x, kLog2e));
    float r = __fmaf_rn(-n, kLn2Hi, x);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = 0x1.a01a02p-13f;              // 1/5040
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);   // 1/720
    p = __fmaf_rn(p, r, 0x1.111112p-7f);    // 1/120
    p = __fmaf_rn(p, r, 0x1.555556p-5f);    // 1/24
    p = __fmaf_rn(p, r, 0x1.555556p-3f);    // 1/6
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    int ni = (int)n;
    if (ni < -126) return __fmul_rn(__fmul_rn(p, pow2_bits(ni + 100)), pow2_bits(-100));
    if (ni > 127) return __fmul_rn(__fmul_rn(p, pow2_bits(ni - 1)), 2.0f);
    return __fmul_rn(p, pow2_bits(ni));
}

// (va, ea) ranks before (vb, eb): larger logit, then lower id; NaN last.
__device__ __forceinline__ bool ranks_before(float va, int ea, float vb, int eb) {
    bool na = va != va, nb = vb != vb;
    if (na != nb) return nb;
    if (!na && va != vb) return va > vb;
    return ea < eb;
}

template <int VPL>
__global__ void __launch_bounds__(256) k_route_topk(const float *__restrict__ logits, int T, int E, int k,
                                                    int32_t *__restrict__ ids, float *__restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    if (t >= T) return;
    const float *l = logits + (size_t)t * E;
    float v[VPL];
    uint32_t avail = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        int e = lane + 32 * i;
        v[i] = 0.0f;
        if (e < E) {
            v[i] = __ldg(l + e);
            avail |= 1u << i;
        }
    }
    float my_v = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        // best available value held by this lane
        bool has = false;
        float bv = 0.0f;
        int be = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            if ((avail >> i) & 1u) {
                int e = lane + 32 * i;
                if (!has || ranks_before(v[i], e, bv, be)) {
                    has = true;
                    bv = v[i];
                    be = e;
                }
            }
        }
        // warp arg-best
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            int oe = __shfl_xor_sync(0xffffffffu, be, off);
            bool oh = __shfl_xor_sync(0xffffffffu, (int)has, off) != 0;
            if (oh && (!has || ranks_before(ov, oe, bv, be))) {
                has = true;
                bv = ov;
                be = oe;
            }
        }
        if (lane == (be & 31)) avail &= ~(1u << (be >> 5));
        if (lane == j) {
            my_v = bv;
            my_e = be;
        }
    }
    const float m = __shfl_sync(0xffffffffu, my_v, 0);
    const float ej = (lane < k) ? exp_p(__fsub_rn(my_v, m)) : 0.0f;
    float S = 0.0f;
    for (int j = 0; j < k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, ej, j));
    if (lane < k) {
        ids[(size_t)t * k + lane] = my_e;
        w[(size_t)t * k + lane] = __fdiv_rn(ej, S);
    }
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

cudaError_t launch_route_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w,
                              cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int vpl = (E + 31) / 32;
    dim3 block(256), grid((unsigned)((T + 7) / 8));
    if (vpl <= 1) k_route_topk<1><<<grid, block, 0, s>>>(logits, T, E, k, ids, w);
    else if (vpl <= 2) k_route_topk<2><<<grid, block, 0, s>>>(logits, T, E, k, ids, w);
    else if (vpl <= 4) k_route_topk<4><<<grid, block, 0, s>>>(logits, T, E, k, ids, w);
    else if (vpl <= 8) k_route_topk<8><<<grid, block, 0, s>>>(logits, T, E, k, ids, w);
    else if (vpl <= 16) k_route_topk<16><<<grid, block, 0, s>>>(logits, T, E, k, ids, w);
    else k_route_topk<32><<<grid, block, 0, s>>>(logits, T, E, k, ids, w);
    return cudaGetLastError();
}

}  // namespace moe
