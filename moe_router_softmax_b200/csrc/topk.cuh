// topk.cuh -- one token's top-k routing by one warp, shared by the routing
// kernels (route.cu) and the one-token FFN kernels that route for themselves
// (ffn_gemv.cu): the same code, so the same ids and weights bit for bit.
//
// ids: the k largest logits in descending order, equal logits to the lower
// expert id (expert_pool.rs ranks equal counts by the lower id), NaN last.
// w: softmax renormalised over the k kept experts, which equals a softmax over
// the kept logits (the full denominator cancels).  All fp32 steps are written
// with explicit round-to-nearest intrinsics so that no multiply-add is fused
// behind our back.
#pragma once

#include "common.cuh"

namespace moe {
namespace topk {

// exp_p -- the library's fp32 exponential, from the mathematics:
//   x = n ln2 + r with n = rint(x log2e), r by a two-constant Cody-Waite
//   reduction (LN2_HI has its low 8 mantissa bits clear, so n*LN2_HI is exact
//   for |n| < 256); e^r by its Taylor series to degree 7 (|r| <= ln2/2, the
//   truncation error is below 6e-9 relative) in fma Horner form; 2^n from the
//   exponent bits, in two steps when 2^n is subnormal.
// Constants: log2(e), ln2 split, and 1/k! -- each the nearest fp32.
__device__ __forceinline__ float pow2_bits(int m) { return __uint_as_float((uint32_t)(m + 127) << 23); }

__device__ __forceinline__ float exp_p(float x) {
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

// The routing order: a larger logit ranks first, equal logits (-0 equal to +0)
// by the lower expert id, NaN after every number.  rank_key gives a 32-bit key
// whose unsigned order is that logit order: NaN below every number (key 0, and
// every NaN alike), -0 equal to +0, otherwise the IEEE bits made monotone
// (negative: all bits flipped; positive: sign set).  Equal keys are then
// ordered by expert id separately.
__device__ __forceinline__ uint32_t rank_key(float v) {
    if (v != v) return 0u;
    const uint32_t b = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Top-k and weights of one token, by one warp.  load(e) returns logit e for
// e < E; lane l holds experts l, l+32, ...; the k winners are taken one at a
// time by a warp arg-best, then the softmax over them (max logit first).
// Each logit's rank key is formed once (plus one, so that 0 marks a taken or
// absent slot below every NaN's key of 1); a lane's best slot is its largest key
// (the first slot on ties: the lower id), the warp's winner the largest key,
// then the lowest id holding it -- the routing order above.
template <int VPL, class Load>
__device__ __forceinline__ void route_token_warp(Load load, int E, int k, int32_t *ids_row, float *w_row) {
    const int lane = threadIdx.x & 31;
    float v[VPL];
    uint32_t key[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        int e = lane + 32 * i;
        v[i] = 0.0f;
        key[i] = 0u;
        if (e < E) {
            v[i] = load(e);
            key[i] = rank_key(v[i]) + 1u;
        }
    }
    float my_v = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = key[0];
        float bv = v[0];
        int bi = 0;
#pragma unroll
        for (int i = 1; i < VPL; ++i)
            if (key[i] > bk) {
                bk = key[i];
                bv = v[i];
                bi = i;
            }
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
        const int cand = (bk != 0u && bk == kmax) ? lane + 32 * bi : 0x7fffffff;
        const int win = __reduce_min_sync(0xffffffffu, cand);
        const float wv = __shfl_sync(0xffffffffu, bv, win & 31);
        if (lane == (win & 31)) {
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (i == (win >> 5)) key[i] = 0u;
        }
        if (lane == j) {
            my_v = wv;
            my_e = win;
        }
    }
    const float m = __shfl_sync(0xffffffffu, my_v, 0);
    const float ej = (lane < k) ? exp_p(__fsub_rn(my_v, m)) : 0.0f;
    float S = 0.0f;
    for (int j = 0; j < k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, ej, j));
    if (lane < k) {
        ids_row[lane] = my_e;
        w_row[lane] = __fdiv_rn(ej, S);
    }
}

}  // namespace topk
}  // namespace moe
