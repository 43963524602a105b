// combine.cu -- weighted gather of each token's k expert rows back to token
// order (remote_experts.cpp, RemoteExperts::finish returns every row to its
// route's position; the router weights it).  One thread per 4 output columns;
// the k terms are summed in route order in fp32; no atomics.
#include "common.cuh"

namespace moe {
namespace {

// KM > 0: k <= KM routes per token, with every route position, weight and row
// load of a thread issued before the first sum (k independent DRAM/L2 round
// trips in flight instead of a chain of them); the sum is taken in the same
// route order, so the result is identical to the general loop (KM = 0).
template <int KM>
__global__ void __launch_bounds__(256) k_combine(const float *__restrict__ rows, const int32_t *__restrict__ route_pos,
                                                 const float *__restrict__ w, int T, int k, int H,
                                                 uint16_t *__restrict__ y) {
    // programmatic dependent launch: wait for the previous kernel before
    // touching memory, then let the next one be scheduled
    pdl_wait();
    pdl_launch_dependents();
    const int q4 = H >> 2;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)T * q4) return;
    const int t = (int)(idx / q4), c = (int)(idx % q4) * 4;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    if (KM > 0) {
        int p[KM > 0 ? KM : 1];
        float wj[KM > 0 ? KM : 1];
        float4 r[KM > 0 ? KM : 1];
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            p[j] = j < k ? __ldg(route_pos + (int64_t)t * k + j) : -1;
            wj[j] = j < k ? __ldg(w + (int64_t)t * k + j) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < KM; ++j)
            r[j] = p[j] >= 0 ? __ldg(reinterpret_cast<const float4 *>(rows + (int64_t)p[j] * H + c))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (p[j] < 0) continue;
            a0 = __fmaf_rn(wj[j], r[j].x, a0);
            a1 = __fmaf_rn(wj[j], r[j].y, a1);
            a2 = __fmaf_rn(wj[j], r[j].z, a2);
            a3 = __fmaf_rn(wj[j], r[j].w, a3);
        }
    } else {
        for (int j = 0; j < k; ++j) {
            const int p = __ldg(route_pos + (int64_t)t * k + j);
            if (p < 0) continue;
            const float wj = __ldg(w + (int64_t)t * k + j);
            const float4 r = __ldg(reinterpret_cast<const float4 *>(rows + (int64_t)p * H + c));
            a0 = __fmaf_rn(wj, r.x, a0);
            a1 = __fmaf_rn(wj, r.y, a1);
            a2 = __fmaf_rn(wj, r.z, a2);
            a3 = __fmaf_rn(wj, r.w, a3);
        }
    }
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_rne(a0) | ((uint32_t)f32_to_bf16_rne(a1) << 16);
    o.y = (uint32_t)f32_to_bf16_rne(a2) | ((uint32_t)f32_to_bf16_rne(a3) << 16);
    *reinterpret_cast<uint2 *>(y + (int64_t)t * H + c) = o;
}

}  // namespace

cudaError_t launch_combine(const float *rows, const int32_t *route_pos, const float *w, int T, int k, int H,
                           uint16_t *y, cudaStream_t s) {
    const int64_t n = (int64_t)T * (H / 4);
    if (n == 0) return cudaSuccess;
    const dim3 grid((unsigned)((n + 255) / 256)), block(256);
    if (k <= 8) return launch_pdl(k_combine<8>, grid, block, 0, s, rows, route_pos, w, T, k, H, y);
    return launch_pdl(k_combine<0>, grid, block, 0, s, rows, route_pos, w, T, k, H, y);
}

}  // namespace moe
