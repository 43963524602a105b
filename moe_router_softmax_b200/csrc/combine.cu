// combine.cu -- weighted gather of each token's k expert rows back to token
// order (remote_experts.cpp, RemoteExperts::finish returns every row to its
// route's position; the router weights it).  One thread per 4 output columns;
// the k terms are summed in route order in fp32; no atomics.
#include "common.cuh"

namespace moe {
namespace {

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
    return launch_pdl(k_combine, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, rows, route_pos, w, T, k, H, y);
}

}  // namespace moe
