// quantize.cu -- one-time weight-only quantisers of the expert pack (prain
// README.md, "Expert formats": int8 with an fp32 scale per row; int4 with a
// bf16 scale per 64 weights chosen by MSE clip).  Every floating-point step
// that decides a code is an explicit round-to-nearest intrinsic, so the codes
// and scales are bit-exact to the recipe in moe.h.
#include "common.cuh"

namespace moe {
namespace {

// int8: one warp per row.
__global__ void __launch_bounds__(256) k_quantize_int8(const uint16_t *__restrict__ w, int rows, int K,
                                                       int8_t *__restrict__ q, float *__restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    if (r >= rows) return;
    const uint16_t *wr = w + (size_t)r * K;
    float amax = 0.0f;
    for (int c = lane; c < K; c += 32) amax = fmaxf(amax, fabsf(bf16_to_f32(wr[c])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = __fdiv_rn(amax, 127.0f);
    if (lane == 0) scale[r] = s;
    for (int c = lane; c < K; c += 32) {
        int qi = 0;
        if (s != 0.0f) {
            qi = (int)rintf(__fdiv_rn(bf16_to_f32(wr[c]), s));
            qi = max(-127, min(127, qi));
        }
        q[(size_t)r * K + c] = (int8_t)qi;
    }
}

// int8, rows of K <= 32 * 16 * 8 with K % 8 == 0: one warp per row, the row
// read once into registers as 16-byte chunks (chunk c of the row on lane
// c % 32), the codes stored 8 at a time; the same fp32 steps as k_quantize_int8.
constexpr int kQ8Chunks = 16;  // chunks per lane
__global__ void __launch_bounds__(256) k_quantize_int8_vec(const uint16_t *__restrict__ w, int rows, int K,
                                                           int8_t *__restrict__ q, float *__restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    if (r >= rows) return;
    const int nch = K / 8;
    const uint4 *src = reinterpret_cast<const uint4 *>(w + (size_t)r * K);
    uint4 u[kQ8Chunks];
#pragma unroll
    for (int i = 0; i < kQ8Chunks; ++i) {
        const int c = lane + 32 * i;
        u[i] = c < nch ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kQ8Chunks; ++i) {
        const uint32_t p[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(p[j])), fabsf(bf16_hi(p[j]))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = __fdiv_rn(amax, 127.0f);
    if (lane == 0) scale[r] = s;
    uint2 *dst = reinterpret_cast<uint2 *>(q + (size_t)r * K);
#pragma unroll
    for (int i = 0; i < kQ8Chunks; ++i) {
        const int c = lane + 32 * i;
        if (c >= nch) continue;
        const uint32_t p[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
        uint32_t o[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float v = (j & 1) ? bf16_hi(p[j >> 1]) : bf16_lo(p[j >> 1]);
            int qi = 0;
            if (s != 0.0f) {
                qi = (int)rintf(__fdiv_rn(v, s));
                qi = max(-127, min(127, qi));
            }
            o[j >> 2] |= ((uint32_t)qi & 0xffu) << (8 * (j & 3));
        }
        dst[c] = make_uint2(o[0], o[1]);
    }
}

__device__ __forceinline__ int int4_code(float v, float s) {
    if (s == 0.0f) return 0;
    int qi = (int)rintf(__fdiv_rn(v, s));
    return max(-8, min(7, qi));
}

// int4: one thread per group of 64 weights; the 16-ratio clip search with the
// error summed in fp64 in weight order (so both the choice and the tie rule are
// reproducible), then the codes of the chosen scale.
__global__ void __launch_bounds__(128) k_quantize_int4(const uint16_t *__restrict__ w, int rows, int K,
                                                       uint8_t *__restrict__ q, uint16_t *__restrict__ scale) {
    const int G = K / 64;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)rows * G) return;
    const int r = (int)(gid / G), g = (int)(gid % G);
    const uint4 *src = reinterpret_cast<const uint4 *>(w + (size_t)r * K + (size_t)g * 64);
    float v[64];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint4 u = __ldg(src + i);
        v[8 * i + 0] = bf16_lo(u.x); v[8 * i + 1] = bf16_hi(u.x);
        v[8 * i + 2] = bf16_lo(u.y); v[8 * i + 3] = bf16_hi(u.y);
        v[8 * i + 4] = bf16_lo(u.z); v[8 * i + 5] = bf16_hi(u.z);
        v[8 * i + 6] = bf16_lo(u.w); v[8 * i + 7] = bf16_hi(u.w);
    }
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 64; ++c) amax = fmaxf(amax, fabsf(v[c]));

    double best = __longlong_as_double(0x7ff0000000000000ll);  // +inf
    float sbest = 0.0f;
    for (int i = 15; i >= 0; --i) {
        const float ratio = __double2float_rn(__ddiv_rn((double)(70 + 2 * i), 100.0));
        const float t = __fdiv_rn(__fmul_rn(ratio, amax), 7.0f);
        const float s = bf16_to_f32(f32_to_bf16_rne(t));
        double err = 0.0;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
            const int qi = int4_code(v[c], s);
            const double d = __dsub_rn((double)v[c], __dmul_rn((double)qi, (double)s));
            err = __dadd_rn(err, __dmul_rn(d, d));
        }
        if (err < best) {
            best = err;
            sbest = s;
        }
    }
    uint32_t words[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t word = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) word |= (uint32_t)(int4_code(v[8 * i + c], sbest) + 8) << (4 * c);
        words[i] = word;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(q + (size_t)r * (K / 2) + (size_t)g * 32);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    scale[(size_t)r * G + g] = f32_to_bf16_rne(sbest);
}

}  // namespace

cudaError_t launch_quantize_int8(const uint16_t *w, int rows, int K, int8_t *q, float *scale, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    // rows of whole 16-byte chunks (at most 16 per lane), aligned buffers: the
    // register-resident kernel; anything else: the element loop
    if (K % 8 == 0 && K / 8 <= 32 * kQ8Chunks && ((uintptr_t)w & 15u) == 0 && ((uintptr_t)q & 7u) == 0)
        k_quantize_int8_vec<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(w, rows, K, q, scale);
    else
        k_quantize_int8<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(w, rows, K, q, scale);
    return cudaGetLastError();
}

cudaError_t launch_quantize_int4(const uint16_t *w, int rows, int K, uint8_t *q, uint16_t *scale, cudaStream_t s) {
    const int64_t n = (int64_t)rows * (K / 64);
    if (n == 0) return cudaSuccess;
    k_quantize_int4<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(w, rows, K, q, scale);
    return cudaGetLastError();
}

}  // namespace moe
