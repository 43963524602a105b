// ffn_gemv.cu -- grouped gated FFN for decode-sized batches: a split-K,
// warp-shuffle-reduced grouped GEMV that streams every routed expert's weights
// from HBM exactly once, dequantising in registers.
//
// What it computes (prain README.md, "Expert formats", for the formats; the
// gated GELU-tanh FFN with w13 = gate rows [0,I) stacked on up rows [I,2I)):
//   phase 1 (k_ffn_gemv<..., 1>):  for every sorted route row s of expert e,
//        g = W13_e x_{token(s)},  h[s][i] = bf16(gelu_tanh(g_i) * g_{I+i})
//   phase 2 (k_ffn_gemv<..., 2>):  rows[s] = W2_e h[s]
// with fp32 accumulation.  token(s) = sorted_route[s] / k (remote_experts.cpp,
// RemoteExperts::begin).  An expert is reached through the slot table
// (expert_blob()).
//
// One token (T = 1) has kernels of its own (k_ffn_gemv_tok, below): the k
// routes' rows are split evenly over all warps, each warp streams its rows
// without pausing between them, and the set-up before the first weight load is
// a single round of loads.  Where they route the token themselves (a
// moe_layer_forward call), phase 2 can also take the combine: each CTA then
// computes every route of its own output rows and writes y (see k_ffn_gemv_tok).
//
// Work decomposition (T > 1).  A work item is (active expert, chunk of <= 8 of its
// routes, tile of output rows).  Each CTA (8 warps) takes a contiguous range
// of items, so consecutive items share an expert and the routes' activations
// stay in shared memory (fp32, bank-conflict-free "sub-plane" layout).  Inside
// a tile, a lane group of LG lanes owns RWP weight rows (phase 1: RWP/2 gate
// rows and their RWP/2 up rows, so the GELU gate is applied in the epilogue
// without a second pass); the lanes of a group split K into 16-byte chunks
// (8 bf16 / 16 int8 / 32 int4 weights) and stream them with 128-bit
// L1-bypassing loads, U chunks per row in flight; the partial dot products
// are reduced across the group with xor shuffles.  LG is chosen so that each
// lane streams about 11 chunks of each row (K = 2816 or 704).
#include <algorithm>

#include "common.cuh"
#include "topk.cuh"

namespace moe {

struct FfnParams {
    LayerView L;
    const uint16_t *x;            // [T][H] bf16
    int T, k;
    const int32_t *counts;        // [E]
    const int32_t *offsets;       // [E+1]
    const int32_t *sorted_route;  // [R]
    uint16_t *h;                  // [R][I] bf16 (phase 1 out / phase 2 in)
    float *rows;                  // [R][H] fp32
    int lg;                       // lanes per row group (power of two, <= 32)
    // one-token kernels: activation floats shared memory holds; passes per unit;
    // the N = k * units split over the W warps of the grid (warp w starts at
    // floor(w * N / W)) and 1 / W; 1 / units per route (division-free indices)
    int xs_floats, passes;
    unsigned n_all, n_warps;
    double inv_warps;
    float inv_units;
    // one-token kernels that route the token themselves (logits != nullptr):
    // its router logits [E], and the routing outputs that CTA 0 of phase 1
    // writes (those of moe_route_permute; counts, offsets and sorted_route then
    // point at the caller's buffers, which the kernels do not read)
    const float *logits;
    uint32_t *hits;
    int32_t *ids_out, *counts_out, *offsets_out, *sorted_out, *pos_out;
    float *w_out;
    // one-token phase 2 with the combine (nullable): y [1][H] bf16
    uint16_t *y;
};

namespace {

// First fault a GEMV kernel recorded (0 = none): 0x2005 for an expert whose
// slot is past the pool (info = the slot id; the expert's routes are skipped),
// 0x2007 for a one-token CTA whose activations would not fit the shared memory
// it was launched with (info = routes; the CTA does nothing; the host's sizing
// rules it out).  Read and cleared by moe_take_device_errors().
__device__ unsigned int g_gemv_error;
__device__ unsigned int g_gemv_error_info;
__device__ __forceinline__ void record_gemv_error(unsigned code, unsigned info) {
    if (atomicCAS(&g_gemv_error, 0u, code) == 0u) g_gemv_error_info = info;
}

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kNTM = 8;  // routes per work item
constexpr size_t kTokSmemMax = 96 * 1024;  // one-token kernels: activation bytes per CTA

template <int FMT> struct Fmt;
template <> struct Fmt<MOE_W_BF16> { static constexpr int kElems = 8; };   // per 16-byte chunk
template <> struct Fmt<MOE_W_INT8> { static constexpr int kElems = 16; };
template <> struct Fmt<MOE_W_INT4> { static constexpr int kElems = 32; };

__device__ __forceinline__ float gelu_tanh(float v) {
    const float c = 0.7978845608028654f;  // sqrt(2/pi)
    const float u = c * (v + 0.044715f * v * v * v);
    return 0.5f * v * (1.0f + tanhf(u));
}

// Decode sub-plane sp (4 consecutive weights) of a 16-byte chunk into fp32.
// bf16: words 2sp, 2sp+1.  int8: word sp, signed bytes (value + 128 placed in
// the mantissa of 2^23, minus 2^23 + 128).  int4: half of word sp/2, nibbles
// (n - 8) the same way (2^23 + n, minus 2^23 + 8).
template <int FMT>
__device__ __forceinline__ void decode4(const uint4 &q, int sp, float w[4]) {
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
    if (FMT == MOE_W_BF16) {
        const uint32_t a = words[2 * sp], b = words[2 * sp + 1];
        w[0] = bf16_lo(a); w[1] = bf16_hi(a); w[2] = bf16_lo(b); w[3] = bf16_hi(b);
    } else if (FMT == MOE_W_INT8) {
        const uint32_t a = words[sp] ^ 0x80808080u;
        w[0] = __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7540)) - 8388736.0f;
        w[1] = __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7541)) - 8388736.0f;
        w[2] = __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7542)) - 8388736.0f;
        w[3] = __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7543)) - 8388736.0f;
    } else {
        const uint32_t word = words[sp >> 1];
        const uint32_t lo = word & 0x0F0F0F0Fu;          // nibbles 0,2,4,6 in bytes 0..3
        const uint32_t hi = (word >> 4) & 0x0F0F0F0Fu;   // nibbles 1,3,5,7
        if ((sp & 1) == 0) {
            w[0] = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540)) - 8388616.0f;
            w[1] = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540)) - 8388616.0f;
            w[2] = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7541)) - 8388616.0f;
            w[3] = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7541)) - 8388616.0f;
        } else {
            w[0] = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7542)) - 8388616.0f;
            w[1] = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7542)) - 8388616.0f;
            w[2] = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7543)) - 8388616.0f;
            w[3] = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7543)) - 8388616.0f;
        }
    }
}

// decode4 as two pairs (w[0], w[1]) and (w[2], w[3]); the int formats' bias is
// taken off both weights of a pair in one packed subtraction (exact: integers
// below 2^24), so the values equal decode4's.
template <int FMT>
__device__ __forceinline__ void decode4_pairs(const uint4 &q, int sp, float2 &lo, float2 &hi) {
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
    if (FMT == MOE_W_BF16) {
        const uint32_t a = words[2 * sp], b = words[2 * sp + 1];
        lo = make_float2(bf16_lo(a), bf16_hi(a));
        hi = make_float2(bf16_lo(b), bf16_hi(b));
    } else if (FMT == MOE_W_INT8) {
        const uint32_t a = words[sp] ^ 0x80808080u;
        const float2 bias = make_float2(-8388736.0f, -8388736.0f);
        lo = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(a, 0x4B000000u, 0x7540)),
                                    __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7541))), bias);
        hi = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(a, 0x4B000000u, 0x7542)),
                                    __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7543))), bias);
    } else {
        const uint32_t word = words[sp >> 1];
        const uint32_t l4 = word & 0x0F0F0F0Fu, h4 = (word >> 4) & 0x0F0F0F0Fu;
        const uint32_t s0 = (sp & 1) ? 0x7542u : 0x7540u, s1 = (sp & 1) ? 0x7543u : 0x7541u;
        const float2 bias = make_float2(-8388616.0f, -8388616.0f);
        lo = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(l4, 0x4B000000u, s0)),
                                    __uint_as_float(__byte_perm(h4, 0x4B000000u, s0))), bias);
        hi = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(l4, 0x4B000000u, s1)),
                                    __uint_as_float(__byte_perm(h4, 0x4B000000u, s1))), bias);
    }
}

// Load the activations of the item's routes into shared memory as fp32.
// Layout: xs[((t * SP + sp) * nchunks + c) * 4 + i] = x_t[c * kElems + 4 sp + i]
// so that lanes reading consecutive chunks of one sub-plane hit consecutive
// 16-byte words (no bank conflicts).
template <int FMT, int PHASE>
__device__ void load_acts(const FfnParams &p, float *xs, int row0, int nt, int K, int nchunks) {
    constexpr int EC = Fmt<FMT>::kElems, SP = EC / 4;
    const int per_t = K / 8;  // 8-element (16-byte bf16) pieces per route
    for (int idx = threadIdx.x; idx < nt * per_t; idx += kThreads) {
        const int t = idx / per_t, piece = idx - t * per_t;
        const uint16_t *src;
        if (PHASE == 1) {
            const int tok = __ldg(p.sorted_route + row0 + t) / p.k;
            src = p.x + (size_t)tok * p.L.H + (size_t)piece * 8;
        } else {
            src = p.h + (size_t)(row0 + t) * p.L.I + (size_t)piece * 8;
        }
        const uint4 u = *reinterpret_cast<const uint4 *>(src);
        const int e0 = piece * 8;             // element index of the piece
        const int c = e0 / EC, sp = (e0 % EC) / 4;
        float4 *d0 = reinterpret_cast<float4 *>(xs + ((size_t)(t * SP + sp) * nchunks + c) * 4);
        float4 *d1 = reinterpret_cast<float4 *>(xs + ((size_t)(t * SP + sp + 1) * nchunks + c) * 4);
        *d0 = make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
        *d1 = make_float4(bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w));
    }
}

// The single token's activations (T = 1: token 0) into shared memory, in
// load_acts's layout.
template <int FMT>
__device__ void load_x0(const FfnParams &p, float *xs, int K, int nchunks) {
    constexpr int EC = Fmt<FMT>::kElems;
    for (int piece = threadIdx.x; piece < K / 8; piece += kThreads) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p.x + (size_t)piece * 8);
        const int e0 = piece * 8;
        const int c = e0 / EC, sp = (e0 % EC) / 4;
        float4 *d0 = reinterpret_cast<float4 *>(xs + ((size_t)sp * nchunks + c) * 4);
        float4 *d1 = reinterpret_cast<float4 *>(xs + ((size_t)(sp + 1) * nchunks + c) * 4);
        *d0 = make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
        *d1 = make_float4(bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w));
    }
}

// One work item for one lane group: RWP rows x NT routes.
template <int FMT, int PHASE, int RWP, int U, int NT>
__device__ __forceinline__ void run_item(const FfnParams &p, const float *xs, const uint8_t *blob, int u0,
                                         int row0, int nt, int K, int nchunks, int li, int lg) {
    constexpr int EC = Fmt<FMT>::kElems, SP = EC / 4;
    constexpr int UPG = PHASE == 1 ? RWP / 2 : RWP;  // units (pairs or rows) per group
    const int I = p.L.I, H = p.L.H;
    const int n_units = PHASE == 1 ? I : H;
    const uint64_t qoff = PHASE == 1 ? p.L.off.q13 : p.L.off.q2;
    const uint64_t soff = PHASE == 1 ? p.L.off.s13 : p.L.off.s2;
    const size_t row_bytes = (size_t)nchunks * 16;

    int row[RWP];
    bool valid[RWP];
#pragma unroll
    for (int q = 0; q < RWP; ++q) {
        const int unit = u0 + (PHASE == 1 ? q / 2 : q);
        valid[q] = unit < n_units;
        const int uu = valid[q] ? unit : 0;
        row[q] = PHASE == 1 ? ((q & 1) ? I + uu : uu) : uu;
    }
    const uint8_t *qbase = blob + qoff;

    float acc[RWP][NT];
#pragma unroll
    for (int q = 0; q < RWP; ++q)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[q][t] = 0.0f;

    for (int c0 = li; c0 < nchunks; c0 += U * lg) {
        uint4 wq[U][RWP];
        float sc[U][RWP];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * lg;
#pragma unroll
            for (int q = 0; q < RWP; ++q) {
                if (c < nchunks) {
                    wq[u][q] = ld_stream_v4(qbase + (size_t)row[q] * row_bytes + (size_t)c * 16);
                    if (FMT == MOE_W_INT4)
                        sc[u][q] = bf16_to_f32(__ldg(reinterpret_cast<const uint16_t *>(blob + soff) +
                                                     (size_t)row[q] * (K / 64) + (c >> 1)));
                } else {
                    wq[u][q] = make_uint4(0, 0, 0, 0);
                    sc[u][q] = 0.0f;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * lg;
            if (c >= nchunks) break;
            if (FMT == MOE_W_INT4) {
                float part[RWP][NT];
#pragma unroll
                for (int q = 0; q < RWP; ++q)
#pragma unroll
                    for (int t = 0; t < NT; ++t) part[q][t] = 0.0f;
#pragma unroll
                for (int sp = 0; sp < SP; ++sp) {
                    float w[RWP][4];
#pragma unroll
                    for (int q = 0; q < RWP; ++q) decode4<FMT>(wq[u][q], sp, w[q]);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const float4 xv = *reinterpret_cast<const float4 *>(xs + ((size_t)(t * SP + sp) * nchunks + c) * 4);
#pragma unroll
                        for (int q = 0; q < RWP; ++q) {
                            part[q][t] = fmaf(w[q][0], xv.x, part[q][t]);
                            part[q][t] = fmaf(w[q][1], xv.y, part[q][t]);
                            part[q][t] = fmaf(w[q][2], xv.z, part[q][t]);
                            part[q][t] = fmaf(w[q][3], xv.w, part[q][t]);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < RWP; ++q)
#pragma unroll
                    for (int t = 0; t < NT; ++t) acc[q][t] = fmaf(sc[u][q], part[q][t], acc[q][t]);
            } else {
#pragma unroll
                for (int sp = 0; sp < SP; ++sp) {
                    float w[RWP][4];
#pragma unroll
                    for (int q = 0; q < RWP; ++q) decode4<FMT>(wq[u][q], sp, w[q]);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const float4 xv = *reinterpret_cast<const float4 *>(xs + ((size_t)(t * SP + sp) * nchunks + c) * 4);
#pragma unroll
                        for (int q = 0; q < RWP; ++q) {
                            acc[q][t] = fmaf(w[q][0], xv.x, acc[q][t]);
                            acc[q][t] = fmaf(w[q][1], xv.y, acc[q][t]);
                            acc[q][t] = fmaf(w[q][2], xv.z, acc[q][t]);
                            acc[q][t] = fmaf(w[q][3], xv.w, acc[q][t]);
                        }
                    }
                }
            }
        }
    }

    // reduce across the lane group
#pragma unroll
    for (int q = 0; q < RWP; ++q)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            float v = acc[q][t];
            for (int off = lg >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            acc[q][t] = v;
        }
    if (FMT == MOE_W_INT8) {
#pragma unroll
        for (int q = 0; q < RWP; ++q) {
            const float s = __ldg(reinterpret_cast<const float *>(blob + soff) + row[q]);
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[q][t] *= s;
        }
    }

    // epilogue: every lane of the group holds every sum; lane li writes the
    // routes t with t % lg == li
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if ((t & (lg - 1)) != li || t >= nt) continue;
        const size_t srow = (size_t)(row0 + t);
        if (PHASE == 1) {
#pragma unroll
            for (int q = 0; q < UPG; ++q) {
                if (!valid[2 * q]) continue;
                const float g = acc[2 * q][t], up = acc[2 * q + 1][t];
                p.h[srow * I + (u0 + q)] = f32_to_bf16_rne(gelu_tanh(g) * up);
            }
        } else {
#pragma unroll
            for (int q = 0; q < RWP; ++q) {
                if (!valid[q]) continue;
                p.rows[srow * H + row[q]] = acc[q][t];
            }
        }
    }
}

template <int FMT, int PHASE, int RWP, int U>
__global__ void __launch_bounds__(kThreads, 2) k_ffn_gemv(FfnParams p) {
    constexpr int UPG = PHASE == 1 ? RWP / 2 : RWP;
    constexpr int EC = Fmt<FMT>::kElems;
    extern __shared__ __align__(16) float xs[];
    __shared__ int s_act[kMaxE];
    __shared__ int s_base[kMaxE + 1];
    __shared__ int s_nact;

    const int E = p.L.E;
    const int K = PHASE == 1 ? p.L.H : p.L.I;
    const int nchunks = K / EC;
    const int lg = p.lg;
    const int n_units = PHASE == 1 ? p.L.I : p.L.H;
    const int groups = kWarps * (32 / lg);
    const int upi = groups * UPG;              // units per item
    const int tiles = (n_units + upi - 1) / upi;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // programmatic dependent launch: phase 1 waits for the permutation before
    // anything else; phase 2 may be scheduled as soon as phase 1 has started
    // (it waits for h itself, after requesting its weights into L2)
    if (PHASE == 1) pdl_wait();
    pdl_launch_dependents();

    // active experts and the prefix of their item counts (one warp)
    if (warp == 0) {
        int n_act = 0, run = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int n = (e < E) ? __ldg(p.counts + e) : 0;
            const bool act = n > 0;
            const unsigned m = __ballot_sync(0xffffffffu, act);
            const int items = act ? tiles * ((n + kNTM - 1) / kNTM) : 0;
            int inc = items;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, off);
                if (lane >= off) inc += v;
            }
            if (act) {
                const int pos = n_act + __popc(m & ((1u << lane) - 1u));
                s_act[pos] = e;
                s_base[pos] = run + inc - items;
            }
            run += __shfl_sync(0xffffffffu, inc, 31);
            n_act += __popc(m);
        }
        if (lane == 0) {
            s_nact = n_act;
            s_base[n_act] = run;
        }
    }
    __syncthreads();
    const int n_act = s_nact;
    const int total = s_base[n_act];
    const int it_begin = (int)(((long long)total * blockIdx.x) / gridDim.x);
    const int it_end = (int)(((long long)total * (blockIdx.x + 1)) / gridDim.x);
    if (it_begin >= it_end) return;

    int a = 0;
    {   // first active expert whose items reach it_begin
        int lo = 0, hi = n_act - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_base[mid] <= it_begin) lo = mid; else hi = mid - 1;
        }
        a = lo;
    }
    if (PHASE == 2 && threadIdx.x == 0) {
        // launched while phase 1 may still run: request this CTA's weight rows
        // into L2 first (they do not depend on phase 1), then wait for h
        const uint64_t row_bytes = (uint64_t)nchunks * 16;
        int pa = a;
        for (int it = it_begin; it < it_end; ++it) {
            while (s_base[pa + 1] <= it) ++pa;
            const int tile = (it - s_base[pa]) % tiles;
            const int r0 = tile * upi, r1 = min(n_units, r0 + upi);
            const uint8_t *blob = expert_blob(p.L, s_act[pa]);
            if (blob == nullptr) continue;  // slot out of the pool: the item is skipped below
            const uint8_t *w = blob + p.L.off.q2 + (uint64_t)r0 * row_bytes;
            for (uint64_t off = 0, n = (uint64_t)(r1 - r0) * row_bytes; off < n; off += 32768) {
                const uint32_t bytes = (uint32_t)(n - off < 32768 ? n - off : 32768);
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(w + off), "r"(bytes) : "memory");
            }
        }
    }
    if (PHASE == 2) pdl_wait();
    const int li = lane & (lg - 1);
    const int gi = warp * (32 / lg) + lane / lg;
    int cur_key = -1;
    for (int it = it_begin; it < it_end; ++it) {
        while (s_base[a + 1] <= it) ++a;
        const int rem = it - s_base[a];
        const int chunk = rem / tiles, tile = rem - chunk * tiles;
        const int e = s_act[a];
        const int n_e = __ldg(p.counts + e);
        const int row0 = __ldg(p.offsets + e) + chunk * kNTM;
        const int nt = min(kNTM, n_e - chunk * kNTM);
        const uint8_t *blob = expert_blob(p.L, e);
        if (blob == nullptr) {
            // the expert's slot is past the pool: nothing of this item is read or
            // written (the same for every thread of the CTA, so no barrier is split)
            if (threadIdx.x == 0) record_gemv_error(0x2005u, (unsigned)__ldg(p.L.slot_table + e));
            continue;
        }
        const int key = a * 65536 + chunk;
        if (key != cur_key) {
            __syncthreads();
            load_acts<FMT, PHASE>(p, xs, row0, nt, K, nchunks);
            __syncthreads();
            cur_key = key;
        }
        const int u0 = tile * upi + gi * UPG;
        if (nt > 4) run_item<FMT, PHASE, RWP, U, 8>(p, xs, blob, u0, row0, nt, K, nchunks, li, lg);
        else if (nt > 2) run_item<FMT, PHASE, RWP, U, 4>(p, xs, blob, u0, row0, nt, K, nchunks, li, lg);
        else if (nt > 1) run_item<FMT, PHASE, RWP, U, 2>(p, xs, blob, u0, row0, nt, K, nchunks, li, lg);
        else run_item<FMT, PHASE, RWP, U, 1>(p, xs, blob, u0, row0, nt, K, nchunks, li, lg);
    }
}

// One token (T = 1: k routes of token 0, sorted by expert).  A unit is one
// gate/up row pair (phase 1) or two consecutive output rows (phase 2) of one
// route; the k x units are split evenly over the warps of the grid, and inside
// a warp its 32/lg lane groups take consecutive units.  A unit is read in P
// passes of C 16-byte chunks per lane and row; while a lane consumes chunk j of
// one pass it already loads chunk j of its next pass (of the same unit or of its
// next one), so a warp's weight stream does not stop between units.  The set-up
// before the first weight load is one round of loads (the offsets), and phase 2
// issues its first weight loads before it waits for phase 1 (they do not
// depend on it).
// a / b for 0 <= a < 2^24 and b >= 1, from inv_b = 1/b rounded to float: the
// float quotient is within 1/16 of a/b there, so one correction step is exact.
__device__ __forceinline__ int div_small(int a, int b, float inv_b) {
    int q = (int)((float)a * inv_b);
    if (q * b > a) --q;
    else if ((q + 1) * b <= a) ++q;
    return q;
}
// floor(a / b) for a < 2^32, 1 <= b < 2^31, from inv_b = 1/b rounded to double
// (quotient within 2^-20 of a/b; one correction step).
__device__ __forceinline__ unsigned div_u32(unsigned a, unsigned b, double inv_b) {
    unsigned q = (unsigned)((double)a * inv_b);
    if ((unsigned long long)q * b > a) --q;
    else if ((unsigned long long)(q + 1) * b <= a) ++q;
    return q;
}

// The one token's routing inside a one-token kernel (E <= 128): warp 0 takes
// the top-k of the logits (topk::route_token_warp, the routing kernels' code)
// while the other threads read the slot table; then route r, in lane r, goes to
// sorted position (routes of lower experts) + (routes of its expert before it),
// the stable grouping of moe_permute, and each sorted position gets its expert's
// blob.  With `write` (CTA 0 of phase 1) warp 0 also stores the routing outputs
// and adds the counts to the hit counters (read before the logits arrive).
// s_posj / s_wj (nullable) get each route's sorted position and weight.
__device__ __forceinline__ void tok_route(const FfnParams &p, bool write, int *s_exp, const uint8_t **s_blob,
                                          int *s_posj = nullptr, float *s_wj = nullptr) {
    constexpr int VPL = 4;  // E <= 128
    __shared__ int32_t s_rid[kMaxK];
    __shared__ float s_rw[kMaxK];
    __shared__ int s_slot[128];
    const int E = p.L.E, k = p.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t hv[VPL];
    if (warp == 0) {
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = lane * VPL + i;
            hv[i] = (write && p.hits != nullptr && e < E) ? p.hits[e] : 0u;
        }
        const float *l = p.logits;
        topk::route_token_warp<VPL>([l](int e) { return __ldg(l + e); }, E, k, s_rid, s_rw);
    } else if (threadIdx.x - 32 < E) {
        const int e = threadIdx.x - 32;
        s_slot[e] = p.L.slot_table ? __ldg(p.L.slot_table + e) : -1;
    }
    __syncthreads();
    if (warp == 0) {
        const int er = lane < k ? s_rid[lane] : -1;
        int lower = 0, same_before = 0;
        int c[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) c[i] = 0;
        for (int r = 0; r < k; ++r) {
            const int e = __shfl_sync(0xffffffffu, er, r);
            lower += (e < er);
            same_before += (r < lane && e == er);
#pragma unroll
            for (int i = 0; i < VPL; ++i) c[i] += (e == lane * VPL + i);
        }
        if (lane < k) {
            const int pos = lower + same_before;
            const int sl = s_slot[er];
            const bool bad = p.L.slot_table != nullptr && sl >= p.L.pool_slots;
            s_exp[pos] = er;
            if (s_posj != nullptr) {
                s_posj[lane] = pos;
                s_wj[lane] = s_rw[lane];
            }
            s_blob[pos] = bad ? nullptr : (sl >= 0 ? p.L.pool + (uint64_t)sl * p.L.stride : p.L.home + (uint64_t)er * p.L.stride);
            if (write) {
                p.ids_out[lane] = er;
                p.w_out[lane] = s_rw[lane];
                p.pos_out[lane] = pos;
                p.sorted_out[pos] = lane;
            }
        }
        if (write) {
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
                const int e = lane * VPL + i;
                if (e < E) {
                    p.counts_out[e] = c[i];
                    p.offsets_out[e] = run;
                    if (p.hits) p.hits[e] = hv[i] + (uint32_t)c[i];
                }
                run += c[i];
            }
            if (lane == 0) p.offsets_out[E] = k;
        }
    }
    __syncthreads();
}

// Y (phase 2 of a routed call only): the combine of the one token in the same
// launch.  The CTA then takes the row pairs [cp0, cp0 + np) of every route (its
// warps split those k * np units, route-major), keeps its rows in shared memory
// instead of writing them out, and writes y for its rows: the k terms in route
// order with the fp32 fma of moe_combine, so y is bit-identical to the two calls.
template <int FMT, int PHASE, int C, bool ROUTE, bool Y = false>
__global__ void __launch_bounds__(kThreads, 2) k_ffn_gemv_tok(FfnParams p) {
    static_assert(!Y || (PHASE == 2 && ROUTE), "the fused combine is phase 2 of a routed call");
    constexpr int EC = Fmt<FMT>::kElems, SP = EC / 4;
    extern __shared__ __align__(16) float xs[];
    __shared__ int s_exp[kMaxK];
    __shared__ const uint8_t *s_blob[kMaxK];
    __shared__ int s_nroutes;
    __shared__ int s_posj[Y ? kMaxK : 1];
    __shared__ float s_wj[Y ? kMaxK : 1];
    const int H = p.L.H, I = p.L.I;
    const int K = PHASE == 1 ? H : I;
    const int nchunks = K / EC;
    const int n_units = PHASE == 1 ? I : (H + 1) / 2;
    const int lg = p.lg, gpw = 32 / lg, P = p.passes;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane & (lg - 1), gi = lane / lg;
    // Y: the CTA's row pairs (one integer division per thread, at set-up)
    const int cp0 = Y ? (int)((long long)blockIdx.x * n_units / gridDim.x) : 0;
    const int np = Y ? (int)((long long)(blockIdx.x + 1) * n_units / gridDim.x) - cp0 : n_units;
    // the warp's units (all k routes' units split evenly over the grid's warps,
    // or for Y the CTA's k * np units over its warps; units of routes the
    // permutation left empty are skipped below) and the routes whose activations
    // the CTA reads: no device data needed yet
    auto warp_start = [&](unsigned w) {
        return Y ? (int)(((long long)w - (long long)blockIdx.x * kWarps) * p.k * np / kWarps)
                 : (int)div_u32(w * p.n_all, p.n_warps, p.inv_warps);
    };
    const int w_u0 = warp_start(blockIdx.x * kWarps + warp), w_u1 = warp_start(blockIdx.x * kWarps + warp + 1);
    const int trips = (w_u1 - w_u0 + gpw - 1) / gpw;
    const int c_u0 = warp_start(blockIdx.x * kWarps), c_u1 = warp_start((blockIdx.x + 1) * kWarps);
    // a CTA without units (fewer units than warps) exits at once, which also
    // releases dependents -- unless it is the CTA that writes the routing
    const bool writer = ROUTE && PHASE == 1 && blockIdx.x == 0;
    if (c_u1 == c_u0 && !writer) return;
    const int s_lo = Y ? 0 : (c_u1 > c_u0 ? div_small(c_u0, n_units, p.inv_units) : 0);
    const int s_hi = Y ? p.k - 1 : (c_u1 > c_u0 ? div_small(c_u1 - 1, n_units, p.inv_units) : 0);
    // Y: the CTA's rows of every route follow the activations, [sorted route][2 np]
    float *s_rows = xs + (size_t)p.k * K;
    if ((PHASE == 1 ? 1 : s_hi - s_lo + 1) * K + (Y ? 2 * p.k * np : 0) > p.xs_floats) {
        // cannot happen with the host's sizing (same for every thread of the CTA)
        if (threadIdx.x == 0) record_gemv_error(0x2007u, (unsigned)(s_hi - s_lo + 1));
        return;
    }
    // the lane group's first unit: route and unit within the route (Y: within
    // the CTA's np pairs)
    int nx_u = w_u0 + gi;
    int nx_sr = Y ? nx_u / np : div_small(nx_u, n_units, p.inv_units);
    int nx_i = nx_u - nx_sr * np;
    int nx_trip = 0, nx_pass = 0;
    // phase 1 waits for the permutation here; phase 2 may be scheduled as soon
    // as phase 1 has started and waits for h further down
    if (PHASE == 1) pdl_wait();
    pdl_launch_dependents();
    if (ROUTE) {
        // the kernel routes the token itself: all k routes are valid
        tok_route(p, writer, s_exp, s_blob, Y ? s_posj : nullptr, Y ? s_wj : nullptr);
        if (c_u1 == c_u0) return;  // the writer without units of its own
        if (threadIdx.x == 0) s_nroutes = p.k;
        __syncthreads();
    } else {
        // expert and blob of every sorted route (sorted position sr lies in
        // [offsets[e], offsets[e+1]); the slot-table entry is read in the same
        // round of loads as the offsets), and the number of routes: offsets[E],
        // which is below k when the permutation dropped invalid ids
        if (threadIdx.x == 0) s_nroutes = min(__ldg(p.offsets + p.L.E), p.k);
        for (int e = threadIdx.x; e < p.L.E; e += kThreads) {
            const int lo = __ldg(p.offsets + e), hi = min(__ldg(p.offsets + e + 1), p.k);
            const uint8_t *blob = expert_blob(p.L, e);
            for (int sr = lo; sr < hi; ++sr) {
                s_exp[sr] = e;
                s_blob[sr] = blob;
            }
        }
        __syncthreads();
    }
    const int R = s_nroutes;
    const uint64_t qoff = PHASE == 1 ? p.L.off.q13 : p.L.off.q2;
    const uint64_t soff = PHASE == 1 ? p.L.off.s13 : p.L.off.s2;
    const size_t row_bytes = (size_t)nchunks * 16;

    // a lane's view of a step (one pass over one unit): route, first row, where
    // its chunks start; w0 == nullptr: nothing to load (past the warp's units, a
    // route the permutation left empty, or a slot fault).  next_step() takes the
    // step after the previous one, walking (trip, pass) and (route, unit).
    struct Step { const uint8_t *w0; const uint16_t *s0; int sr, r0, c0; bool live, v1; };
    const size_t dw = PHASE == 1 ? (size_t)I * row_bytes : row_bytes;  // second row - first row
    const int ds = PHASE == 1 ? I * (K / 64) : K / 64;                  // the same for int4 scales
    auto next_step = [&](Step &x) {
        x.live = nx_trip < trips && nx_u < w_u1 && nx_sr < R;
        x.c0 = nx_pass * lg * C + li;
        x.sr = nx_sr;
        x.r0 = PHASE == 1 ? nx_i : 2 * (cp0 + nx_i);
        x.v1 = PHASE == 1 || x.r0 + 1 < H;
        x.w0 = nullptr; x.s0 = nullptr;
        if (x.live) {
            const uint8_t *blob = s_blob[x.sr];
            if (blob != nullptr) {
                x.w0 = blob + qoff + (size_t)x.r0 * row_bytes;
                if (FMT == MOE_W_INT4) x.s0 = reinterpret_cast<const uint16_t *>(blob + soff) + (size_t)x.r0 * (K / 64);
            }
        }
        if (++nx_pass == P) {
            nx_pass = 0;
            ++nx_trip;
            nx_u += gpw;
            nx_i += gpw;
            while (nx_i >= np) { nx_i -= np; ++nx_sr; }
        }
    };

    uint4 wq[C][2];
    float sc[C][2];
    Step cur;
    next_step(cur);
    {
        const size_t d1 = cur.v1 ? dw : 0;
        const int e1 = cur.v1 ? ds : 0;
#pragma unroll
        for (int j = 0; j < C; ++j) {
            const int c = cur.c0 + j * lg;
            const bool ok = cur.w0 != nullptr && c < nchunks;
            wq[j][0] = ok ? ld_stream_v4(cur.w0 + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
            wq[j][1] = ok ? ld_stream_v4(cur.w0 + d1 + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
            if (FMT == MOE_W_INT4) {
                sc[j][0] = ok ? bf16_to_f32(__ldg(cur.s0 + (c >> 1))) : 0.0f;
                sc[j][1] = ok ? bf16_to_f32(__ldg(cur.s0 + e1 + (c >> 1))) : 0.0f;
            }
        }
    }
    if (PHASE == 2) pdl_wait();
    if (PHASE == 1) load_x0<FMT>(p, xs, K, nchunks);
    else load_acts<FMT, 2>(p, xs, s_lo, s_hi - s_lo + 1, K, nchunks);
    __syncthreads();

    float a0 = 0.0f, a1 = 0.0f;
    const int steps = trips * P;
    for (int st = 0; st < steps; ++st) {
        Step nx;
        next_step(nx);
        // a lane group past its warp's units computes nothing (its loads were
        // skipped too) and stays on the first route's activations
        const int tx = (PHASE == 1 || !cur.live) ? 0 : cur.sr - s_lo;
        const float *xt = xs + (size_t)tx * SP * nchunks * 4;
#pragma unroll
        for (int j = 0; j < C; ++j) {
            const int c = cur.c0 + j * lg;
            const uint4 q0 = wq[j][0], q1 = wq[j][1];
            const float s0 = FMT == MOE_W_INT4 ? sc[j][0] : 1.0f, s1 = FMT == MOE_W_INT4 ? sc[j][1] : 1.0f;
            {   // chunk j of the next step
                const int cn = nx.c0 + j * lg;
                const bool ok = nx.w0 != nullptr && cn < nchunks;
                const size_t d1 = nx.v1 ? dw : 0;
                wq[j][0] = ok ? ld_stream_v4(nx.w0 + (size_t)cn * 16) : make_uint4(0, 0, 0, 0);
                wq[j][1] = ok ? ld_stream_v4(nx.w0 + d1 + (size_t)cn * 16) : make_uint4(0, 0, 0, 0);
                if (FMT == MOE_W_INT4) {
                    const int e1 = nx.v1 ? ds : 0;
                    sc[j][0] = ok ? bf16_to_f32(__ldg(nx.s0 + (cn >> 1))) : 0.0f;
                    sc[j][1] = ok ? bf16_to_f32(__ldg(nx.s0 + e1 + (cn >> 1))) : 0.0f;
                }
            }
            if (cur.live && c < nchunks) {
                // even and odd weights in two packed partial sums (sm_100 packed
                // fp32 fma: half the fma instructions)
                float2 p0 = make_float2(0.0f, 0.0f), p1 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int spi = 0; spi < SP; ++spi) {
                    float2 w0l, w0h, w1l, w1h;
                    decode4_pairs<FMT>(q0, spi, w0l, w0h);
                    decode4_pairs<FMT>(q1, spi, w1l, w1h);
                    const float4 xv = *reinterpret_cast<const float4 *>(xt + ((size_t)spi * nchunks + c) * 4);
                    const float2 xl = make_float2(xv.x, xv.y), xh = make_float2(xv.z, xv.w);
                    p0 = __ffma2_rn(w0l, xl, p0); p0 = __ffma2_rn(w0h, xh, p0);
                    p1 = __ffma2_rn(w1l, xl, p1); p1 = __ffma2_rn(w1h, xh, p1);
                }
                const float r0 = p0.x + p0.y, r1 = p1.x + p1.y;
                if (FMT == MOE_W_INT4) { a0 = fmaf(s0, r0, a0); a1 = fmaf(s1, r1, a1); }
                else { a0 += r0; a1 += r1; }
            }
        }
        if ((st + 1) % P == 0) {  // the unit's last pass: reduce over the group, write
            for (int off = lg >> 1; off > 0; off >>= 1) {
                a0 += __shfl_xor_sync(0xffffffffu, a0, off);
                a1 += __shfl_xor_sync(0xffffffffu, a1, off);
            }
            if (cur.live && li == 0) {
                if (cur.w0 == nullptr) {
                    record_gemv_error(0x2005u, (unsigned)__ldg(p.L.slot_table + s_exp[cur.sr]));
                } else {
                    const int r1 = PHASE == 1 ? I + cur.r0 : cur.r0 + 1;
                    if (FMT == MOE_W_INT8) {
                        const float *sp = reinterpret_cast<const float *>(cur.w0 - qoff - (size_t)cur.r0 * row_bytes + soff);
                        a0 *= __ldg(sp + cur.r0);
                        if (cur.v1) a1 *= __ldg(sp + r1);
                    }
                    if (PHASE == 1) {
                        p.h[(size_t)cur.sr * I + cur.r0] = f32_to_bf16_rne(gelu_tanh(a0) * a1);
                    } else if (Y) {
                        float *yr = s_rows + (size_t)cur.sr * 2 * np + (cur.r0 - 2 * cp0);
                        yr[0] = a0;
                        if (cur.v1) yr[1] = a1;
                    } else {
                        p.rows[(size_t)cur.sr * H + cur.r0] = a0;
                        if (cur.v1) p.rows[(size_t)cur.sr * H + r1] = a1;
                    }
                }
            }
            a0 = 0.0f; a1 = 0.0f;
        }
        cur = nx;
    }
    if (Y) {
        // y for the CTA's rows 2 cp0 .. 2 (cp0 + np) - 1: the routes in route order
        __syncthreads();
        const int n_rows = min(2 * np, H - 2 * cp0);
        for (int lr = threadIdx.x; lr < n_rows; lr += kThreads) {
            float a = 0.0f;
            for (int j = 0; j < p.k; ++j) a = __fmaf_rn(s_wj[j], s_rows[(size_t)s_posj[j] * 2 * np + lr], a);
            p.y[2 * cp0 + lr] = f32_to_bf16_rne(a);
        }
    }
}

// Lanes per row group: the largest power of two <= 32 that leaves every lane
// at least `per_lane` chunks of a row (so a group is never mostly idle).
int pick_lg(int nchunks, int per_lane) {
    int lg = 32;
    while (lg > 1 && nchunks < lg * per_lane) lg >>= 1;
    return lg;
}

template <int FMT, int PHASE, int RWP, int U>
cudaError_t launch_phase(const FfnParams &p0, int n_sm, cudaStream_t s) {
    FfnParams p = p0;
    const int K = PHASE == 1 ? p.L.H : p.L.I;
    const int nchunks = K / Fmt<FMT>::kElems;
    p.lg = pick_lg(nchunks, 8);
    const size_t smem = (size_t)kNTM * K * sizeof(float);
    auto kern = k_ffn_gemv<FMT, PHASE, RWP, U>;
    // one-time set-up per device and shared-memory size (kept out of stream
    // capture: after the first call a launch is the only API call made here)
    static int cached_smem[kMaxDevices] = {}, cached_per_sm[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if ((size_t)cached_smem[dev] < smem) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        int per_sm = 0;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
        if (err != cudaSuccess) return err;
        cached_per_sm[dev] = per_sm < 1 ? 1 : per_sm;
        cached_smem[dev] = (int)smem;
    }
    const int per_sm = cached_per_sm[dev];
    // programmatic dependent launch (see the kernel's first lines)
    return launch_pdl(kern, dim3((unsigned)(n_sm * per_sm)), dim3(kThreads), smem, s, p);
}


// Shared-memory floats a one-token kernel needs for a CTA's activations
// (phase 1: the token; phase 2: the h rows of the routes its units touch),
// with a grid of at least n_sm CTAs: a CTA takes at most N / n_sm + 1 of the
// N units, consecutive ones.
size_t tok_xs_floats(const FfnParams &p, int phase, int n_sm) {
    if (phase == 1) return (size_t)p.L.H;
    const long long n_units = (p.L.H + 1) / 2, N = (long long)p.k * n_units;
    const long long per_cta = N / n_sm + 1;
    const long long span = std::min<long long>(p.k, (per_cta - 1) / n_units + 2);
    return (size_t)span * p.L.I;
}

// Phase 2 with the combine (Y): the h rows of all k routes, then the CTA's rows
// of every route (at most ceil(units / n_sm) row pairs each).
size_t tok_y_floats(const FfnParams &p, int n_sm) {
    const long long n_units = (p.L.H + 1) / 2;
    return (size_t)p.k * p.L.I + (size_t)(2 * p.k * ((n_units + n_sm - 1) / n_sm));
}

// The one-token kernels take the call: T = 1, a CTA's activations fit in shared
// memory beside a second CTA, and w * N stays below 2^32 for every warp w (at up
// to 8 CTAs per SM).
bool tok_fits(const FfnParams &p, int n_sm) {
    const unsigned long long max_units = (unsigned long long)p.k * std::max(p.L.I, (p.L.H + 1) / 2);
    return p.T == 1 && p.k <= kMaxK && tok_xs_floats(p, 1, n_sm) * 4 <= kTokSmemMax &&
           tok_xs_floats(p, 2, n_sm) * 4 <= kTokSmemMax &&
           max_units * (unsigned long long)(n_sm * 8 * kWarps) < (1ull << 32);
}

template <int FMT, int PHASE, int C, bool ROUTE, bool Y = false>
cudaError_t launch_tok(const FfnParams &p0, int n_sm, cudaStream_t s) {
    FfnParams p = p0;
    const int nchunks = (PHASE == 1 ? p.L.H : p.L.I) / Fmt<FMT>::kElems;
    int lg = 1;  // the narrowest group that covers a row in one pass, at most a warp
    while (lg < 32 && lg * C < nchunks) lg <<= 1;
    p.lg = lg;
    p.passes = (nchunks + lg * C - 1) / (lg * C);
    p.xs_floats = (int)(Y ? tok_y_floats(p, n_sm) : tok_xs_floats(p, PHASE, n_sm));
    const int n_units = PHASE == 1 ? p.L.I : (p.L.H + 1) / 2;
    p.inv_units = 1.0f / (float)n_units;
    const size_t smem = (size_t)p.xs_floats * sizeof(float);
    auto kern = k_ffn_gemv_tok<FMT, PHASE, C, ROUTE, Y>;
    static size_t cached_smem[kMaxDevices] = {};
    static int cached_per_sm[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (cached_smem[dev] < smem) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        int per_sm = 0;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
        if (err != cudaSuccess) return err;
        cached_per_sm[dev] = per_sm < 1 ? 1 : per_sm;
        cached_smem[dev] = smem;
    }
    const int grid = n_sm * cached_per_sm[dev];
    p.n_all = (unsigned)(p.k * n_units);
    p.n_warps = (unsigned)(grid * kWarps);
    p.inv_warps = 1.0 / (double)p.n_warps;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), smem, s, p);
}

template <int FMT>
cudaError_t launch_fmt(const FfnParams &p, int n_sm, cudaStream_t s) {
    // rows per lane group: 2 (one gate/up pair in phase 1); U chunks
    // of each row in flight, so a lane keeps 8 x 16 bytes of weights in flight
    constexpr int RWP = 2;
    constexpr int U = 8 / RWP;
    // one token: the streaming kernels above when tok_fits (at H = 2816, I = 704
    // the activations take 11 KiB in phase 1, 5.5 KiB in phase 2); chunks per lane
    // and row in each pass: 6 (4 for int4, whose scales take registers too)
    if (tok_fits(p, n_sm)) {
        constexpr int C = FMT == MOE_W_INT4 ? 4 : 6;
        if (p.logits != nullptr) {
            cudaError_t err = launch_tok<FMT, 1, C, true>(p, n_sm, s);
            if (err != cudaSuccess) return err;
            if (p.y != nullptr) {
                if (tok_y_floats(p, n_sm) * 4 > kTokSmemMax) return cudaErrorInvalidValue;
                return launch_tok<FMT, 2, C, true, true>(p, n_sm, s);
            }
            return launch_tok<FMT, 2, C, true>(p, n_sm, s);
        }
        cudaError_t err = launch_tok<FMT, 1, C, false>(p, n_sm, s);
        if (err != cudaSuccess) return err;
        return launch_tok<FMT, 2, C, false>(p, n_sm, s);
    }
    cudaError_t err = launch_phase<FMT, 1, RWP, U>(p, n_sm, s);
    if (err != cudaSuccess) return err;
    return launch_phase<FMT, 2, RWP, U>(p, n_sm, s);
}

}  // namespace

size_t ffn_gemv_workspace(int T, int k, int I) { return (size_t)T * k * I * sizeof(uint16_t); }

cudaError_t gemv_take_error(unsigned *code, unsigned *info) {
    unsigned zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_gemv_error, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(info, g_gemv_error_info, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gemv_error_info, &zero, sizeof(unsigned));
    return e;
}

bool ffn_gemv_can_route(const LayerView &L, int T, int k) {
    int n_sm = 0;
    if (sm_count(&n_sm) != cudaSuccess) return false;
    FfnParams p{};
    p.L = L;
    p.T = T;
    p.k = k;
    return T == 1 && L.E <= 128 && tok_fits(p, n_sm);
}

bool ffn_gemv_can_combine(const LayerView &L, int T, int k) {
    int n_sm = 0;
    if (!ffn_gemv_can_route(L, T, k) || sm_count(&n_sm) != cudaSuccess) return false;
    FfnParams p{};
    p.L = L;
    p.T = T;
    p.k = k;
    return tok_y_floats(p, n_sm) * 4 <= kTokSmemMax;
}

cudaError_t launch_ffn_gemv_routed(const LayerView &L, const uint16_t *x, const float *logits, int k,
                                   uint32_t *hits, int32_t *ids, float *w, int32_t *counts, int32_t *offsets,
                                   int32_t *sorted_route, int32_t *route_pos, float *rows, void *ws,
                                   uint16_t *y, cudaStream_t s) {
    int n_sm = 0;
    cudaError_t err = sm_count(&n_sm);
    if (err != cudaSuccess) return err;
    FfnParams p{};
    p.L = L;
    p.x = x;
    p.T = 1;
    p.k = k;
    p.counts = counts;
    p.offsets = offsets;
    p.sorted_route = sorted_route;
    p.h = static_cast<uint16_t *>(ws);
    p.rows = rows;
    p.logits = logits;
    p.hits = hits;
    p.ids_out = ids;
    p.w_out = w;
    p.counts_out = counts;
    p.offsets_out = offsets;
    p.sorted_out = sorted_route;
    p.pos_out = route_pos;
    p.y = y;
    if (L.fmt == MOE_W_BF16) return launch_fmt<MOE_W_BF16>(p, n_sm, s);
    if (L.fmt == MOE_W_INT8) return launch_fmt<MOE_W_INT8>(p, n_sm, s);
    return launch_fmt<MOE_W_INT4>(p, n_sm, s);
}

cudaError_t launch_ffn_gemv(const LayerView &L, const uint16_t *x, int T, int k, const int32_t *counts,
                            const int32_t *offsets, const int32_t *sorted_route, float *rows, void *ws,
                            cudaStream_t s) {
    int n_sm = 0;
    cudaError_t err = sm_count(&n_sm);
    if (err != cudaSuccess) return err;
    FfnParams p{};
    p.L = L;
    p.x = x;
    p.T = T;
    p.k = k;
    p.counts = counts;
    p.offsets = offsets;
    p.sorted_route = sorted_route;
    p.h = static_cast<uint16_t *>(ws);
    p.rows = rows;
    if (L.fmt == MOE_W_BF16) return launch_fmt<MOE_W_BF16>(p, n_sm, s);
    if (L.fmt == MOE_W_INT8) return launch_fmt<MOE_W_INT8>(p, n_sm, s);
    return launch_fmt<MOE_W_INT4>(p, n_sm, s);
}

}  // namespace moe
