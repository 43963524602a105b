// permute.cu -- stable counting sort of routes by expert, and the expert-hit
// histogram.
//
// Grouping follows Winery-Strata remote_experts.cpp (RemoteExperts::begin): a
// route r = t*k + j belongs to token r / k, and inside an expert's group the
// routes keep ascending r.  Groups are laid out by ascending expert id (an
// exclusive scan of the counts).  Routes whose id is outside [0,E) are
// dropped, as that page skips them.  The hit histogram is expert_pool.rs's
// count_hits (a bincount that ignores ids >= E).
//
// One CTA of 32 warps.  Warp w owns a contiguous segment of routes; pass 1
// counts each warp's routes per expert with a peer mask (no atomics, so
// the counts and the layout are deterministic); a scan in (expert, warp)
// order gives every warp its base row per expert; pass 2 re-walks the
// segment and places each route at base + its rank among equal ids before it.
// A segment is read in chunks of kChunk rounds of 32 routes, all of a chunk's
// loads issued before the first is used; a segment of one chunk (R <= 32 * 32 *
// kChunk) stays in registers for pass 2, longer ones are read again.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = 32;
constexpr int kChunk = 8;  // rounds of 32 routes a lane holds at once

// The lanes of the warp holding the same value as this lane (what
// __match_any_sync returns), from one ballot per bit: e in [-1, 2^(nbits-1)),
// bit nbits-1 set only for -1.  The match instruction's cost grows with the
// number of distinct values in the warp; with 8 ballots (E = 128) the 8192-route
// permute takes 15 us instead of 22.
__device__ __forceinline__ unsigned peers_of(int e, int nbits) {
    unsigned peers = 0xffffffffu;
    for (int b = 0; b < nbits; ++b) {
        const bool bit = (e >> b) & 1;
        const unsigned m = __ballot_sync(0xffffffffu, bit);
        peers &= bit ? m : ~m;
    }
    return peers;
}

__global__ void __launch_bounds__(1024) k_permute(const int32_t *__restrict__ ids, int R, int E,
                                                  int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                                                  int32_t *__restrict__ sorted_route,
                                                  int32_t *__restrict__ route_pos, uint32_t *__restrict__ hits) {
    extern __shared__ int smem[];
    int *s_w = smem;                    // [kWarps][E] per-warp counts, then bases
    int *s_scan = smem + kWarps * E;    // [1024] scan scratch
    __shared__ int s_total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // programmatic dependent launch: wait for the previous kernel before
    // touching memory, then let the next one be scheduled
    pdl_wait();
    pdl_launch_dependents();

    for (int i = tid; i < kWarps * E; i += blockDim.x) s_w[i] = 0;
    __syncthreads();

    const int seg = (R + kWarps - 1) / kWarps;
    const int r_begin = warp * seg;
    const int r_end = min(R, r_begin + seg);
    const unsigned lt_mask = (1u << lane) - 1u;

    // the ids of one chunk of the segment (-1 past its end or out of [0, E))
    int ev[kChunk];
    auto load_chunk = [&](int base) {
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            const int r = base + 32 * i + lane;
            ev[i] = r < r_end ? __ldg(ids + r) : -1;
        }
#pragma unroll
        for (int i = 0; i < kChunk; ++i)
            if (ev[i] < 0 || ev[i] >= E) ev[i] = -1;
    };
    const bool one_chunk = r_end - r_begin <= 32 * kChunk;
    int nbits = 1;  // value bits of E - 1, plus the bit that marks -1
    while ((1 << (nbits - 1)) < E) ++nbits;

    // pass 1: per-warp counts
    for (int base = r_begin; base < r_end; base += 32 * kChunk) {
        load_chunk(base);
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            if (base + 32 * i >= r_end) break;  // warp-uniform
            const int e = ev[i];
            const unsigned peers = peers_of(e, nbits);
            if (e >= 0 && (peers & lt_mask) == 0) s_w[warp * E + e] += __popc(peers);
        }
    }
    __syncthreads();

    // totals per expert, exclusive scan over experts (E <= 1024 = blockDim)
    int total = 0;
    if (tid < E)
        for (int w = 0; w < kWarps; ++w) total += s_w[w * E + tid];
    // inclusive scan: within each warp by shuffles, then over the 32 warp sums
    int incl = total;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) s_scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int ws = s_scan[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ws, off);
            if (lane >= off) ws += v;
        }
        s_scan[32 + lane] = ws - s_scan[lane];  // exclusive: the warps before
    }
    __syncthreads();
    incl += s_scan[32 + warp];
    const int excl = incl - total;
    if (tid < E) {
        counts[tid] = total;
        offsets[tid] = excl;
        if (hits) hits[tid] += (uint32_t)total;
        int run = excl;
        for (int w = 0; w < kWarps; ++w) {
            int c = s_w[w * E + tid];
            s_w[w * E + tid] = run;
            run += c;
        }
    }
    if (tid == E - 1) {
        offsets[E] = incl;
        s_total = incl;
    }
    __syncthreads();

    // pass 2: stable placement (a one-chunk segment is still in ev)
    for (int base = r_begin; base < r_end; base += 32 * kChunk) {
        if (!one_chunk) load_chunk(base);
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            if (base + 32 * i >= r_end) break;  // warp-uniform
            const int r = base + 32 * i + lane;
            const int e = ev[i];
            const unsigned peers = peers_of(e, nbits);
            if (r < r_end) {
                if (e >= 0) {
                    const int pos = s_w[warp * E + e] + __popc(peers & lt_mask);
                    sorted_route[pos] = r;
                    route_pos[r] = pos;
                } else {
                    route_pos[r] = -1;
                }
            }
            __syncwarp();
            if (e >= 0 && (peers & lt_mask) == 0) s_w[warp * E + e] += __popc(peers);
            __syncwarp();
        }
    }
    for (int i = s_total + tid; i < R; i += blockDim.x) sorted_route[i] = -1;
}

__global__ void k_expert_hits(const int32_t *__restrict__ ids, int64_t n, int E, uint32_t *__restrict__ hits) {
    extern __shared__ unsigned s_h[];
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_h[i] = 0;
    __syncthreads();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        int e = __ldg(ids + i);
        if (e >= 0 && e < E) atomicAdd(&s_h[e], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x)
        if (s_h[i]) atomicAdd(hits + i, s_h[i]);
}

}  // namespace

size_t permute_smem_bytes(int E) { return (size_t)(kWarps * E + 1024) * sizeof(int); }

cudaError_t launch_permute(const int32_t *ids, int R, int E, int32_t *counts, int32_t *offsets,
                           int32_t *sorted_route, int32_t *route_pos, uint32_t *hits, cudaStream_t s) {
    size_t smem = permute_smem_bytes(E);
    static size_t cached[kMaxDevices] = {};  // one-time attribute per device
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (cached[dev] < smem) {
        err = cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        cached[dev] = smem;
    }
    return launch_pdl(k_permute, dim3(1), dim3(1024), smem, s, ids, R, E, counts, offsets, sorted_route, route_pos,
                      hits);
}

cudaError_t launch_expert_hits(const int32_t *ids, int64_t n, int E, uint32_t *hits, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 296) blocks = 296;
    k_expert_hits<<<(unsigned)blocks, 256, (size_t)E * sizeof(unsigned), s>>>(ids, n, E, hits);
    return cudaGetLastError();
}

}  // namespace moe
