// placement_dev.cu -- the expert residency pool's refresh on the device, and
// the promotion copies it implies (rlx_runtime expert_pool.rs:
// target_gpu_from_counts, then apply_target_placement; the same results as
// moe_refresh_target + moe_apply_placement on the host, bit for bit).
//
// Done on the device, a refresh needs no host round trip: the hit histogram,
// the slot table and the promotion list stay in HBM, the two launches can be
// captured in a CUDA graph, and the copies can run on a second stream while the
// following layers compute (the caller orders the layer's next forward after
// them).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kPlaceThreads = 1024;

// exclusive prefix sum of one int per thread over the whole block (<= 1024
// threads); *total receives the sum
__device__ int block_exclusive_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += u;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int nw = (blockDim.x + 31) >> 5;
        int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += u;
        }
        s_warp[lane] = w;  // inclusive prefix of the warp sums
    }
    __syncthreads();
    const int before = (warp > 0 ? s_warp[warp - 1] : 0) + inc - v;
    *total = s_warp[((blockDim.x + 31) >> 5) - 1];
    __syncthreads();
    return before;
}

// One CTA of kPlaceThreads threads; thread i owns expert i and slot i.
// status[0] = promotions, status[1] = demotions, status[2] = 0, or 1 when the
// slot table was inconsistent (a slot out of range or held twice: then nothing
// is changed and no promotion is listed).
__global__ void __launch_bounds__(kPlaceThreads) k_refresh_placement(const uint32_t *__restrict__ hits, int E,
                                                                     int budget, int32_t *__restrict__ slot_of,
                                                                     int n_slots, int32_t *__restrict__ promo,
                                                                     int32_t *__restrict__ status) {
    __shared__ uint32_t s_hits[kMaxE];
    __shared__ int s_slot[kMaxE];       // slot of expert e before the refresh, or -1
    __shared__ int s_owner[kMaxE];      // expert holding slot s, or -1
    __shared__ int s_by_rank[kMaxE];    // target experts in rank order
    __shared__ int s_demote[kMaxE];     // demote candidates in id order
    __shared__ int s_free[kMaxE];       // initially free slots in slot order
    __shared__ int s_promote[kMaxE];    // promoted experts in rank order
    __shared__ int s_warp[32];
    __shared__ int s_bad;
    const int i = threadIdx.x;
    const bool is_e = i < E, is_s = i < n_slots;
    const int my_slot = is_e ? slot_of[i] : -1;
    if (i == 0) s_bad = 0;
    if (is_e) {
        s_hits[i] = hits[i];
        s_slot[i] = my_slot;
    }
    if (is_s) s_owner[i] = -1;
    __syncthreads();
    if (my_slot >= n_slots) s_bad = 1;
    if (my_slot >= 0 && my_slot < n_slots && atomicCAS(&s_owner[my_slot], -1, i) != -1) s_bad = 1;
    __syncthreads();
    if (s_bad) {
        if (i == 0) {
            status[0] = 0;
            status[1] = 0;
            status[2] = 1;
        }
        return;
    }

    // rank among the experts with hits: count descending, id ascending
    const uint32_t h = is_e ? s_hits[i] : 0u;
    int rank = 0;
    if (h > 0)
        for (int e = 0; e < E; ++e) {
            const uint32_t he = s_hits[e];
            rank += (he > h || (he == h && e < i)) ? 1 : 0;
        }
    int n_hit;
    block_exclusive_scan(h > 0 ? 1 : 0, s_warp, &n_hit);
    const int n_target = min(budget, n_hit);
    const bool in_target = h > 0 && rank < n_target;
    if (in_target) s_by_rank[rank] = i;
    __syncthreads();

    // promotions: targets without a slot, in rank order
    const int te = i < n_target ? s_by_rank[i] : -1;
    const bool prom = te >= 0 && s_slot[te] < 0;
    int n_prom;
    const int pi = block_exclusive_scan(prom ? 1 : 0, s_warp, &n_prom);
    if (prom) s_promote[pi] = te;
    // demote candidates: resident, not in the target, in id order
    const bool cand = my_slot >= 0 && !in_target;
    int n_cand;
    const int di = block_exclusive_scan(cand ? 1 : 0, s_warp, &n_cand);
    if (cand) s_demote[di] = i;
    // free slots, in slot order
    const bool fr = is_s && s_owner[i] < 0;
    int n_free;
    const int fi = block_exclusive_scan(fr ? 1 : 0, s_warp, &n_free);
    if (fr) s_free[fi] = i;
    __syncthreads();

    const int n_dem = min(n_prom, n_cand);
    // the demoted experts lose their slot; promotion j takes demoted expert j's
    // slot, or past the demotions the (j - n_dem)-th free slot
    if (i < n_dem) slot_of[s_demote[i]] = -1;
    if (i < n_prom) {
        const int e = s_promote[i];
        int slot = -1;
        if (i < n_dem) {
            slot = s_slot[s_demote[i]];
        } else if (i - n_dem < n_free) {
            slot = s_free[i - n_dem];
        }
        slot_of[e] = slot;
        promo[2 * i] = e;
        promo[2 * i + 1] = slot;
    }
    if (i == 0) {
        status[0] = n_prom;
        status[1] = n_dem;
        status[2] = 0;
    }
}

// Promotion copies: promo[2j] = expert, promo[2j+1] = slot for j < status[0];
// expert blob e of `home` to slot s of `pool`, 16 bytes per thread and step.
__global__ void __launch_bounds__(256) k_promote_copies(const uint4 *__restrict__ home, uint4 *__restrict__ pool,
                                                        uint64_t blob_vec, const int32_t *__restrict__ promo,
                                                        const int32_t *__restrict__ status, int max_promo) {
    const int n = min(__ldg(status), max_promo);
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (int j = 0; j < n; ++j) {
        const int e = __ldg(promo + 2 * j), sl = __ldg(promo + 2 * j + 1);
        if (e < 0 || sl < 0) continue;
        const uint4 *src = home + (uint64_t)e * blob_vec;
        uint4 *dst = pool + (uint64_t)sl * blob_vec;
        for (uint64_t o = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; o < blob_vec; o += stride)
            dst[o] = __ldg(src + o);
    }
}

}  // namespace

cudaError_t launch_refresh_placement(const uint32_t *hits, int E, int budget, int32_t *slot_of, int n_slots,
                                     int32_t *promo, int32_t *status, cudaStream_t s) {
    k_refresh_placement<<<1, kPlaceThreads, 0, s>>>(hits, E, budget, slot_of, n_slots, promo, status);
    return cudaGetLastError();
}

cudaError_t launch_promote_copies(const void *home, void *pool, uint64_t expert_bytes, const int32_t *promo,
                                  const int32_t *status, int max_promo, cudaStream_t s) {
    int n_sm = 0;
    cudaError_t err = sm_count(&n_sm);
    if (err != cudaSuccess) return err;
    k_promote_copies<<<n_sm * 4, 256, 0, s>>>(static_cast<const uint4 *>(home), static_cast<uint4 *>(pool),
                                             expert_bytes / 16, promo, status, max_promo);
    return cudaGetLastError();
}

}  // namespace moe
