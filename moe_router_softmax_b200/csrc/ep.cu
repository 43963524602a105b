// ep.cu -- expert parallelism across GPUs: the row movement on each side of
// the all-to-all exchanges, and the host plan of their split sizes.
//
// Rank d of N holds experts [d*El, (d+1)*El) of a layer, El = E/N.  This is the
// B200 form of the pages' remote-expert runtime (Winery-Strata
// src/core/remote_experts.cpp: a secondary GPU owns a claimed subset of the
// experts; RemoteExperts::begin groups the routes by expert and stages the
// routed rows for it, RemoteExperts::finish copies the compact result rows back
// to their routes).  Here the staging is a device gather into the sender's
// expert-sorted order, the transfer is the caller's all-to-all (NCCL over
// NVLink), and the owner's grouped FFN reads the received rows in place.
#include <stdint.h>

#include "common.cuh"

namespace moe {
namespace {

// dst row i = src row (index[i] / divisor), copied in 16-byte chunks, for
// 0 <= index[i] / divisor < src_rows; every other row of dst is left as it is.
// One CTA per row, grid-stride over rows.
__global__ void __launch_bounds__(128) k_ep_gather_rows(const uint4 *__restrict__ src, int src_rows, int chunks,
                                                        const int32_t *__restrict__ index, int n, int divisor,
                                                        uint4 *__restrict__ dst) {
    pdl_wait();
    pdl_launch_dependents();
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const int r = __ldg(index + i);
        if (r < 0 || r / divisor >= src_rows) continue;
        const uint4 *s = src + (int64_t)(r / divisor) * chunks;
        uint4 *d = dst + (int64_t)i * chunks;
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) d[c] = __ldg(s + c);
    }
}

// Inclusive scan of one value per thread over a block of up to 1024 threads.
__device__ __forceinline__ int block_inclusive_scan(int v, int *warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        const int nw = (blockDim.x + 31) >> 5;
        int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += u;
        }
        if (lane < nw) warp_tot[lane] = t;
    }
    __syncthreads();
    return v + (warp > 0 ? warp_tot[warp - 1] : 0);
}

// The received rows arrive grouped by source rank and, inside a source, by
// local expert: counts[s*El + e] rows from source s for local expert e.  Row j
// gets the local expert of the (s, e) entry whose range holds it; rows at or
// past the total get -1.  Every CTA scans the m = N*El counts itself (m <=
// 1024, one per thread), then labels a slice of the rows by binary search.
__global__ void __launch_bounds__(1024) k_ep_recv_ids(const int32_t *__restrict__ counts, int m, int El,
                                                      int32_t *__restrict__ ids, int n) {
    __shared__ int start[kMaxE + 1];
    __shared__ int warp_tot[32];
    pdl_wait();
    pdl_launch_dependents();
    const int t = threadIdx.x;
    const int v = t < m ? max(__ldg(counts + t), 0) : 0;
    const int incl = block_inclusive_scan(v, warp_tot);
    if (t < m) start[t] = incl - v;
    if (t == m - 1) start[m] = incl;
    __syncthreads();
    const int total = start[m];
    for (int j = blockIdx.x * blockDim.x + t; j < n; j += gridDim.x * blockDim.x) {
        int out = -1;
        if (j < total) {
            int lo = 0, hi = m - 1;  // the last entry q with start[q] <= j
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (start[mid] <= j) lo = mid;
                else hi = mid - 1;
            }
            out = lo % El;
        }
        ids[j] = out;
    }
}

}  // namespace

}  // namespace moe

using namespace moe;

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

extern "C" {

moe_status moe_gather_rows(const void *src, int32_t src_rows, int32_t row_bytes, const int32_t *index, int32_t n,
                           int32_t divisor, void *dst, moe_stream_t stream) {
    if (n < 0 || src_rows < 0) return set_error(MOE_ERR_INVALID_ARG, "moe_gather_rows: n=%d src_rows=%d", n, src_rows);
    if (row_bytes <= 0 || row_bytes % 16 != 0)
        return set_error(MOE_ERR_INVALID_ARG, "moe_gather_rows: row_bytes=%d must be a positive multiple of 16",
                         row_bytes);
    if (divisor < 1) return set_error(MOE_ERR_INVALID_ARG, "moe_gather_rows: divisor=%d must be >= 1", divisor);
    if (n == 0 || src_rows == 0) return MOE_OK;
    if (!src || !index || !dst) return set_error(MOE_ERR_INVALID_ARG, "moe_gather_rows: NULL pointer");
    if (!aligned16(src) || !aligned16(dst))
        return set_error(MOE_ERR_INVALID_ARG, "moe_gather_rows: src and dst must be 16-byte aligned");
    int n_sm = 0;
    cudaError_t e = sm_count(&n_sm);
    if (e == cudaSuccess) {
        const int grid = n < n_sm * 16 ? n : n_sm * 16;
        e = launch_pdl(k_ep_gather_rows, dim3(grid), dim3(128), 0, (cudaStream_t)stream,
                       static_cast<const uint4 *>(src), (int)src_rows, (int)(row_bytes / 16), index, (int)n,
                       (int)divisor, static_cast<uint4 *>(dst));
    }
    if (e != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "moe_gather_rows launch: %s (CUDA error %d)", cudaGetErrorString(e), (int)e);
    return MOE_OK;
}

moe_status moe_ep_recv_ids(const int32_t *recv_counts, int32_t N, int32_t El, int32_t *ids, int32_t n,
                           moe_stream_t stream) {
    if (N < 1 || El < 1 || (int64_t)N * El > kMaxE)
        return set_error(MOE_ERR_INVALID_ARG, "moe_ep_recv_ids: N=%d El=%d (N*El must be in [1, %d])", N, El, kMaxE);
    if (n < 0) return set_error(MOE_ERR_INVALID_ARG, "moe_ep_recv_ids: n=%d is negative", n);
    if (n == 0) return MOE_OK;
    if (!recv_counts || !ids) return set_error(MOE_ERR_INVALID_ARG, "moe_ep_recv_ids: NULL pointer");
    int n_sm = 0;
    cudaError_t e = sm_count(&n_sm);
    if (e == cudaSuccess) {
        const int blocks = (n + 1023) / 1024;
        e = launch_pdl(k_ep_recv_ids, dim3(blocks < n_sm ? blocks : n_sm), dim3(1024), 0, (cudaStream_t)stream,
                       recv_counts, (int)(N * El), (int)El, ids, (int)n);
    }
    if (e != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "moe_ep_recv_ids launch: %s (CUDA error %d)", cudaGetErrorString(e), (int)e);
    return MOE_OK;
}

moe_status moe_ep_splits(const int32_t *counts, int32_t E, const int32_t *recv_counts, int32_t N, int32_t *send_rows,
                         int32_t *recv_rows) {
    if (!counts || !recv_counts || !send_rows || !recv_rows)
        return set_error(MOE_ERR_INVALID_ARG, "moe_ep_splits: NULL pointer");
    if (E < 1 || E > kMaxE || N < 1 || E % N != 0)
        return set_error(MOE_ERR_INVALID_ARG, "moe_ep_splits: E=%d must be in [1, %d] and a multiple of N=%d", E, kMaxE,
                         N);
    const int El = E / N;
    int64_t send_total = 0, recv_total = 0;
    for (int d = 0; d < N; ++d) {
        int64_t s = 0, r = 0;
        for (int e = 0; e < El; ++e) {
            const int32_t c = counts[d * El + e], q = recv_counts[d * El + e];
            if (c < 0 || q < 0)
                return set_error(MOE_ERR_INVALID_ARG, "moe_ep_splits: negative count for rank %d, local expert %d", d, e);
            s += c;
            r += q;
        }
        send_total += s;
        recv_total += r;
        if (send_total > INT32_MAX || recv_total > INT32_MAX)
            return set_error(MOE_ERR_INVALID_ARG, "moe_ep_splits: row totals do not fit in int32");
        send_rows[d] = (int32_t)s;
        recv_rows[d] = (int32_t)r;
    }
    return MOE_OK;
}

}  // extern "C"
