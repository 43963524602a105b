// ffn_tc.cu -- grouped gated FFN on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM, operands staged in shared memory by TMA).
//
// The same two steps as the GEMV path (gated GELU-tanh FFN, w13 gate rows
// [0,I) and up rows [I,2I), then w2), as ragged grouped GEMMs with the weight
// rows as the M = 128 operand ("swap AB") and each expert's routes as N:
//   phase 1:  D[128 x N] = [W13 gate rows i0..i0+63 ; up rows i0..i0+63] . Xs^T
//             epilogue h[s][i] = bf16(gelu_tanh(D[i]) * D[64 + i])
//   phase 2:  D[128 x N] = W2[m0..m0+127] . h^T,   epilogue rows[s][m] = D[m]
// Xs is x gathered into sorted-route order (k_gather_rows), so every B tile is
// a plain 2-D TMA box.  For bf16 weights TMA writes the A tile straight into
// the 128-byte-swizzled K-major layout the MMA reads from shared memory.
// int8/int4 codes land raw (128-byte swizzled, so the dequant warps read them
// without bank conflicts); a group of eight dequant warps expands each stage
// into bf16 (int8 codes exactly, with the per-row scale applied in the
// epilogue; int4 as bf16(q * s) with the group scale, one rounding) and stores
// it in tensor memory, where the MMA takes its A operand: the expanded weights
// never touch shared memory, whose bandwidth the MMAs' operand reads would
// otherwise share with the expansion.
//
// Persistent CTAs (one per SM, or two for int8/int4 decode batches: TcCfg);
// warp roles:
//   warp 0      TMA producer of A: the weight tiles (bf16) or the raw codes
//               (int8 / int4)
//   warp 1      TMEM allocation and the single-thread MMA issuer
//   warps 2..5  epilogue (TMEM -> registers -> global); warp w reads TMEM
//               lanes 32*(w%4) .. +31
//   warp 6      TMA producer of B: the routes' activation tiles
//   warps 7..   dequantisation (int8 / int4 only): groups of eight warps taking
//               alternate stages (two groups, or one with two CTAs per SM)
// Pipelines: separate rings for A, B and (int formats) raw codes, each with
// full / empty mbarriers, so a slow operand never holds the other's slots; B
// slots are sized by the busiest expert's route count, so small decode blocks
// get many stages in flight; two TMEM accumulators (full / empty) let the
// epilogue of one item overlap the main loop of the next.  Launches are
// programmatic dependent launches: only the B producer waits for the previous
// kernel.  Every mbarrier wait is bounded (and suspends in hardware while it
// waits); on timeout the kernel records an error word and every role drains
// out.  The weight loads carry an evict-first L2 policy (each weight is read
// once) and the route-tile loads an evict-last one (every M tile of an expert
// re-reads them), so the weight stream does not push xs and h out of L2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kBlockM = 128;          // weight rows per tile (TMEM lanes)
constexpr int kBlockK = 64;           // bf16 elements per swizzle atom = one 128-byte swizzle row
constexpr int kNMax = 128;            // max routes per block (TMEM columns per accumulator)
constexpr int kAccBufs = 2;
constexpr int kAccCols = kNMax * kAccBufs;   // TMEM columns of the accumulators
constexpr int kEpiWarps = 4;
constexpr int kDeqWarps = 8;          // per group: two threads per tile row, one 64-wide atom each
constexpr uint32_t kATileBytes = kBlockM * kBlockK * 2;   // 16 KB
constexpr int kMaxBSlots = 32;
constexpr int kRawRowBytes = 128;     // per raw stage row
constexpr long long kWaitCycles = 4000000000ll;           // ~2 s at 2 GHz
constexpr long long kReadySpins = 8000000ll;              // phase 2's wait for an expert's h: > 1 s of 128-ns sleeps
constexpr int kXPitch = 17;                               // exchange row pitch (floats): no bank conflicts

// Three rings of stages, each with its own full / empty mbarriers, so no
// operand's load latency holds another's slots:
//  A:   kAStages weight tiles of 128 rows x kKS bf16 (bf16 weights: TMA into
//       shared memory; int8/int4: the dequant warps, into tensor memory);
//  B:   up to kMaxBSlots activation tiles of n_block rows x kKS bf16 (TMA), as
//       many as fit in kBRegion bytes for this launch's route block;
//  raw: kRawStages stages of 128 code bytes per row (int formats: 256 int4 or
//       128 int8 weights, kSub A stages each), whole 128-byte runs of a row.
// For int8 / int4 the A ring lives in tensor memory instead (kASmem = 0): the
// dequant warps store the bf16 tiles with tcgen05.st and the MMAs read A from
// TMEM, so the expanded weights never pass through shared memory.
// A stage covers kKS = 128 of K (two 64-wide swizzle atoms), so that the
// single MMA-issuing thread pays one round of barrier waits and commits per 8
// MMAs instead of per 4 (each tcgen05 instruction and each barrier wait costs
// that thread tens of nanoseconds, which otherwise bounds a decode batch's
// small MMAs).
// kSub A stages share one raw stage of kRawRowBytes per row (kSubBytes each).
template <int FMT> struct TcFmt;
template <> struct TcFmt<MOE_W_BF16> {
    static constexpr int kKS = 128, kSub = 1, kSubBytes = 0, kAStages = 4, kASmem = 1, kRawStages = 0;
    static constexpr int kBRegion = 64 * 1024, kTmemCols = kAccCols;
};
template <> struct TcFmt<MOE_W_INT8> {
    static constexpr int kKS = 128, kSub = 1, kSubBytes = 128, kAStages = 4, kASmem = 0, kRawStages = 6;
    static constexpr int kBRegion = 96 * 1024, kTmemCols = 512;  // accumulators, then 4 A stages of 64 columns
};
template <> struct TcFmt<MOE_W_INT4> {
    static constexpr int kKS = 128, kSub = 2, kSubBytes = 64, kAStages = 4, kASmem = 0, kRawStages = 6;
    static constexpr int kBRegion = 96 * 1024, kTmemCols = 512;
};

// Launch configuration.  CFG 0: one CTA per SM (above).  CFG 1, for int8/int4
// decode batches (route blocks <= 64): two CTAs per SM, each with half the
// accumulator width, one dequant group, shallower rings and half the tensor
// memory -- two MMA-issuing threads per SM, which is what bounds the int formats
// at decode (measured 16-19% faster at 64 tokens; the prefill case needs the
// wider accumulators and stays on CFG 0).
template <int FMT, int CFG> struct TcCfg : TcFmt<FMT> {
    static constexpr int kNMax = 128, kDeqGroups = 2, kMinBlocks = 1;
    static constexpr int kAccCols = kNMax * kAccBufs;
};
template <int FMT> struct TcCfg<FMT, 1> : TcFmt<FMT> {
    static constexpr int kNMax = 64, kDeqGroups = 1, kMinBlocks = 2;
    static constexpr int kAccCols = kNMax * kAccBufs;
    static constexpr int kAStages = 2, kRawStages = 3, kBRegion = 32 * 1024, kTmemCols = 256;
};

// First problem a tensor-core kernel recorded (0 = none): 0x1000 | role for
// a bounded wait that gave up; 0x2000 | site for an index check that failed
// (the access is skipped).  Read and cleared by moe_take_device_errors().
__device__ unsigned int g_tc_error;
__device__ unsigned int g_tc_error_info;
__device__ __forceinline__ void record_error(unsigned code, unsigned info) {
    if (atomicCAS(&g_tc_error, 0u, code) == 0u) g_tc_error_info = info;
}

struct TcParams {
    LayerView L;
    int R;                 // rows of xs / h / rows (T * k)
    const int32_t *counts, *offsets;
    int n_block;           // cap on the route block (multiple of 16, <= kNMax)
    int K;                 // reduction length: H (phase 1) or I (phase 2)
    int n_units;           // output rows of the weight: 2I (phase 1) or H (phase 2)
    uint16_t *h;           // [R][I] bf16: phase-1 output
    float *rows;           // [R][H] fp32: phase-2 output
    // per expert, h values published by phase 1: each of an item's two gate-row
    // epilogue warps adds the item's route count once its h entries are written,
    // so expert e is complete at 2 * (I / 64) * counts[e]; zeroed by the gather
    unsigned *ready;
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// try_wait suspends the thread in hardware until the phase completes or the
// hint (ns) expires, so waiting roles do not spin on the issue slots.
constexpr uint32_t kSuspendNs = 100000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}
// Non-blocking test of a phase (the common case: it has already completed).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false (and the abort flag set) if the phase did not complete in
// time or another role already gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_test_wait(bar, parity)) return true;
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
            *abort_flag = 1;
            record_error(0x1000u | (threadIdx.x >> 5), (unsigned)((smem_u32(bar) << 1) | (parity & 1)));
            return false;
        }
    }
}
// Bounded wait that ignores the abort flag (for the drain after an abort).
__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity, long long cycles) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > cycles) return false;
    return true;
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// L2 policies: the weight stream is read once (evict first); the route tiles
// are re-read by every M tile of an expert (evict last).
__device__ __forceinline__ uint64_t l2_policy_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Stores of the intermediates a later launch re-reads (xs by every M tile of
// phase 1, h by every M tile of phase 2) with the evict-last policy, so they
// stay in L2 beside the evict-first weight stream instead of going to DRAM
// and back.
__device__ __forceinline__ void st_v4_hint(void *dst, uint4 u, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst), "r"(u.x), "r"(u.y),
                 "r"(u.z), "r"(u.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_u16_hint(uint16_t *dst, uint16_t v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.u16 [%0], %1, %2;" ::"l"(dst), "h"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                            uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;"
        ::"r"(smem_u32(smem_dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(pol)
        : "memory");
}
// 3-D box {x, y, z} of a weight map: x along the row, y the row of the matrix,
// z the blob (expert or pool slot).  Coordinates past an extent read zeros.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                            int z, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;"
        ::"r"(smem_u32(smem_dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// A from tensor memory (columns a_tmem.. of lanes 0..127, bf16 pairs), B from
// shared memory.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 16 consecutive 32-bit columns of this thread's TMEM lane (asynchronous:
// tmem_st_wait() orders them before what follows).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float v[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float gelu_tanh(float v) {
    const float c = 0.7978845608028654f;  // sqrt(2/pi)
    const float u = c * (v + 0.044715f * v * v * v);
    return 0.5f * v * (1.0f + tanhf(u));
}


// ------------------------------------------------------------- work items
// Item = (active expert a, block of <= kNMax of its routes, M tile); M tiles
// fastest so the CTAs working on one expert share its activation tiles in L2.
// The route block n_block (rows of one B tile, columns of one accumulator) is
// the busiest expert's route count rounded up to 16, capped by p.n_block: every
// expert then fits one block, and a decode batch whose experts hold a handful of
// routes gets small B slots, so many B stages are in flight.
struct Items {
    int n_act, total, m_tiles, n_block, b_rows, b_slots;
};

// Called by every thread of the CTA (it holds a __syncthreads).  The counts are
// read in one round of loads by the whole CTA into s_base, which warp 0 then
// overwrites in place with the item prefix (a write at position pos <= e never
// reaches a count not yet read: reads run ahead in e).
__device__ void build_items(const TcParams &p, int m_tiles, int b_region, int atoms, int *s_act, int *s_base,
                            Items *it) {
    const int lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < p.L.E; e += blockDim.x) s_base[e] = __ldg(p.counts + e);
    __syncthreads();
    if (threadIdx.x < 32) {
        int n_max = 1;
        for (int e = lane; e < p.L.E; e += 32) n_max = max(n_max, s_base[e]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) n_max = max(n_max, __shfl_xor_sync(0xffffffffu, n_max, off));
        const int n_block = min(p.n_block, (n_max + 15) & ~15);
        int n_act = 0, run = 0;
        for (int e0 = 0; e0 < p.L.E; e0 += 32) {
            const int e = e0 + lane;
            const int n = (e < p.L.E) ? s_base[e] : 0;
            __syncwarp();  // every lane has read its count before any prefix is written
            const bool act = n > 0;
            const unsigned m = __ballot_sync(0xffffffffu, act);
            const int items = act ? m_tiles * ((n + n_block - 1) / n_block) : 0;
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
            s_base[n_act] = run;
            it->n_act = n_act;
            it->total = run;
            it->m_tiles = m_tiles;
            it->n_block = n_block;
            // B slot rows: a block over 32 routes is loaded in 64-row boxes (two to
            // four TMA instructions per stage instead of up to sixteen)
            const int b_rows = n_block <= 32 ? n_block : (n_block + 63) & ~63;
            it->b_rows = b_rows;
            it->b_slots = min(kMaxBSlots, b_region / (b_rows * 128 * atoms));
        }
    }
}

struct ItemInfo {
    int e, row0, n, n_mma, m0;
};

__device__ __forceinline__ ItemInfo decode_item(const TcParams &p, const int *s_act, const int *s_base, int n_act,
                                                int m_tiles, int n_block, int item) {
    int lo = 0, hi = n_act - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_base[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int rem = item - s_base[lo];
    const int nb = rem / m_tiles, mt = rem - nb * m_tiles;
    ItemInfo r;
    r.e = s_act[lo];
    const int n_e = __ldg(p.counts + r.e);
    r.row0 = __ldg(p.offsets + r.e) + nb * n_block;
    r.n = min(n_block, n_e - nb * n_block);
    r.n_mma = (r.n + 15) & ~15;
    bool bad_slot;
    expert_slot(p.L, r.e, &bad_slot);
    if (bad_slot) record_error(0x2006u, (unsigned)__ldg(p.L.slot_table + r.e));
    if (r.n <= 0 || r.n_mma > n_block || r.row0 < 0 || r.row0 + r.n > p.R || bad_slot) {
        if (!bad_slot) record_error(0x2003u, (unsigned)item);
        r.n = 0;       // nothing is written for an item that fails the check (its
        r.n_mma = 16;  // weights are read from home), and its tiles stay inside
        r.row0 = 0;    // their slots
    }
    r.m0 = mt;  // tile index; callers scale it
    return r;
}

// Blob coordinate (z) of expert e in the home or pool weight map.  An expert
// whose slot is past the pool is read from home (its item writes nothing).
__device__ __forceinline__ int a_blob_coord(const TcParams &p, int e, bool *in_pool) {
    bool bad;
    const int s = expert_slot(p.L, e, &bad);
    *in_pool = s >= 0;
    return s >= 0 ? s : e;
}

// Blob of expert e for the scale reads; home for an expert whose slot is past
// the pool (its item writes nothing).
__device__ __forceinline__ const uint8_t *scale_blob(const TcParams &p, int e) {
    const uint8_t *b = expert_blob(p.L, e);
    return b ? b : p.L.home + (uint64_t)e * p.L.stride;
}

// Storage column of K element c in the int4 kernels' B operand (xs, h): within
// every run of 8, elements 1 and 2, 5 and 6 trade places (the order in which
// the int4 expansion lays out A; an involution).  Identity for bf16 and int8.
template <int FMT>
__host__ __device__ __forceinline__ int k_order(int c) {
    return FMT == MOE_W_INT4 ? ((c & ~3) | ((c & 1) << 1) | ((c >> 1) & 1)) : c;
}

// ---------------------------------------------------------------- the kernel
template <int FMT>
__host__ __device__ constexpr int kRawBytes() { return FMT == MOE_W_BF16 ? 0 : kRawRowBytes * kBlockM; }

// warps: 0 A/raw producer, 1 MMA, 2..5 epilogue, 6 B producer, 7.. dequant
// (kDeqGroups groups of kDeqWarps), then one gate warp per dequant group
constexpr int kWarpB = 2 + kEpiWarps;
constexpr int kWarpDeq0 = kWarpB + 1;

template <int FMT, int CFG>
__host__ __device__ constexpr int tc_threads() {
    return 32 * (kWarpDeq0 + (FMT == MOE_W_BF16 ? 0 : TcCfg<FMT, CFG>::kDeqGroups * (kDeqWarps + 1)));
}

// Named hardware barriers between a dequant group's gate warp and its eight
// warps (id 0 is __syncthreads): one per (group, A slot).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int FMT, int PHASE, int CFG>
__global__ void __launch_bounds__(tc_threads<FMT, CFG>(), TcCfg<FMT, CFG>::kMinBlocks)
k_ffn_tc(const __grid_constant__ CUtensorMap map_home, const __grid_constant__ CUtensorMap map_pool,
         const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_b64, const TcParams p) {
    using C = TcCfg<FMT, CFG>;
    constexpr int SA = C::kAStages;
    constexpr int SR = C::kRawStages;
    constexpr int RAW = kRawBytes<FMT>();
    constexpr int SUB = C::kSub;
    constexpr bool kDeq = FMT != MOE_W_BF16;
    constexpr int KS = C::kKS, ATOMS = KS / kBlockK;
    constexpr int A_COLS = KS / 2;  // TMEM columns of one A stage (int formats: bf16 pairs)

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned carve-up: A ring | B region | raw ring | exchange | barriers
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = sA + (C::kASmem ? SA * ATOMS * kATileBytes : 0);
    uint8_t *sRaw = sB + C::kBRegion;
    float *sX = reinterpret_cast<float *>(sRaw + SR * RAW);       // [2][64][kXPitch] gate/up exchange
    uint64_t *bars = reinterpret_cast<uint64_t *>(sX + 2 * 64 * kXPitch);
    uint64_t *a_full = bars;                       // A tile ready (TMA bytes, or the dequant warps)
    uint64_t *a_empty = a_full + SA;               // MMAs done reading the A tile
    uint64_t *b_full = a_empty + SA;               // B tile landed
    uint64_t *b_empty = b_full + kMaxBSlots;       // MMAs done reading the B tile
    uint64_t *tfull = b_empty + kMaxBSlots;        // accumulator ready
    uint64_t *tempty = tfull + kAccBufs;           // accumulator drained
    uint64_t *xfull = tempty + kAccBufs;           // up values written to the exchange
    uint64_t *xempty = xfull + 2;                  // exchange read by the gate warps
    uint64_t *r_full = xempty + 2;                 // raw codes landed (int formats)
    uint64_t *r_empty = r_full + SR;               // raw codes consumed by the dequant warps

    __shared__ int s_act[kMaxE];
    __shared__ int s_base[kMaxE + 1];
    __shared__ Items s_items;
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tiles = PHASE == 1 ? p.L.I / 64 : (p.L.H + kBlockM - 1) / kBlockM;
    // The next launch (phase 2 after phase 1, the combine after phase 2) may
    // take over SMs as this grid's CTAs finish; it waits for this grid's
    // results itself where it reads them.  Phase 1 releases phase 2 only from its
    // B producer, once the gather has completed: phase 2 reads the per-expert
    // counters the gather zeroes.
    constexpr bool kEarly = FMT == MOE_W_BF16;  // phase 2 starts per expert (see the B producer)
    if (PHASE == 2 || !kEarly) pdl_launch_dependents();
    const int nk = (p.K + KS - 1) / KS;  // stages; the last may hold fewer atoms (p.K is a multiple of 64)
    auto atoms_at = [&](int kk) { return min(ATOMS, (p.K - kk * KS) / kBlockK); };

    if (threadIdx.x == 0) {
        for (int i = 0; i < SA; ++i) {
            mbar_init(&a_full[i], kDeq ? kDeqWarps + 1 : 1);  // int: eight dequant warps and the gate
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < kMaxBSlots; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&xfull[b], 2);
            mbar_init(&xempty[b], 2);
        }
        for (int r = 0; r < SR; ++r) {
            mbar_init(&r_full[r], 1);
            mbar_init(&r_empty[r], C::kDeqGroups * kDeqWarps);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(C::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    build_items(p, m_tiles, C::kBRegion, ATOMS, s_act, s_base, &s_items);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int n_act = s_items.n_act, total = s_items.total;
    const int n_block = s_items.n_block, b_slots = s_items.b_slots;
    // With a small route block the four 16-wide K steps of a 64-wide atom go
    // to nacc separate partial accumulators (n_block columns apart inside the
    // accumulator's C::kNMax columns), which the epilogue adds up, so that
    // consecutive MMAs do not update the same small tile.
    const int nacc = n_block <= C::kNMax / 4 ? 4 : (n_block <= C::kNMax / 2 ? 2 : 1);
    const uint32_t b_atom_bytes = (uint32_t)s_items.b_rows * 128;  // one 64-wide atom of a B slot
    const uint32_t b_slot_bytes = b_atom_bytes * ATOMS;

    if (warp == 0) {
        // ------------------------------------- A producer: weights or raw codes
        if (lane == 0) {
            const uint64_t pol = l2_policy_first();
            int stage = 0;
            uint32_t phase = 0;
            for (int item = blockIdx.x; item < total && !s_abort; item += gridDim.x) {
                const ItemInfo it = decode_item(p, s_act, s_base, n_act, m_tiles, n_block, item);
                bool pool;
                const int za = a_blob_coord(p, it.e, &pool);
                int ya0, ya1;  // rows of the matrix of the two 64-row halves of the tile
                if (PHASE == 1) {
                    ya0 = it.m0 * 64;
                    ya1 = p.L.I + it.m0 * 64;
                } else {
                    ya0 = it.m0 * kBlockM;
                    ya1 = ya0 + 64;
                }
                const CUtensorMap *ma = pool ? &map_pool : &map_home;
                bool ok = true;
                if (kDeq) {
                    for (int rs = 0; rs < (nk + SUB - 1) / SUB; ++rs) {
                        if (!mbar_wait(&r_empty[stage], phase ^ 1, &s_abort)) { ok = false; break; }
                        mbar_arrive_expect_tx(&r_full[stage], (uint32_t)RAW);
                        uint8_t *dst = sRaw + stage * RAW;
                        tma_load_3d(dst, ma, &r_full[stage], rs * kRawRowBytes, ya0, za, pol);
                        tma_load_3d(dst + 64 * kRawRowBytes, ma, &r_full[stage], rs * kRawRowBytes, ya1, za, pol);
                        if (++stage == SR) { stage = 0; phase ^= 1; }
                    }
                } else {
                    for (int kk = 0; kk < nk; ++kk) {
                        const int na = atoms_at(kk);
                        if (!mbar_wait(&a_empty[stage], phase ^ 1, &s_abort)) { ok = false; break; }
                        mbar_arrive_expect_tx(&a_full[stage], (uint32_t)na * kATileBytes);
                        for (int a = 0; a < na; ++a) {
                            uint8_t *dst = sA + (stage * ATOMS + a) * kATileBytes;
                            tma_load_3d(dst, ma, &a_full[stage], (kk * ATOMS + a) * kBlockK, ya0, za, pol);
                            tma_load_3d(dst + kATileBytes / 2, ma, &a_full[stage], (kk * ATOMS + a) * kBlockK, ya1,
                                        za, pol);
                        }
                        if (++stage == SA) { stage = 0; phase ^= 1; }
                    }
                }
                if (!ok) break;
            }
        }
    } else if (warp == kWarpB) {
        // ------------------------------------------------ B producer: routes
        if (lane == 0) {
            // the B operand is the one input an earlier launch writes.  Phase 1
            // (xs from k_gather_rows) waits for the gather here, while the other
            // roles already stream weights.  Phase 2 (h) waits per item only for
            // the phase-1 items of the item's expert, through the counters, so it
            // starts while phase 1's last items still run elsewhere.
            if (PHASE == 1 || !kEarly) pdl_wait();
            if (PHASE == 1 && kEarly) pdl_launch_dependents();
            const uint64_t pol = l2_policy_last();
            int stage = 0;
            uint32_t phase = 0;
            for (int item = blockIdx.x; item < total && !s_abort; item += gridDim.x) {
                const ItemInfo it = decode_item(p, s_act, s_base, n_act, m_tiles, n_block, item);
                bool ok = true;
                if (kEarly && PHASE == 2) {
                    const unsigned target = 2u * (unsigned)(p.L.I / 64) * (unsigned)__ldg(p.counts + it.e);
                    long long spins = 0;
                    while (ld_acquire_gpu(p.ready + it.e) < target) {
                        if (++spins > kReadySpins || s_abort) {
                            if (!s_abort) record_error(0x1000u | (unsigned)kWarpB, (unsigned)it.e);
                            s_abort = 1;
                            ok = false;
                            break;
                        }
                        __nanosleep(128);
                    }
                    if (!ok) break;
                    // h was written through the generic proxy by other CTAs; the
                    // route tiles are read by TMA (the async proxy)
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                // up to 32 routes: 16-row boxes; more: 64-row boxes (rows past
                // the block are another expert's or out of range and zero-filled;
                // the slot holds them, the MMAs read only the first n_mma)
                const bool big = it.n_mma > 32 && p.R >= 64;  // the 64-row map exists from 64 rows
                const int rows_ld = big ? (it.n_mma + 63) & ~63 : it.n_mma;
                for (int kk = 0; kk < nk; ++kk) {
                    const int na = atoms_at(kk);
                    if (!mbar_wait(&b_empty[stage], phase ^ 1, &s_abort)) { ok = false; break; }
                    mbar_arrive_expect_tx(&b_full[stage], (uint32_t)(na * rows_ld * 128));
                    uint8_t *db = sB + stage * b_slot_bytes;
                    for (int a = 0; a < na; ++a)
                        for (int j = 0; j < rows_ld; j += big ? 64 : 16)
                            tma_load_2d(db + a * b_atom_bytes + j * 128, big ? &map_b64 : &map_b, &b_full[stage],
                                        (kk * ATOMS + a) * kBlockK, it.row0 + j, pol);
                    if (++stage == b_slots) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int sa = 0, sb = 0;
            uint32_t pa = 0, pb = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            // K step j of an atom accumulates into partial accumulator j % nacc
            // (columns dj[j]); it overwrites it on the atom's first use (j < nacc).
            // nacc is 1, 2 or 4: a mask and a shift, no division per MMA.
            const int lg_acc = nacc == 4 ? 2 : (nacc == 2 ? 1 : 0);
            uint32_t dj[kBlockK / 16];
#pragma unroll
            for (int j = 0; j < kBlockK / 16; ++j) dj[j] = (uint32_t)((j & (nacc - 1)) * n_block);
            for (int item = blockIdx.x; item < total && !s_abort; item += gridDim.x) {
                const ItemInfo it = decode_item(p, s_act, s_base, n_act, m_tiles, n_block, item);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, &s_abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * C::kNMax);
                const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(it.n_mma >> 3) << 17) |
                                       ((uint32_t)(kBlockM >> 4) << 24);
                bool ok = true;
                for (int kk = 0; kk < nk; ++kk) {
                    if (!mbar_wait(&a_full[sa], pa, &s_abort)) { ok = false; break; }
                    // int formats: the dequant warps saw this B slot land before
                    // they completed a_full, so only bf16 waits for it here
                    if (!kDeq && !mbar_wait(&b_full[sb], pb, &s_abort)) { ok = false; break; }
                    tc_fence_after();
                    // descriptors of the stage's first K step; one 16-wide K step is 32
                    // bytes, 2 in the descriptor's start-address field (which cannot
                    // carry: every address stays below 256 KB)
                    const uint64_t bd = sw128_desc(smem_u32(sB + sb * b_slot_bytes));
                    const int na = atoms_at(kk);
                    if (kDeq) {
                        // A stage sa: TMEM columns C::kAccCols + A_COLS sa .., 32 per atom,
                        // 8 per 16-wide K step
                        const uint32_t a_t = tmem + (uint32_t)(C::kAccCols + sa * A_COLS);
                        for (int a = 0; a < na; ++a) {
                            const uint64_t bda = bd + (uint64_t)((a * b_atom_bytes) >> 4);
#pragma unroll
                            for (int j = 0; j < kBlockK / 16; ++j)
                                tc_mma_bf16_ts(d + dj[j], a_t + 32 * a + 8 * j, bda + (uint64_t)(2 * j), idesc,
                                               (kk | a | (j >> lg_acc)) != 0);
                        }
                    } else {
                        const uint64_t ad = sw128_desc(smem_u32(sA + sa * ATOMS * kATileBytes));
                        for (int a = 0; a < na; ++a) {
                            const uint64_t ada = ad + (uint64_t)((a * kATileBytes) >> 4);
                            const uint64_t bda = bd + (uint64_t)((a * b_atom_bytes) >> 4);
#pragma unroll
                            for (int j = 0; j < kBlockK / 16; ++j)
                                tc_mma_bf16(d + dj[j], ada + (uint64_t)(2 * j), bda + (uint64_t)(2 * j), idesc,
                                            (kk | a | (j >> lg_acc)) != 0);
                        }
                    }
                    tc_commit(&a_empty[sa]);
                    tc_commit(&b_empty[sb]);
                    if (++sa == SA) { sa = 0; pa ^= 1; }
                    if (++sb == b_slots) { sb = 0; pb ^= 1; }
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
                if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1; }
            }
        }
    } else if (warp < 2 + kEpiWarps) {
        // --------------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int lrow = q * 32 + lane;         // tile row held by this thread
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t xcount = 0;  // exchange chunks used so far (buffer = xcount & 1)
        const uint64_t h_pol = l2_policy_last();
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok && !s_abort; item += gridDim.x) {
            const ItemInfo it = decode_item(p, s_act, s_base, n_act, m_tiles, n_block, item);
            if (!mbar_wait(&tfull[acc], acc_phase, &s_abort)) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::kNMax);
            const uint8_t *blob = scale_blob(p, it.e);
            float scale = 1.0f;
            if (FMT == MOE_W_INT8) {
                const int wrow = PHASE == 1 ? (lrow < 64 ? it.m0 * 64 + lrow : p.L.I + it.m0 * 64 + lrow - 64)
                                            : min(it.m0 * kBlockM + lrow, p.n_units - 1);
                scale = __ldg(reinterpret_cast<const float *>(blob + (PHASE == 1 ? p.L.off.s13 : p.L.off.s2)) + wrow);
            }
            for (int c0 = 0; c0 < it.n_mma; c0 += 16) {
                float v[16];
                tmem_ld16(taddr + (uint32_t)c0, v);
                for (int pa = 1; pa < nacc; ++pa) {
                    float w[16];
                    tmem_ld16(taddr + (uint32_t)(pa * n_block + c0), w);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] += w[i];
                }
                if (PHASE == 1) {
                    // tile rows 64..127 hold the up projection, rows 0..63 the gate of
                    // the same intermediate columns: the up warps pass their values
                    // through shared memory to the gate warps
                    const uint32_t xb = xcount & 1, xpar = (xcount >> 1) & 1;
                    float *xrow = sX + (size_t)xb * 64 * kXPitch + (size_t)(lrow & 63) * kXPitch;
                    if (lrow >= 64) {
                        if (!mbar_wait(&xempty[xb], xpar ^ 1, &s_abort)) { ok = false; break; }
#pragma unroll
                        for (int i = 0; i < 16; ++i) xrow[i] = v[i] * scale;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&xfull[xb]);
                    } else {
                        if (!mbar_wait(&xfull[xb], xpar, &s_abort)) { ok = false; break; }
                        const int icol = it.m0 * 64 + lrow;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int j = c0 + i;
                            if (j < it.n) {
                                if (it.row0 + j >= p.R || icol >= p.L.I || it.row0 + j < 0) {
                                    record_error(0x2001u, (unsigned)(it.row0 + j));
                                    continue;
                                }
                                const float g = v[i] * scale, up = xrow[i];
                                st_u16_hint(p.h + (size_t)(it.row0 + j) * p.L.I + k_order<FMT>(icol),
                                            f32_to_bf16_rne(gelu_tanh(g) * up), h_pol);
                            }
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&xempty[xb]);
                    }
                    ++xcount;
                } else {
                    const int m = it.m0 * kBlockM + lrow;
                    if (m < p.L.H) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int j = c0 + i;
                            if (j < it.n) {
                                if (it.row0 + j >= p.R || it.row0 + j < 0) {
                                    record_error(0x2002u, (unsigned)(it.row0 + j));
                                    continue;
                                }
                                p.rows[(size_t)(it.row0 + j) * p.L.H + m] = v[i] * scale;
                            }
                        }
                    }
                }
            }
            if (!ok) break;
            if (kEarly && PHASE == 1 && lrow < 64) {
                // this warp's h entries of the item are written: publish them
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(p.ready + it.e, (unsigned)it.n);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1; }
        }
    } else if (kDeq && warp >= kWarpDeq0 + C::kDeqGroups * kDeqWarps) {
        // ---------------------------------------------------- gate warps
        // One per dequant group: for each of the group's stages it waits until
        // the codes have landed and the MMAs are done with the A slot, releases
        // the group's eight warps through a named barrier, then waits for the
        // stage's B slot and arrives on a_full with them.  Every mbarrier wait
        // costs a warp ~130 cycles even when the phase has completed; taking all
        // of them here leaves the dequant warps one hardware barrier per stage.
        // The gate never skips a release (after an abort it releases without
        // waiting), so the dequant warps cannot block on a stage that is never
        // released.
        const int group = warp - (kWarpDeq0 + C::kDeqGroups * kDeqWarps);
        int stage = 0, rstage = 0, bstage = 0;
        uint32_t phase = 0, rphase = 0, bphase = 0;
        uint32_t step = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x) {
            for (int kk = 0; kk < nk; ++kk, ++step) {
                const int sub = kk % SUB;
                const bool raw_last = sub == SUB - 1 || kk == nk - 1;
                if ((int)(step % C::kDeqGroups) == group) {
                    bool ok = !s_abort;
                    // a single group takes both halves of an int4 raw stage and
                    // waits for its codes once; two groups each wait for their half
                    if (ok && (sub == 0 || C::kDeqGroups > 1)) ok = mbar_wait(&r_full[rstage], rphase, &s_abort);
                    if (ok) ok = mbar_wait(&a_empty[stage], phase ^ 1, &s_abort);
                    // after an abort the slot's waits are skipped, so make sure the
                    // group has left this slot's previous release (its warps and
                    // this gate arrive on a_full after every release) before
                    // releasing it again: a named barrier must never collect two
                    // releases at once
                    if (!ok) mbar_wait_for(&a_full[stage], phase ^ 1, kWaitCycles / 4);
                    __syncwarp();
                    named_arrive(1 + group * SA + stage, 32 * (kDeqWarps + 1));
                    // while the group expands the stage, wait for its B slot; the
                    // gate's own arrival on a_full then tells the MMA issuer that A
                    // and B are both ready
                    if (ok) mbar_wait(&b_full[bstage], bphase, &s_abort);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&a_full[stage]);
                }
                if (++stage == SA) { stage = 0; phase ^= 1; }
                if (++bstage == b_slots) { bstage = 0; bphase ^= 1; }
                if (raw_last && ++rstage == SR) { rstage = 0; rphase ^= 1; }
            }
        }
    } else if (kDeq) {
        // ---------------------------------------------------- dequantisation
        // two threads per tile row, each expanding one 64-wide atom of the
        // stage (64 weights): raw codes -> 32 bf16 pairs -> TMEM lane r,
        // columns 32 hf .. 32 hf + 31 of the A stage.  A warp may only reach
        // TMEM lanes 32 (warp % 4) .. +31, so the row is taken from the warp's
        // lane quadrant; the eight warps of a group cover each quadrant twice
        // (both atoms of its rows).  A stage starts when the group's gate warp
        // releases it (codes, A slot and B slot all ready), so a completed
        // a_full means A and B are both ready for the MMAs.
        const int dw = warp - kWarpDeq0;              // 0 .. C::kDeqGroups*kDeqWarps-1
        const int group = dw / kDeqWarps;
        const int quad = warp & 3;
        const int r = quad * 32 + lane, hf = (dw % kDeqWarps) / 4;
        int stage = 0, rstage = 0;
        uint32_t step = 0;                              // stages seen, across items
        int a_cur = 0;                                  // active expert of the current item
        for (int item = blockIdx.x; item < total; item += gridDim.x) {
            // int4: the group scale of this thread's atom is loaded one of the
            // group's stages ahead (the scales are read from global memory, where
            // a miss costs a few hundred cycles that the current stage then hides).
            // int8 needs nothing per item here (its scale is the epilogue's), so
            // its warps skip decoding the item: that alone is 4% at decode.
            const uint16_t *srow = nullptr;
            if (FMT == MOE_W_INT4) {
                // the item's active expert: items come in increasing order, so the
                // search starts at the previous item's (and, unlike decode_item, it
                // reads no route counts or offsets from global memory)
                int hi = n_act - 1;
                while (a_cur < hi) {
                    const int mid = (a_cur + hi + 1) >> 1;
                    if (s_base[mid] <= item) a_cur = mid; else hi = mid - 1;
                }
                const int mt = (item - s_base[a_cur]) % m_tiles;
                const int wrow = PHASE == 1 ? (r < 64 ? mt * 64 + r : p.L.I + mt * 64 + r - 64)
                                            : min(mt * kBlockM + r, p.n_units - 1);
                srow = reinterpret_cast<const uint16_t *>(scale_blob(p, s_act[a_cur]) +
                                                          (PHASE == 1 ? p.L.off.s13 : p.L.off.s2)) +
                       (size_t)wrow * (p.K / 64);
            }
            auto scale_at = [&](int kq) -> uint16_t {
                return (kq < nk && hf < atoms_at(kq)) ? __ldg(srow + kq * ATOMS + hf) : (uint16_t)0;
            };
            uint16_t s_next = 0;
            if (FMT == MOE_W_INT4) {
                const int k0 = (int)((group - (int)(step % C::kDeqGroups) + C::kDeqGroups) % C::kDeqGroups);
                s_next = scale_at(k0);
            }
            for (int kk = 0; kk < nk; ++kk, ++step) {
                const int sub = kk % SUB;
                const bool raw_last = sub == SUB - 1 || kk == nk - 1;  // last stage of this raw stage
                if ((int)(step % C::kDeqGroups) != group) {   // the other group's stage
                    if (++stage == SA) stage = 0;
                    if (raw_last) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&r_empty[rstage]);
                        if (++rstage == SR) rstage = 0;
                    }
                    continue;
                }
                const bool mine = hf < atoms_at(kk);  // this thread's atom lies inside K
                __nv_bfloat162 s2 = __floats2bfloat162_rn(0.0f, 0.0f);
                if (FMT == MOE_W_INT4) {
                    s2 = __bfloat162bfloat162(__ushort_as_bfloat16(s_next));
                    s_next = scale_at(kk + C::kDeqGroups);
                }
                named_sync(1 + group * SA + stage, 32 * (kDeqWarps + 1));
                tc_fence_after();
                if (mine && !s_abort) {
                    // the raw tile landed 128-byte swizzled (16-byte chunk j of row r
                    // at chunk j ^ (r % 8)), so the 32 rows a warp reads at once
                    // spread over all banks
                    const uint8_t *src = sRaw + rstage * RAW + r * kRawRowBytes;
                    // first 16-byte chunk of this thread's atom: 64 codes = 32 (int4) / 64 (int8) bytes
                    const int cj0 = sub * (C::kSubBytes / 16) + hf * (FMT == MOE_W_INT4 ? 2 : 4);
                    uint32_t o[32];  // bf16 pairs (weights 64 hf + 2j, +1 in the low, high half)
                    if (FMT == MOE_W_INT4) {
                        // bf16 128 + n (n in the low mantissa bits of 128.0 = 0x4300),
                        // minus 136 -> n - 8 exactly, times s -> one rounding.
                        // A word holds weights 0..7 of a run of 8 (byte j: 2j low, 2j+1
                        // high nibble).  Masking the low and the high nibbles gives two
                        // words of one nibble per byte, and each byte permute then pairs
                        // two of them with the 0x43 exponent byte: pairs (0,2) (1,3)
                        // (4,6) (5,7).  So within every run of 8 the A columns hold K
                        // order 0 2 1 3 4 6 5 7 (swap 1<->2 and 5<->6); the B operand of
                        // the int4 kernels (xs and h) is stored in the same order, which
                        // leaves every dot product unchanged.
                        const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const uint4 u = *reinterpret_cast<const uint4 *>(src + (((cj0 + c) ^ (r & 7)) << 4));
                            const uint32_t words[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint32_t lo = words[i] & 0x0F0F0F0Fu, hi = (words[i] >> 4) & 0x0F0F0F0Fu;
                                const uint32_t pr[4] = {__byte_perm(lo, 0x43434343u, 0x4140),
                                                        __byte_perm(hi, 0x43434343u, 0x4140),
                                                        __byte_perm(lo, 0x43434343u, 0x4342),
                                                        __byte_perm(hi, 0x43434343u, 0x4342)};
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    uint32_t v = pr[j];
                                    __nv_bfloat162 q = *reinterpret_cast<__nv_bfloat162 *>(&v);
                                    q = __hmul2(__hsub2(q, bias), s2);
                                    o[16 * c + 4 * i + j] = *reinterpret_cast<uint32_t *>(&q);
                                }
                            }
                        }
                    } else {
                        // a code c (two's complement) as bf16, exactly: 0x43 over the low
                        // seven bits is 128 + (c & 127); minus 128 (0x4300) when c >= 0,
                        // minus 256 (0x4380, the sign bit as the low byte) when c < 0.
                        // Two masks per word, then per pair of codes two byte permutes and
                        // one subtraction, in the codes' order (the same selectors as int4).
#pragma unroll
                        for (int c = 0; c < 4; ++c) {  // 16 codes per chunk -> 8 bf16 pairs (codes exact in bf16)
                            const uint4 u = *reinterpret_cast<const uint4 *>(src + (((cj0 + c) ^ (r & 7)) << 4));
                            const uint32_t words[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint32_t lo = words[i] & 0x7F7F7F7Fu, sg = words[i] & 0x80808080u;
#pragma unroll
                                for (int j = 0; j < 2; ++j) {
                                    const uint32_t sel = j ? 0x4342u : 0x4140u;
                                    uint32_t v = __byte_perm(lo, 0x43434343u, sel), b = __byte_perm(sg, 0x43434343u, sel);
                                    __nv_bfloat162 q = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&v),
                                                               *reinterpret_cast<__nv_bfloat162 *>(&b));
                                    o[8 * c + 2 * i + j] = *reinterpret_cast<uint32_t *>(&q);
                                }
                            }
                        }
                    }
                    const uint32_t ta = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(C::kAccCols + stage * A_COLS + 32 * hf);
                    tmem_st16(ta, o);
                    tmem_st16(ta + 16, o + 16);
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&a_full[stage]);
                    if (raw_last) mbar_arrive(&r_empty[rstage]);
                }
                if (++stage == SA) stage = 0;
                if (raw_last && ++rstage == SR) rstage = 0;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                     : "memory");
    }
}

// x rows gathered into sorted-route order: xs[s] = x[sorted_route[s] / k] for
// s < offsets[E].  One warp per row (grid-stride over rows): the route is read
// once, then each lane loads up to kGatherPer 16-byte pieces of the row before
// it stores any, so a row takes one round trip.  With `perm` (the int4 kernels)
// each run of 8 elements is stored in the order k_order<MOE_W_INT4> gives.
constexpr int kGatherPer = 12;  // pieces per lane in flight (a 2816-wide row: 11)
__global__ void __launch_bounds__(256) k_gather_rows(const uint16_t *__restrict__ x,
                                                     const int32_t *__restrict__ sorted_route,
                                                     const int32_t *__restrict__ offsets, int E, int k, int H, int R,
                                                     int perm, uint16_t *__restrict__ xs,
                                                     unsigned *__restrict__ ready) {
    // programmatic dependent launch: wait for the previous kernel before
    // touching memory, then let the next one be scheduled
    pdl_wait();
    pdl_launch_dependents();
    // the per-expert counters of this call's phase 1 (nullable: gather only)
    if (ready != nullptr && blockIdx.x == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) ready[e] = 0u;
    const int per = H / 8;  // 16-byte pieces per row
    const int n_valid = min(__ldg(offsets + E), R);
    const uint64_t pol = l2_policy_last();
    const int lane = threadIdx.x & 31;
    const int n_warps = (int)(gridDim.x * (blockDim.x >> 5));
    for (int s = (int)(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)); s < n_valid; s += n_warps) {
        const int route = __ldg(sorted_route + s);
        if (route < 0 || route >= R) {
            if (lane == 0) record_error(0x2004u, (unsigned)s);
            continue;
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)(route / k) * H);
        uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)s * H);
        for (int c0 = 0; c0 < per; c0 += 32 * kGatherPer) {
            uint4 u[kGatherPer];
#pragma unroll
            for (int j = 0; j < kGatherPer; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c < per) u[j] = __ldg(src + c);
            }
#pragma unroll
            for (int j = 0; j < kGatherPer; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c >= per) break;
                uint4 v = u[j];
                if (perm) {  // elements (0,1)(2,3)(4,5)(6,7) -> (0,2)(1,3)(4,6)(5,7)
                    v.x = __byte_perm(u[j].x, u[j].y, 0x5410);
                    v.y = __byte_perm(u[j].x, u[j].y, 0x7632);
                    v.z = __byte_perm(u[j].z, u[j].w, 0x5410);
                    v.w = __byte_perm(u[j].z, u[j].w, 0x7632);
                }
                st_v4_hint(dst + c, v, pol);
            }
        }
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// 3-D map over `blobs` matrices of `rows` rows of `row_elems` elements, one
// matrix per blob (`blob_stride` bytes apart, starting at `base`); box =
// box_inner elements x box_rows rows of one matrix.
bool encode_3d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t row_elems,
               uint64_t rows, uint64_t blobs, uint64_t blob_stride, uint32_t box_inner, uint32_t box_rows,
               CUtensorMapSwizzle sw) {
    cuuint64_t dims[3] = {row_elems, rows, blobs};
    cuuint64_t strides[2] = {row_elems * (uint64_t)elem_bytes, blob_stride};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return g_encode(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over `rows` rows of `row_bytes` bytes; box = box_inner elements x box_rows.
bool encode_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t row_elems,
               uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
    cuuint64_t dims[2] = {row_elems, rows};
    cuuint64_t strides[1] = {row_elems * (uint64_t)elem_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, int CFG>
constexpr size_t smem_bytes() {
    using C = TcCfg<FMT, CFG>;
    return 1024 + (size_t)(C::kASmem ? C::kAStages * (C::kKS / kBlockK) : 0) * kATileBytes + C::kBRegion +
           (size_t)C::kRawStages * kRawBytes<FMT>() + 2 * 64 * kXPitch * 4 +
           (size_t)(2 * C::kAStages + 2 * kMaxBSlots + 2 * kAccBufs + 4 + 2 * C::kRawStages) * 8;
}
// dynamic + static shared memory (s_act, s_base, ...: 9216 bytes) within the
// 232448-byte per-block limit; two CTAs per SM (with 1 KB reserved by the
// system each) within the SM's 233472 bytes
static_assert(smem_bytes<MOE_W_BF16, 0>() + 9216 <= 232448, "bf16 tensor-core kernel exceeds shared memory");
static_assert(smem_bytes<MOE_W_INT8, 0>() + 9216 <= 232448, "int8 tensor-core kernel exceeds shared memory");
static_assert(smem_bytes<MOE_W_INT4, 0>() + 9216 <= 232448, "int4 tensor-core kernel exceeds shared memory");
static_assert(2 * (smem_bytes<MOE_W_INT8, 1>() + 9216 + 1024) <= 233472, "int8 two-CTA config exceeds shared memory");
static_assert(2 * (smem_bytes<MOE_W_INT4, 1>() + 9216 + 1024) <= 233472, "int4 two-CTA config exceeds shared memory");
static_assert(2 * TcCfg<MOE_W_INT4, 1>::kTmemCols <= 512 && TcCfg<MOE_W_INT4, 1>::kAccCols +
                  TcCfg<MOE_W_INT4, 1>::kAStages * TcCfg<MOE_W_INT4, 1>::kKS / 2 <= TcCfg<MOE_W_INT4, 1>::kTmemCols,
              "two-CTA config exceeds tensor memory");

template <int FMT, int PHASE, int CFG>
cudaError_t launch_one(const CUtensorMap &mh, const CUtensorMap &mp, const CUtensorMap &mb, const CUtensorMap &mb64,
                       const TcParams &p, int n_sm, cudaStream_t s) {
    auto kern = k_ffn_tc<FMT, PHASE, CFG>;
    const size_t smem = smem_bytes<FMT, CFG>();
    static bool attr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!attr[dev]) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        attr[dev] = true;
    }
    // programmatic dependent launch (the B producer waits for the previous launch)
    return launch_pdl(kern, dim3((unsigned)(n_sm * TcCfg<FMT, CFG>::kMinBlocks)), dim3((unsigned)tc_threads<FMT, CFG>()),
                      smem, s, mh, mp, mb, mb64, p);
}

}  // namespace

size_t ffn_tc_workspace(int T, int k, int E, int H, int I) {
    const size_t R = (size_t)T * k;
    const size_t xs = (R * H * 2 + 255) & ~(size_t)255;
    const size_t h = (R * I * 2 + 255) & ~(size_t)255;
    return xs + h + (size_t)E * 4;  // xs | h | per-expert phase-1 counters
}

bool ffn_tc_supports(int fmt, int H, int I, uint64_t stride) {
    (void)fmt;
    // the weight maps are 3-D (row, matrix row, blob), so any blob stride that is a
    // multiple of 16 bytes works; every row length (H or I times 2, 1 or 1/2
    // bytes) is a multiple of 32 bytes and every matrix piece starts 16-byte aligned
    return H % 64 == 0 && I % 64 == 0 && stride % 16 == 0 && get_encoder() == cudaSuccess;
}

cudaError_t launch_ffn_tc(const LayerView &L, const uint16_t *x, int T, int k, const int32_t *counts,
                          const int32_t *offsets, const int32_t *sorted_route, float *rows, void *ws,
                          cudaStream_t s) {
    cudaError_t err = get_encoder();
    if (err != cudaSuccess) return err;
    if (!ffn_tc_supports(L.fmt, L.H, L.I, L.stride)) return cudaErrorNotSupported;
    int n_sm = 0;
    if ((err = sm_count(&n_sm)) != cudaSuccess) return err;
    const int R = T * k;
    const int H = L.H, I = L.I, fmt = L.fmt;
    uint16_t *xs = static_cast<uint16_t *>(ws);
    const size_t xs_bytes = ((size_t)R * H * 2 + 255) & ~(size_t)255, h_bytes = ((size_t)R * I * 2 + 255) & ~(size_t)255;
    uint16_t *h = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + xs_bytes);
    unsigned *ready = reinterpret_cast<unsigned *>(static_cast<char *>(ws) + xs_bytes + h_bytes);

    // 1. activations into sorted-route order
    {
        // one warp per row, eight rows per CTA, at most 8 CTAs per SM
        const int blocks = (int)std::min<int64_t>(((int64_t)R + 7) / 8, (int64_t)n_sm * 8);
        err = launch_pdl(k_gather_rows, dim3((unsigned)blocks), dim3(256), 0, s, x, sorted_route, offsets, L.E, k, H, R,
                         (int)(L.fmt == MOE_W_INT4), xs, ready);
        if (err != cudaSuccess) return err;
    }
    // 2. tensor maps: weights (home and pool, as rows of one matrix), activations
    const bool bf = fmt == MOE_W_BF16;
    const CUtensorMapDataType dt = bf ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const int eb = bf ? 2 : 1;
    const CUtensorMapSwizzle swa = CU_TENSOR_MAP_SWIZZLE_128B;  // weight tiles and raw code tiles alike
    const uint32_t raw_inner = kRawRowBytes;
    CUtensorMap mh1, mp1, mh2, mp2, mb1, mb2, mbb1, mbb2;
    for (int ph = 1; ph <= 2; ++ph) {
        const int K = ph == 1 ? H : I;
        const uint64_t row_elems = bf ? (uint64_t)K : (fmt == MOE_W_INT8 ? (uint64_t)K : (uint64_t)K / 2);
        const uint32_t box_inner = bf ? kBlockK : raw_inner;
        CUtensorMap *mh = ph == 1 ? &mh1 : &mh2, *mp = ph == 1 ? &mp1 : &mp2;
        // one matrix (w13 codes, or w2 codes) per blob: E blobs of home, pool_slots
        // of the pool (home again when the layer has no slot table)
        const uint64_t piece = ph == 1 ? L.off.q13 : L.off.q2;
        const uint64_t mrows = ph == 1 ? 2 * (uint64_t)I : (uint64_t)H;
        if (!encode_3d(mh, L.home + piece, dt, eb, row_elems, mrows, (uint64_t)L.E, L.stride, box_inner, 64, swa))
            return cudaErrorInvalidValue;
        const bool slotted = L.slot_table != nullptr && L.pool != nullptr && L.pool_slots > 0;
        if (!encode_3d(mp, (slotted ? L.pool : L.home) + piece, dt, eb, row_elems, mrows,
                       slotted ? (uint64_t)L.pool_slots : (uint64_t)L.E, L.stride, box_inner, 64, swa))
            return cudaErrorInvalidValue;
        CUtensorMap *mb = ph == 1 ? &mb1 : &mb2, *mbb = ph == 1 ? &mbb1 : &mbb2;
        if (!encode_2d(mb, ph == 1 ? (const void *)xs : (const void *)h, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                       (uint64_t)K, (uint64_t)R, kBlockK, 16, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        // 64-row boxes for route blocks over 32 (only used when a block that large
        // exists, i.e. R > 32)
        if (!encode_2d(mbb, ph == 1 ? (const void *)xs : (const void *)h, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                       (uint64_t)K, (uint64_t)R, kBlockK, R >= 64 ? 64 : 16, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    TcParams p{};
    p.L = L;
    p.R = R;
    p.counts = counts;
    p.offsets = offsets;
    // cap on the route block: an expert never gets a token twice, so min(T, 128)
    // rows hold all of an expert's routes in one block (smaller blocks would
    // re-stream the weights of busier experts); the kernels shrink it to the
    // busiest expert's count
    // int formats with a decode batch (every route block <= 64) run two CTAs per SM
    const bool two = !bf && T <= TcCfg<MOE_W_INT4, 1>::kNMax;
    p.n_block = std::min(two ? TcCfg<MOE_W_INT4, 1>::kNMax : kNMax, (std::max(T, 1) + 15) / 16 * 16);
    p.h = h;
    p.rows = rows;
    p.ready = ready;
    // every pointer the kernels write through must be set (host-side guard)
    if (p.h == nullptr || p.rows == nullptr || p.counts == nullptr || p.offsets == nullptr || xs == nullptr)
        return cudaErrorInvalidValue;
    // phase 1
    {
        p.K = H;
        p.n_units = 2 * I;
        if (fmt == MOE_W_BF16) err = launch_one<MOE_W_BF16, 1, 0>(mh1, mp1, mb1, mbb1, p, n_sm, s);
        else if (fmt == MOE_W_INT8) err = two ? launch_one<MOE_W_INT8, 1, 1>(mh1, mp1, mb1, mbb1, p, n_sm, s)
                                              : launch_one<MOE_W_INT8, 1, 0>(mh1, mp1, mb1, mbb1, p, n_sm, s);
        else err = two ? launch_one<MOE_W_INT4, 1, 1>(mh1, mp1, mb1, mbb1, p, n_sm, s)
                       : launch_one<MOE_W_INT4, 1, 0>(mh1, mp1, mb1, mbb1, p, n_sm, s);
        if (err != cudaSuccess) return err;
    }
    // phase 2
    {
        p.K = I;
        p.n_units = H;
        if (fmt == MOE_W_BF16) err = launch_one<MOE_W_BF16, 2, 0>(mh2, mp2, mb2, mbb2, p, n_sm, s);
        else if (fmt == MOE_W_INT8) err = two ? launch_one<MOE_W_INT8, 2, 1>(mh2, mp2, mb2, mbb2, p, n_sm, s)
                                              : launch_one<MOE_W_INT8, 2, 0>(mh2, mp2, mb2, mbb2, p, n_sm, s);
        else err = two ? launch_one<MOE_W_INT4, 2, 1>(mh2, mp2, mb2, mbb2, p, n_sm, s)
                       : launch_one<MOE_W_INT4, 2, 0>(mh2, mp2, mb2, mbb2, p, n_sm, s);
    }
    return err;
}

cudaError_t tc_take_error(unsigned *code, unsigned *info) {
    unsigned zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_tc_error, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(info, g_tc_error_info, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_tc_error_info, &zero, sizeof(unsigned));
    return e;
}

}  // namespace moe
