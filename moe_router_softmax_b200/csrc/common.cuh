// common.cuh -- small device/host helpers shared by the library's kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int kMaxDevices = 64;

// SM count of the current device (cached per device).
inline cudaError_t sm_count(int *n) {
    static int cached[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (cached[dev] == 0) {
        err = cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
    }
    *n = cached[dev];
    return cudaSuccess;
}

// ------------------------------------------------------------------ errors
// Thread-local last error (moe_last_error); set_error returns the status.
moe_status set_error(moe_status st, const char *fmt, ...);

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// fp32 -> bf16 bits, round to nearest even; NaN stays a quiet NaN.
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// ------------------------------------------------------------------ loads
// Streaming loads of data read once (expert weights): no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ld_stream_v2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// ------------------------------------------------------------------ blobs
// Byte offsets of the pieces of one expert blob (w13 codes, s13, w2 codes, s2).
struct BlobOffsets {
    uint64_t q13, s13, q2, s2, total;
};

inline BlobOffsets blob_offsets(int fmt, int H, int I) {
    BlobOffsets o{};
    uint64_t h = (uint64_t)H, i = (uint64_t)I;
    if (fmt == MOE_W_BF16) {
        o.q13 = 0;
        o.s13 = 2 * i * h * 2;
        o.q2 = o.s13;
        o.s2 = o.q2 + h * i * 2;
        o.total = o.s2;
    } else if (fmt == MOE_W_INT8) {
        o.q13 = 0;
        o.s13 = 2 * i * h;
        o.q2 = o.s13 + 2 * i * 4;
        o.s2 = o.q2 + h * i;
        o.total = o.s2 + h * 4;
    } else {
        o.q13 = 0;
        o.s13 = 2 * i * (h / 2);
        o.q2 = o.s13 + 2 * i * (h / 64) * 2;
        o.s2 = o.q2 + h * (i / 2);
        o.total = o.s2 + h * (i / 64) * 2;
    }
    return o;
}

// Device view of one layer's experts.
struct LayerView {
    int fmt, E, H, I;
    const int32_t *slot_table;
    const uint8_t *pool;
    const uint8_t *home;
    uint64_t stride;
    int pool_slots;  // blobs in pool (meaningful with a slot table)
    BlobOffsets off;
};

// Slot of expert e: -1 for home, else a pool slot below pool_slots.  A table
// entry at or past pool_slots is out of the pool: *bad is set (and -1 returned,
// so that an address computed from it stays inside home).
__device__ __forceinline__ int expert_slot(const LayerView &L, int e, bool *bad) {
    const int s = L.slot_table ? __ldg(L.slot_table + e) : -1;
    *bad = s >= L.pool_slots && L.slot_table != nullptr;
    return (s >= 0 && !*bad) ? s : -1;
}

// Blob of expert e through the slot table, or nullptr when its slot is out of
// the pool (the caller skips the expert and records the fault).
__device__ __forceinline__ const uint8_t *expert_blob(const LayerView &L, int e) {
    bool bad;
    const int s = expert_slot(L, e, &bad);
    if (bad) return nullptr;
    return s >= 0 ? L.pool + (uint64_t)s * L.stride : L.home + (uint64_t)e * L.stride;
}

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch: the next kernel in the stream may be scheduled
// as soon as every CTA of this one has signalled (or finished), and
// griddepcontrol.wait blocks until the previous kernel has completed and its
// writes are visible.  Both are no-ops for a kernel launched without the
// programmatic-serialization attribute.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch `kern` on `s` with programmatic stream serialization allowed, so it
// may start while the previous kernel in the stream is still running (it must
// call pdl_wait() before reading that kernel's results).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace moe
