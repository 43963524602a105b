// ffn_noalloc.cu -- moe_grouped_ffn_noalloc: the grouped FFN for callers that
// cannot allocate device memory.
//
// moe_grouped_ffn needs a scratch buffer for the bf16 intermediate h (one row
// of I values per route) and asks the caller for it.  Some callers have no way
// to provide one: a plugin or serving runtime that hands the library only its
// input and output buffers and owns every other byte of device memory, or a
// latency-critical loop that must never call cudaMalloc (which can synchronise
// the device and can fail under fragmentation).  For them this entry point
// keeps its scratch in a fixed, file-scope device array instead.
//
// It always runs the split-K GEMV kernels (their only scratch is h, T*k*I*2
// bytes); the tensor-core kernels would also need a sorted copy of the
// activations.  Its rows therefore equal moe_grouped_ffn's where that call picks
// the GEMV kernels, and agree within the FFN tolerance where it picks the tensor
// cores; prefill-sized batches run slower than through moe_grouped_ffn.
//
// The array is a module global: every GPU that loads the library reserves it
// (kNoAllocScratchBytes) until the process exits, and every call shares it.
// Nothing in it has to start at zero -- each call writes every h row it later
// reads -- but its contents persist from the previous call, and two calls whose
// work overlaps on the GPU (different streams, or different threads on one
// device) race on it.
#include <mutex>

#include "common.cuh"

namespace moe {
size_t ffn_gemv_workspace(int T, int k, int I);
moe_status check_ffn_args(const moe_layer *layer, int T, int k);
}

namespace {

// 16 MiB: the bf16 intermediate of T*k routes must fit, T*k*I*2 bytes
// (8192 routes at I = 704 need 11.5 MB).
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device, looked up once with that
// device current (on the host the symbol name is only a stand-in, never a
// device pointer).  The cached address belongs to the device's primary
// context: after a cudaDeviceReset it is stale, so the entry point must not be
// called again in that process.
void *g_scratch_addr[moe::kMaxDevices];
std::mutex g_scratch_mutex;

moe_status scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return moe::set_error(MOE_ERR_CUDA, "moe_grouped_ffn_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= moe::kMaxDevices)
        return moe::set_error(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_noalloc: device %d beyond %d", dev,
                              moe::kMaxDevices);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return moe::set_error(MOE_ERR_CUDA, "moe_grouped_ffn_noalloc: cudaGetSymbolAddress of the scratch: %s",
                                  cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_grouped_ffn_noalloc(const moe_layer *layer, const uint16_t *x, int32_t T, int32_t k,
                                   const int32_t *counts, const int32_t *offsets, const int32_t *sorted_route,
                                   float *rows, moe_stream_t stream) {
    // the layer and the sizes first, so that a bad argument is reported as what
    // it is rather than as a scratch overflow
    moe_status st = moe::check_ffn_args(layer, T, k);
    if (st != MOE_OK) return st;
    // the GEMV kernels' scratch: the bf16 intermediate, T*k*I*2 bytes
    const size_t need = moe::ffn_gemv_workspace(T, k, layer->I);
    if (need > kNoAllocScratchBytes)
        return moe::set_error(MOE_ERR_INVALID_ARG,
                              "moe_grouped_ffn_noalloc: T*k=%lld routes at I=%d need %zu bytes of scratch; the fixed "
                              "scratch holds %zu bytes (use moe_grouped_ffn with a workspace instead)",
                              (long long)T * k, layer->I, need, kNoAllocScratchBytes);
    void *scratch = nullptr;
    st = scratch_for_current_device(&scratch);
    if (st != MOE_OK) return st;
    return moe_grouped_ffn_path(layer, x, T, k, counts, offsets, sorted_route, rows, scratch, kNoAllocScratchBytes,
                                MOE_FFN_GEMV, stream);
}

}  // extern "C"
