// ffn_tc.cu -- grouped gated FFN on the tcgen05 tensor cores (prefill-sized
// batches).  Placeholder until the tensor-core kernels land: the path reports
// itself unsupported, so MOE_FFN_AUTO keeps every call on the GEMV kernels.
#include "common.cuh"

namespace moe {

size_t ffn_tc_workspace(int, int, int, int, int) { return 0; }
bool ffn_tc_supports(int, int, int) { return false; }
cudaError_t launch_ffn_tc(const LayerView &, const uint16_t *, int, int, const int32_t *, const int32_t *,
                          const int32_t *, float *, void *, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace moe
