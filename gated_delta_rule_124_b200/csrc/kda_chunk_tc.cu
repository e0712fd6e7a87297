// Tensor-core chunkwise prefill (bf16, dk = dv = 128, chunk = 64): not built yet.
#include "kda_chunk_tc.cuh"

namespace kda {

bool tc_path_available() { return false; }

cudaError_t launch_chunk_fwd_tc(const void*, const void*, const void*, const float*,
                                const float*, const float*, const int32_t*, int, int, int,
                                const int*, uint32_t*, void*, float*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace kda
