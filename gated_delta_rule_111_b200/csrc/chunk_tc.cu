// Tensor-core (tcgen05) chunkwise prefill -- not yet enabled; the FP32
// CUDA-core kernel serves every configuration until it is.
#include "common.cuh"

namespace gdn2 {

bool chunk_tc_supported(int, int, gdn2_dtype) { return false; }

cudaError_t launch_chunk_tc(const void *, const void *, const void *, const float *, const float *,
                            const float *, const float *, void *, float *, int, int, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gdn2
