// Launcher of the confidence-unmasking step (unmask.cu).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace tt {
cudaError_t launch_confidence_unmask(const void* logits, int B, int S, int V, float gamma, int min_one,
                                     int32_t* tokens, uint8_t* masked, float* p_max, int32_t* argmax,
                                     int32_t* n_committed, cudaStream_t stream);
}  // namespace tt
