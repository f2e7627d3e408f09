// Launcher of the committed-block cache update (kv_append.cu).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace tt {
cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_ctx, void* v_ctx, int32_t* ctx_lens,
                             int B, int S, int Hkv, int D, int Lcap, int advance, unsigned* err_word,
                             cudaStream_t stream);
}  // namespace tt
