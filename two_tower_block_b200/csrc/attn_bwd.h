// Block-causal backward pass (attn_bwd.cu): problem description and launcher.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tt {

struct BwdProblem {
  int B, Hq, Hkv, g, D, S, R, N, NB;   // N = sequence length, NB = N / S blocks
  float scale, scale_log2;
  const __nv_bfloat16 *q, *k_ctx, *v_ctx, *k_blk, *v_blk;   // forward inputs (block-causal layouts)
  const float *out, *lse;                                     // forward outputs
  const __nv_bfloat16* dout;                                  // dL/dout
  float *dq, *dk_blk, *dv_blk;                                // gradients; dk_blk / dv_blk start at zero
};

cudaError_t launch_attn_bwd(const BwdProblem& p, cudaStream_t stream);

}  // namespace tt
