// Block-causal backward pass (attn_bwd.cu): problem description and launcher.
#pragma once
#include <cuda.h>
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
  unsigned* err_word;                                         // device error word (timeouts)
  unsigned long long wait_limit_ns;                           // limit of one pipeline wait
};

// TMA tensor maps of the tcgen05 backward: q and dout as [tokens][Hq][D] with a box of
// (64 dims, g heads, tokens of one 128-row M-tile); k_ctx / v_ctx as [B*Hkv*N rows][D]
// with a box of 64 rows; k_blk / v_blk as [tokens][Hkv][D] with a box of min(S, 64) tokens.
struct BwdMaps {
  CUtensorMap q, dout, k_ctx, v_ctx, k_blk, v_blk;
};

// Warp-level tensor-core backward (mma.sync): every shape the forward supports.
cudaError_t launch_attn_bwd(const BwdProblem& p, cudaStream_t stream);
// tcgen05 backward: head_dim 64 or 128, S <= 32, and S*g <= 128 or 128 % g == 0 with S*g <= 256.
bool attn_bwd_tc_supported(const BwdProblem& p);
cudaError_t launch_attn_bwd_tc(const BwdProblem& p, const BwdMaps& maps, int num_ctas, cudaStream_t stream);

}  // namespace tt
