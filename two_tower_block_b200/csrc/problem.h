// Problem description handed to every kernel (by value, as a kernel parameter).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sched.cuh"

namespace tt {

enum Mode : int { kDecode = 0, kBlockCausal = 1 };

// Keys per pipeline tile of each kernel (the work split counts tiles of this size).
// The default tcgen05 kernel runs 64-key tiles with two S buffers per M-tile, so the
// scores of tile j+1 are computed while the softmax works on tile j; it also runs
// 128-key tiles with one S buffer (see tcgen05_key_tile_supported), which the
// transposed-PV and 2-SM forms require.
constexpr int kTcgen05KeyTile = 64;
constexpr int kMmaSyncKeyTile = 64;

struct Problem {
  // geometry
  int mode;        // kDecode or kBlockCausal
  int B, Hq, Hkv, g, D, S, R;  // R = S * g packed rows of one unit (row = t * g + j)
  int NB;          // blocks per sequence: 1 for decode, N / S for block-causal
  int ctx_stride;  // tokens per (n, h) slab of k_ctx / v_ctx: Lcap or N
  float scale_log2;  // softmax scale * log2(e)
  // tensors (caller-owned device memory)
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_ctx;
  const __nv_bfloat16* v_ctx;
  const __nv_bfloat16* k_blk;
  const __nv_bfloat16* v_blk;
  const int* ctx_lens;  // decode only
  float* out;           // fp32, or bf16 when out_bf16 (the pointer then addresses bf16 elements)
  float* lse;           // may be null
  int out_bf16;         // final output rows in bf16 (round to nearest even); partials stay fp32
  // work split
  int C;                // ranges
  int key_tile;         // keys per tile
  int blk_tiles;        // tiles holding the block's own keys: ceil(S / key_tile)
  long long T_causal;   // block-causal: total tiles (decode computes T on the device)
  const int* causal_pref;  // block-causal: tiles before block b within one (n, h); NB + 1 entries
  const long long* causal_starts;  // block-causal: range boundary table (min(C, T) + 1 entries) or
                                   // null for the uniform split
  // plan-owned scratch
  float* part_o;        // [2C][R][D]
  float* part_lse;      // [2C][R]
  SplitRecord* records; // [C]
  unsigned* err_word;
  unsigned long long wait_limit_ns;
  int variant;          // tcgen05 kernel: 0 = S/P aliasing in TMEM (default), 2 = transposed PV,
                        // 3 = 2-SM pairs (head_dim 128)
  // default tcgen05 kernel launched cooperatively: every CTA adds one to its range's entry
  // (per-range launch counts that only grow) once its partials are written, waits for the
  // ranges that share its cut units to reach the same count, and combines its share of
  // those units' rows; null: the separate combine kernel runs instead
  unsigned* arrivals;
  // paged context cache (decode only; null page_table: contiguous k_ctx / v_ctx).
  // k_ctx / v_ctx then point at pools [num_pages][Hkv][page_size][D]; context position
  // pos of sequence n sits in page page_table[n * pages_per_seq + (pos >> page_shift)]
  // at row pos & (page_size - 1).  ctx_stride = pages_per_seq * page_size.
  const int* page_table;
  int page_shift;       // log2(page_size); page_size is a power of two >= 16
  int pages_per_seq;
  int num_pages;
};

// Host launchers (each returns the cudaError_t of its launch).
cudaError_t launch_attn_mma_sync(const Problem& p, cudaStream_t stream);
cudaError_t launch_combine(const Problem& p, cudaStream_t stream);
cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t stream);
cudaError_t launch_wait_selftest(unsigned* err_word, unsigned long long limit_ns, cudaStream_t stream);

struct TmaMaps {
  CUtensorMap q, k_ctx, v_ctx, k_blk, v_blk;
};
cudaError_t launch_attn_tcgen05(const Problem& p, const TmaMaps& maps, cudaStream_t stream);
bool tcgen05_key_tile_supported(int key_tile);
cudaError_t launch_attn_pt(const Problem& p, const TmaMaps& maps, cudaStream_t stream);
// 2-SM kernel (cluster of two CTAs, one range per cluster): head_dim 128, 128 % g == 0
bool attn_2sm_supported(int D, int g);
int attn_2sm_max_clusters();
cudaError_t launch_attn_2sm(const Problem& p, cudaStream_t stream);
size_t attn_pt_smem_bytes();
size_t attn_tcgen05_smem_bytes(int D);
size_t attn_mma_sync_smem_bytes(int D);

}  // namespace tt
