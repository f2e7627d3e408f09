// Committed-block cache update.
//
// The method (paperfeed.app review of arXiv 2606.26493, section "The idea: freeze
// the reader, train the writer"): once a block is committed, the frozen context
// tower ingests it causally and its per-layer caches grow by the block's S
// positions.  This kernel writes the context tower's layer-i K/V of those
// positions (computed by the caller) into the cache at [L_n, L_n + S) and, on
// request, advances L_n.  One CTA per sequence: it reads L_n once, copies the
// S x Hkv rows of K and of V with 16-byte accesses (coalesced on both sides:
// a row is D contiguous bf16 in each layout), then advances the length.  A
// sequence without room (L_n < 0 or L_n + S > capacity) raises the error word
// and is left untouched.
#include "kv_append.h"

#include "errbits.h"

namespace tt {
namespace {

constexpr int kThreads = 512;
constexpr int kPerThread = 4;   // chunks of K and of V a thread loads before it stores

__global__ void __launch_bounds__(kThreads)
    kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_ctx,
                     uint4* __restrict__ v_ctx, int32_t* ctx_lens, int S, int Hkv, int chunks, int Lcap,
                     int advance, unsigned* err_word) {
  __shared__ int s_len;
  const int n = blockIdx.x;
  if (threadIdx.x == 0) {
    const int L = ctx_lens[n];
    const bool ok = L >= 0 && L <= Lcap - S;
    if (!ok) atomicOr(err_word, kErrDeviceArg);
    s_len = ok ? L : -1;
  }
  __syncthreads();
  const int L = s_len;
  if (L < 0) return;
  const int total = S * Hkv * chunks;   // 16-byte chunks of one sequence's new rows
  const uint4* kn = k_new + (size_t)n * total;
  const uint4* vn = v_new + (size_t)n * total;
  for (int i0 = threadIdx.x; i0 < total; i0 += kThreads * kPerThread) {
    uint4 kr[kPerThread], vr[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int i = i0 + u * kThreads;
      if (i < total) {
        kr[u] = kn[i];
        vr[u] = vn[i];
      }
    }
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int i = i0 + u * kThreads;
      if (i < total) {
        const int c = i % chunks, row = i / chunks;   // row = t * Hkv + h
        const int h = row % Hkv, t = row / Hkv;
        const size_t dst = (((size_t)n * Hkv + h) * Lcap + L + t) * chunks + c;
        k_ctx[dst] = kr[u];
        v_ctx[dst] = vr[u];
      }
    }
  }
  __syncthreads();   // every thread has read L before it moves
  if (advance && threadIdx.x == 0) ctx_lens[n] = L + S;
}

}  // namespace

cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_ctx, void* v_ctx, int32_t* ctx_lens,
                             int B, int S, int Hkv, int D, int Lcap, int advance, unsigned* err_word,
                             cudaStream_t stream) {
  kv_append_kernel<<<B, kThreads, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_ctx),
      static_cast<uint4*>(v_ctx), ctx_lens, S, Hkv, D / 8, Lcap, advance, err_word);
  return cudaGetLastError();
}

}  // namespace tt
