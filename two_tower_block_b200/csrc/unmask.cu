// Confidence-unmasking step of block sampling.
//
// The method (paperfeed.app review of arXiv 2606.26493, section "Training and
// sampling"; kongchang explainer, section "Sudoku"): every masked position of the
// block is predicted in parallel and each prediction whose confidence is above
// gamma = 0.8 is committed; the rest stay masked for the next denoising step.
// Confidence = softmax probability of the argmax token (lowest index among equal
// maxima).  With min_one, a sequence whose step passes nothing commits its most
// confident masked position (lowest position among equals).
//
// Kernel 1: one CTA per (sequence, position) row that is still masked.  It streams
// the row's V bf16 logits once with 16-byte loads, keeping an online (max, sum of
// 2^(x - max), argmax) per thread in the log2 domain, merged across the CTA; the
// probability of the argmax token is 1 / sum.  Kernel 2: one CTA per sequence
// applies the commit rule to tokens and mask.
#include "unmask.h"

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace tt {
namespace {

constexpr int kScanThreads = 512;
constexpr float kLog2e = 1.4426950408889634f;

struct Acc {
  float m;    // running maximum (log2 units)
  float s;    // sum of 2^(x - m)
  int arg;    // index of the first maximum
};

__device__ __forceinline__ void acc_push(Acc& a, float x, int idx) {
  const float z = x * kLog2e;
  if (z > a.m) {
    a.s = a.s * fast_exp2(a.m - z) + 1.f;
    a.m = z;
    a.arg = idx;
  } else {
    a.s += fast_exp2(z - a.m);
  }
}

__device__ __forceinline__ Acc acc_merge(const Acc& a, const Acc& b) {
  if (b.m == -INFINITY) return a;
  if (a.m == -INFINITY) return b;
  Acc r;
  r.m = fmaxf(a.m, b.m);
  r.s = a.s * fast_exp2(a.m - r.m) + b.s * fast_exp2(b.m - r.m);
  r.arg = a.m > b.m ? a.arg : (b.m > a.m ? b.arg : min(a.arg, b.arg));
  return r;
}

__global__ void __launch_bounds__(kScanThreads)
    unmask_scan_kernel(const __nv_bfloat16* __restrict__ logits, const uint8_t* __restrict__ masked, int V,
                       float* __restrict__ p_max, int32_t* __restrict__ argmax) {
  const int row = blockIdx.x;
  if (!masked[row]) {
    if (threadIdx.x == 0) {
      p_max[row] = 0.f;
      argmax[row] = -1;
    }
    return;
  }
  const __nv_bfloat16* x = logits + (size_t)row * V;
  Acc a{-INFINITY, 0.f, 0};
  if ((V & 7) == 0) {
    const uint4* x8 = reinterpret_cast<const uint4*>(x);
    const int n8 = V >> 3;
    constexpr int kDepth = 4;   // 16-byte loads a thread has in flight
    for (int i0 = threadIdx.x; i0 < n8; i0 += kDepth * kScanThreads) {
      uint4 v[kDepth];
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
        const int i = i0 + u * kScanThreads;
        if (i < n8) v[u] = __ldcs(x8 + i);   // streamed once
      }
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {   // ascending index order within the thread
        const int i = i0 + u * kScanThreads;
        if (i < n8) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            acc_push(a, __uint_as_float(w[k] << 16), 8 * i + 2 * k);
            acc_push(a, __uint_as_float(w[k] & 0xFFFF0000u), 8 * i + 2 * k + 1);
          }
        }
      }
    }
  } else {
    for (int i = threadIdx.x; i < V; i += kScanThreads) acc_push(a, __bfloat162float(x[i]), i);
  }
  // merge across the warp, then across the CTA
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Acc b{__shfl_xor_sync(0xffffffffu, a.m, o), __shfl_xor_sync(0xffffffffu, a.s, o),
          __shfl_xor_sync(0xffffffffu, a.arg, o)};
    a = acc_merge(a, b);
  }
  __shared__ Acc part[kScanThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) part[warp] = a;
  __syncthreads();
  if (warp == 0) {
    a = lane < kScanThreads / 32 ? part[lane] : Acc{-INFINITY, 0.f, 0};
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Acc b{__shfl_xor_sync(0xffffffffu, a.m, o), __shfl_xor_sync(0xffffffffu, a.s, o),
            __shfl_xor_sync(0xffffffffu, a.arg, o)};
      a = acc_merge(a, b);
    }
    if (lane == 0) {
      p_max[row] = 1.f / a.s;
      argmax[row] = a.arg;
    }
  }
}

__global__ void unmask_commit_kernel(int S, float gamma, int min_one, int32_t* tokens, uint8_t* masked,
                                     const float* __restrict__ p_max, const int32_t* __restrict__ argmax,
                                     int32_t* n_committed) {
  const int n = blockIdx.x, s = threadIdx.x;
  __shared__ unsigned long long best;   // (confidence bits << 32) | (~position): the most confident, first
  __shared__ int any_pass, count;
  if (s == 0) {
    best = 0ull;
    any_pass = 0;
    count = 0;
  }
  __syncthreads();
  const int idx = n * S + s;
  const bool m = s < S && masked[idx] != 0;
  const float p = m ? p_max[idx] : 0.f;
  const bool pass = m && p > gamma;
  if (pass) atomicOr(&any_pass, 1);
  if (m) atomicMax(&best, ((unsigned long long)__float_as_uint(p) << 32) | (0xFFFFFFFFu - (unsigned)s));
  __syncthreads();
  bool commit = pass;
  if (min_one && !any_pass && m) commit = (unsigned)(0xFFFFFFFFu - (unsigned)(best & 0xFFFFFFFFull)) == (unsigned)s;
  if (commit) {
    tokens[idx] = argmax[idx];
    masked[idx] = 0;
    atomicAdd(&count, 1);
  }
  __syncthreads();
  if (s == 0 && n_committed) n_committed[n] = count;
}

}  // namespace

cudaError_t launch_confidence_unmask(const void* logits, int B, int S, int V, float gamma, int min_one,
                                     int32_t* tokens, uint8_t* masked, float* p_max, int32_t* argmax,
                                     int32_t* n_committed, cudaStream_t stream) {
  unmask_scan_kernel<<<B * S, kScanThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(logits), masked, V,
                                                          p_max, argmax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int threads = ((S + 31) / 32) * 32;
  unmask_commit_kernel<<<B, threads, 0, stream>>>(S, gamma, min_one, tokens, masked, p_max, argmax, n_committed);
  return cudaGetLastError();
}

}  // namespace tt
