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
// probability of the argmax token is 1 / sum.  Each thread takes its logits in batches
// of 32 (four 16-byte loads in flight), rescaling its sum once per batch; 1024 threads
// per row keep 64 KB of loads in flight per SM.  One exponential pair in four is computed
// on the FMA pipe (ptx.cuh: exp2_poly2) to relieve the MUFU.  Kernel 2 is launched as a
// programmatic dependent of kernel 1, so its launch overlaps the scan.  Kernel 2: one CTA per sequence
// applies the commit rule to tokens and mask.
#include "unmask.h"

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace tt {
namespace {

constexpr int kScanThreads = 1024;   // one CTA per row
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

__global__ void __launch_bounds__(kScanThreads, 1)
    unmask_scan_kernel(const __nv_bfloat16* __restrict__ logits, const uint8_t* __restrict__ masked, int V,
                       float* __restrict__ p_max, int32_t* __restrict__ argmax) {
  // the commit kernel may be scheduled now; it waits for this grid's results itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
    // batches of kBatch 16-byte loads per thread, all in flight together; per batch one
    // maximum (and the first index reaching it, in ascending index order), one rescale of
    // the running sum, then the batch's exponentials as independent pairs
    const uint4* x8 = reinterpret_cast<const uint4*>(x);
    const int n8 = V >> 3, lo8 = 0;
    constexpr int kBatch = 4;
    const float2 c2 = make_float2(kLog2e, kLog2e);
    constexpr uint32_t kNegInf2 = 0xFF80FF80u;   // two bf16 -inf
    for (int base = lo8; base < n8; base += kBatch * kScanThreads) {
      uint4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = base + u * kScanThreads + threadIdx.x;
        v[u] = i < n8 ? __ldcs(x8 + i) : make_uint4(kNegInf2, kNegInf2, kNegInf2, kNegInf2);
      }
      // batch maximum and the first index reaching it: four independent trackers (one per
      // 32-bit word of a load), each visiting its values in ascending index order, merged
      // with the lower index winning ties
      float bm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      int barg[4] = {0, 0, 0, 0};
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = base + u * kScanThreads + threadIdx.x;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
          if (lo > bm[k]) {
            bm[k] = lo;
            barg[k] = 8 * i + 2 * k;
          }
          if (hi > bm[k]) {
            bm[k] = hi;
            barg[k] = 8 * i + 2 * k + 1;
          }
        }
      }
#pragma unroll
      for (int k = 1; k < 4; ++k) {
        if (bm[k] > bm[0] || (bm[k] == bm[0] && barg[k] < barg[0])) {
          bm[0] = bm[k];
          barg[0] = barg[k];
        }
      }
      const float z = bm[0] * kLog2e;
      if (z > a.m) {
        a.s *= fast_exp2(a.m - z);
        a.m = z;
        a.arg = barg[0];
      }
      const float2 nm2 = make_float2(-a.m, -a.m);
      float2 s0 = make_float2(0.f, 0.f), s1 = s0;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 t = __ffma2_rn(make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u)),
                                      c2, nm2);
          // one pair in four on the FMA pipe (exp2_poly2, relative error 7.5e-5): the MUFU's
          // exp2 rate bounds the scan together with its loads
          const float2 e = k == 3 ? exp2_poly2(t) : make_float2(fast_exp2(t.x), fast_exp2(t.y));
          if (k & 1) s1 = __fadd2_rn(s1, e);
          else s0 = __fadd2_rn(s0, e);
        }
      }
      a.s += (s0.x + s0.y) + (s1.x + s1.y);
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
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the scan grid's results are complete and visible
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
  // the commit kernel is launched as a programmatic dependent of the scan: its launch
  // overlaps the scan, and it waits for the scan's results on the device
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B, 1, 1);
  cfg.blockDim = dim3(((S + 31) / 32) * 32, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, unmask_commit_kernel, S, gamma, min_one, tokens, masked,
                            static_cast<const float*>(p_max), static_cast<const int32_t*>(argmax), n_committed);
}

}  // namespace tt
