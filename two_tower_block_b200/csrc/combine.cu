// Log-sum-exp combine of the units that a range boundary cut into segments,
// and the bounded-wait self test.
//
// A cut unit's segments each hold O_s = (sum over its keys of e^{s-m_s} v) /
// l_s and lse_s = m_s + ln l_s.  The joint softmax over all keys of the unit
// is recovered exactly: with M = max_s lse_s and w_s = e^{lse_s - M},
//     out = sum_s w_s O_s / sum_s w_s,     lse = M + ln sum_s w_s.
#include "problem.h"
#include "ptx.cuh"
#include "walker.cuh"

namespace tt {
namespace {

constexpr int kRowsPerBlock = 8;   // one warp per row
constexpr int kThreads = 256;
constexpr int kGroup = 8;          // segments whose rows a warp loads together

template <int D>
__global__ void __launch_bounds__(kThreads) combine_kernel(const Problem p) {
  const int c = blockIdx.x;
  const SplitRecord rec = p.records[c];
  if (rec.unit < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * kRowsPerBlock + warp;
  if (r >= p.R) return;
  const Unit x = make_unit(p, rec.unit, 0);
  const int nseg = rec.last_range - c + 1;
  constexpr int V = D / 32;  // columns per lane
  auto slot_of = [&](int s) { return s == 0 ? 2 * c + rec.first_which : 2 * (c + s); };
  auto load_row = [&](int s, float* a) {
    const float* src = p.part_o + ((size_t)slot_of(s) * p.R + r) * D + lane * V;
    if constexpr (V == 4) {
      const float4 t = __ldcg(reinterpret_cast<const float4*>(src));
      a[0] = t.x; a[1] = t.y; a[2] = t.z; a[3] = t.w;
    } else {
      const float2 t = __ldcg(reinterpret_cast<const float2*>(src));
      a[0] = t.x; a[1] = t.y;
    }
  };
  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  float M = -INFINITY, wsum = 0.f;
  // segments in sweeps of 32 (lane s holds segment s0 + s): the lse values and the first
  // kGroup rows are requested together, the rest kGroup at a time
  for (int s0 = 0; s0 < nseg; s0 += 32) {
    const int n = min(32, nseg - s0);
    const float lse_lane = lane < n ? __ldcg(p.part_lse + (size_t)slot_of(s0 + lane) * p.R + r) : -INFINITY;
    float a[kGroup][V];
#pragma unroll
    for (int u = 0; u < kGroup; ++u)
      if (u < n) load_row(s0 + u, a[u]);
    float Ms = lse_lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ms = fmaxf(Ms, __shfl_xor_sync(0xffffffffu, Ms, o));
    // fold this sweep into the running (M, wsum, acc)
    const float Mn = fmaxf(M, Ms);
    const float scale_old = M == -INFINITY ? 0.f : expf(M - Mn);
    wsum *= scale_old;
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] *= scale_old;
    M = Mn;
    const float w_lane = lane < n ? expf(lse_lane - M) : 0.f;
    float ws = w_lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
    wsum += ws;
    for (int k = 0; k < n; k += kGroup) {
      if (k > 0) {
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
          if (k + u < n) load_row(s0 + k + u, a[u]);
      }
#pragma unroll
      for (int u = 0; u < kGroup; ++u) {
        const float w = __shfl_sync(0xffffffffu, w_lane, (k + u) & 31);
        if (k + u < n) {
#pragma unroll
          for (int v = 0; v < V; ++v) acc[v] = fmaf(w, a[u][v], acc[v]);
        }
      }
    }
  }
  const float inv = 1.f / wsum;
  const int t = r / p.g, j = r - (r / p.g) * p.g;
  float* dst = p.out + ((size_t)(x.ns * p.S + t) * p.Hq + x.h * p.g + j) * D + lane * V;
  if constexpr (V == 4) {
    *reinterpret_cast<float4*>(dst) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  } else {
    *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && p.lse)
    p.lse[(size_t)(x.n * p.Hq + x.h * p.g + j) * (p.NB * p.S) + x.b * p.S + t] = M + logf(wsum);
}

// One thread waits on a barrier that nothing arrives at; the bounded wait must
// give up, raise kErrTimeout and return.
__global__ void wait_selftest_kernel(unsigned* err_word, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx w{&abort_flag, err_word, limit_ns};
    if (mbar_wait(smem_u32(&bar), 0, w)) atomicOr(err_word, 0x80000000u);  // must not happen
  }
  __syncthreads();
}

// The FMA-pipe exp2 of the softmax (ptx.cuh: exp2_poly2) on n arguments.
__global__ void exp2_selftest_kernel(const float* x, float* y, int n) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
  if (i + 1 < n) {
    const float2 e = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = e.x;
    y[i + 1] = e.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

}  // namespace

cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t stream) {
  exp2_selftest_kernel<<<(n + 511) / 512, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_combine(const Problem& p, cudaStream_t stream) {
  dim3 grid(p.C, (p.R + kRowsPerBlock - 1) / kRowsPerBlock);
  if (p.D == 128) combine_kernel<128><<<grid, kThreads, 0, stream>>>(p);
  else combine_kernel<64><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(unsigned* err_word, unsigned long long limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(err_word, limit_ns);
  return cudaGetLastError();
}

}  // namespace tt
