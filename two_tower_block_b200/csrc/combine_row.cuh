// One row of the log-sum-exp combine, done by one warp: used by the combine kernel and
// by the fused tail of the default attention kernel.
//
// A cut unit's segments each hold O_s = (sum over its keys of e^{s-m_s} v) / l_s and
// lse_s = m_s + ln l_s.  The joint softmax over all keys of the unit is recovered
// exactly: with M = max_s lse_s and w_s = e^{lse_s - M},
//     out = sum_s w_s O_s / sum_s w_s,     lse = M + ln sum_s w_s.
// The warp requests every lse value and the first kGroup segments' rows before the first
// use, and folds sweeps of 32 segments online (running maximum, rescaled sums).
#pragma once
#include "problem.h"
#include "sched.cuh"
#include "walker.cuh"

namespace tt {

// kGroup rows are loaded per round: 8 in the separate kernel (more would cost occupancy), 16 in
// the attention kernel's tail, whose registers are there anyway.
template <int D, int kGroup = 8>
__device__ __forceinline__ void combine_row(const Problem& p, int c, const SplitRecord& rec, int r, int lane) {
  constexpr int V = D / 32;  // columns per lane
  const Unit x = make_unit(p, rec.unit, 0);
  const int nseg = rec.last_range - c + 1;
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
  const size_t off = out_offset(p, x, r, D) + lane * V;
  if constexpr (V == 4) {
    store_out4(p, off, make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv));
  } else {
    store_out2(p, off, make_float2(acc[0] * inv, acc[1] * inv));
  }
  if (lane == 0 && p.lse)
    p.lse[(size_t)(x.n * p.Hq + x.h * p.g + j) * (p.NB * p.S) + x.b * p.S + t] = M + logf(wsum);
}

}  // namespace tt
