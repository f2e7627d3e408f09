// Device helpers shared by the tcgen05 attention kernels: row maximum and
// exponentials of one key tile of a softmax row held in registers, and the
// output-row address of a packed query row.
#pragma once
#include "problem.h"
#include "ptx.cuh"
#include "walker.cuh"

namespace tt {

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// Output row pointer of packed row r of unit x (final output or segment partial).
__device__ __forceinline__ float* out_row(const Problem& p, const Unit& x, const Segment& sg, int r, int D) {
  if (sg.full) {
    const int t = r / p.g, j = r - (r / p.g) * p.g;
    return p.out + ((size_t)(x.ns * p.S + t) * p.Hq + x.h * p.g + j) * D;
  }
  return p.part_o + ((size_t)sg.slot * p.R + r) * D;
}

// Two non-negative finite weights rounded to bf16 precision on the integer pipe (round half
// up on the magnitude: add half a bf16 ulp, clear the low 16 bits), returned as fp32 bit
// patterns whose high halves are the bf16 values.  This keeps the packed conversion off the
// pipe the exponentials use; only exact ties round differently from round-to-nearest-even.
__device__ __forceinline__ uint2 round_pair_bf16(float a, float b) {
  return make_uint2((__float_as_uint(a) + 0x8000u) & 0xFFFF0000u, (__float_as_uint(b) + 0x8000u) & 0xFFFF0000u);
}

// Row maximum of the first `count` raw scores of a tile (all NK when kFull).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int NK, bool kFull>
__device__ __forceinline__ float tile_row_max(const uint32_t* v, int count) {
  // four running maxima, each taking two new scores per three-input max
  float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int k = 0; k < NK; k += 2) {
    const float x0 = (kFull || k < count) ? __uint_as_float(v[k]) : -INFINITY;
    const float x1 = (kFull || k + 1 < count) ? __uint_as_float(v[k + 1]) : -INFINITY;
    m[(k >> 1) & 3] = max3f(m[(k >> 1) & 3], x0, x1);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// p = 2^(s*c - m_ref) for the tile's keys (0 beyond `count`), rounded to bf16
// (round_pair_bf16) and written to TMEM as pairs over the first columns of the S buffer: keys
// [32ch, 32ch+32) -> columns [16ch, 16ch+16).  Returns the row sum of the
// rounded weights, so that numerator and denominator use the same values.
// One pair in kPolyEvery is computed on the FMA pipe (exp2_poly2, relative error 7.5e-5,
// far below the bf16 rounding that follows) instead of the MUFU, whose exp2 throughput
// bounds this loop; one in eight measured fastest (one in four or three was slower).
constexpr int kPolyEvery = 8;
template <int NK, bool kFull>
__device__ __forceinline__ float tile_exp_store(const uint32_t* v, int count, float c, float m_ref,
                                                uint32_t s_addr) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m_ref, -m_ref);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int ch = 0; ch < NK / 32; ++ch) {
    if (!kFull && 32 * ch >= count) break;
    uint32_t pk[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int c0 = 32 * ch + 2 * k;
      const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[c0]), __uint_as_float(v[c0 + 1])), c2, nm2);
      float a, b;
      if (k % kPolyEvery == kPolyEvery - 1) {
        const float2 e = exp2_poly2(x);
        a = e.x;
        b = e.y;
      } else {
        a = fast_exp2(x.x);
        b = fast_exp2(x.y);
      }
      if (!kFull) {
        a = c0 < count ? a : 0.f;
        b = c0 + 1 < count ? b : 0.f;
      }
      const uint2 r = round_pair_bf16(a, b);
      pk[k] = __byte_perm(r.x, r.y, 0x7632);
      acc = __fadd2_rn(acc, make_float2(__uint_as_float(r.x), __uint_as_float(r.y)));
    }
    tmem_st16(s_addr + 16 * ch, pk);
  }
  return acc.x + acc.y;
}

// p = 2^(s*c - m_ref) for the tile's keys (0 beyond `count`), rounded to bf16 and
// packed in pairs into pk[NK/2] (keys 2k, 2k+1 -> pk[k], low half first).  Returns the
// row sum of the rounded weights.
template <int NK, bool kFull>
__device__ __forceinline__ float tile_exp_pack(const uint32_t* v, int count, float c, float m_ref, uint32_t* pk) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m_ref, -m_ref);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < NK / 2; ++k) {
    const int c0 = 2 * k;
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[c0]), __uint_as_float(v[c0 + 1])), c2, nm2);
    float a = fast_exp2(x.x), b = fast_exp2(x.y);
    if (!kFull) {
      a = c0 < count ? a : 0.f;
      b = c0 + 1 < count ? b : 0.f;
    }
    const uint2 r = round_pair_bf16(a, b);
    pk[k] = __byte_perm(r.x, r.y, 0x7632);
    acc = __fadd2_rn(acc, make_float2(__uint_as_float(r.x), __uint_as_float(r.y)));
  }
  return acc.x + acc.y;
}

}  // namespace tt
