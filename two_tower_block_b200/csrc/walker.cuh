// Device-side walk over one range of the global tile sequence (see sched.cuh).
#pragma once
#include "problem.h"
#include "ptx.cuh"
#include "sched.cuh"

namespace tt {

struct Unit {
  int u;          // unit index
  int tiles;      // number of key tiles
  int L;          // visible context keys
  int n, h, b;    // sequence, KV head, block index within the sequence
  int ns;         // block-sequence index n * NB + b (row block of q / k_blk / out)
  long long Tu;   // first global tile of the unit
};

__device__ __forceinline__ int clamp_len(const Problem& p, int n, bool report) {
  int L = __ldg(p.ctx_lens + n);
  if (L < 0 || L > p.ctx_stride) {
    if (report) raise_error(p.err_word, kErrDeviceArg);
    L = L < 0 ? 0 : p.ctx_stride;
  }
  return L;
}

__device__ __forceinline__ int unit_tiles_k(const Problem& p, int L) {
  return p.blk_tiles + ceil_div(L, p.key_tile);
}

__device__ __forceinline__ Unit make_unit(const Problem& p, int u, long long Tu) {
  Unit x;
  x.u = u;
  x.Tu = Tu;
  if (p.mode == kDecode) {
    x.n = u / p.Hkv;
    x.h = u - x.n * p.Hkv;
    x.b = 0;
    x.L = clamp_len(p, x.n, false);
  } else {
    int nh = u / p.NB;
    x.b = u - nh * p.NB;
    x.n = nh / p.Hkv;
    x.h = nh - x.n * p.Hkv;
    x.L = p.S * x.b;
  }
  x.ns = x.n * p.NB + x.b;
  x.tiles = unit_tiles_k(p, x.L);
  return x;
}

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The boundary table of the call's split, or null for the uniform one.
__device__ __forceinline__ const long long* range_table(const Problem& p) {
  return p.mode == kDecode ? nullptr : p.causal_starts;
}

// Called by one full warp.  Finds the total tile count T, this range's
// [start, end) and the unit containing `start` (valid only if start < end).
__device__ __forceinline__ void find_range(const Problem& p, int c, long long& T, long long& start,
                                           long long& end, Unit& first) {
  const int lane = threadIdx.x & 31;
  if (p.mode == kDecode) {
    long long tot = 0;
    for (int base = 0; base < p.B; base += 32) {
      int n = base + lane;
      long long t = 0;
      if (n < p.B) t = (long long)p.Hkv * unit_tiles_k(p, clamp_len(p, n, c == 0));
      tot += warp_sum_ll(t);
    }
    T = tot;
  } else {
    T = p.T_causal;
  }
  const int Ce = used_ranges(T, p.C);
  if (c >= Ce) {
    start = end = T;
    return;
  }
  const long long* tab = range_table(p);
  start = range_start_tab(tab, T, Ce, c);
  end = range_start_tab(tab, T, Ce, c + 1);
  if (p.mode == kDecode) {
    long long acc = 0;
    for (int base = 0; base < p.B; base += 32) {
      int n = base + lane;
      long long t = 0;
      if (n < p.B) t = (long long)p.Hkv * unit_tiles_k(p, clamp_len(p, n, false));
      long long incl = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      long long total = __shfl_sync(0xffffffffu, incl, 31);
      if (acc + total > start) {
        unsigned m = __ballot_sync(0xffffffffu, acc + incl > start);
        int src = __ffs(m) - 1;
        long long pn = acc + __shfl_sync(0xffffffffu, incl - t, src);
        int nn = base + src;
        int tn = unit_tiles_k(p, clamp_len(p, nn, false));
        int h = (int)((start - pn) / tn);
        first = make_unit(p, nn * p.Hkv + h, pn + (long long)h * tn);
        return;
      }
      acc += total;
    }
  } else {
    const long long Tnh = p.causal_pref[p.NB];
    const int nh = (int)(start / Tnh);
    const long long rem = start - (long long)nh * Tnh;
    int lo = 0, hi = p.NB - 1;  // largest b with pref[b] <= rem
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (p.causal_pref[mid] <= rem) lo = mid; else hi = mid - 1;
    }
    first = make_unit(p, nh * p.NB + lo, (long long)nh * Tnh + p.causal_pref[lo]);
  }
}

// Segment of the current unit inside [start, end).
struct Segment {
  int lo, hi;     // unit-local tiles [lo, hi)
  bool full;      // covers the whole unit: write the final output
  int slot;       // partial slot when !full
  bool last;      // last segment of the range
};

__device__ __forceinline__ Segment segment_of(const Unit& x, long long start, long long end, int c) {
  Segment s;
  long long lo = start > x.Tu ? start - x.Tu : 0;
  long long hi = end - x.Tu < x.tiles ? end - x.Tu : x.tiles;
  s.lo = (int)lo;
  s.hi = (int)hi;
  s.full = (s.lo == 0 && s.hi == x.tiles);
  s.slot = 2 * c + ((x.Tu + lo == start) ? 0 : 1);
  s.last = (x.Tu + x.tiles >= end);
  return s;
}

// The record of range c: the cut unit that begins in c and runs past its end.
// C is the plan's range count; the split uses min(C, T) of them.
__device__ __forceinline__ SplitRecord record_of(const Unit& last, long long T, int C, long long start,
                                                 long long end, const long long* tab) {
  C = used_ranges(T, C);
  SplitRecord r;
  r.unit = -1;
  r.last_range = -1;
  r.first_which = 0;
  r.pad = 0;
  if (last.Tu >= start && last.Tu + last.tiles > end) {
    r.unit = last.u;
    r.last_range = range_of_tile_tab(tab, T, C, last.Tu + last.tiles - 1);
    r.first_which = (last.Tu == start) ? 0 : 1;
  }
  return r;
}

// Element offset of packed row r of unit x in the final output [.., S, Hq, D].
__device__ __forceinline__ size_t out_offset(const Problem& p, const Unit& x, int r, int D) {
  const int t = r / p.g, j = r - (r / p.g) * p.g;
  return ((size_t)(x.ns * p.S + t) * p.Hq + x.h * p.g + j) * D;
}
// Four (or two) consecutive final-output values at element offset off: fp32, or bf16 pairs
// rounded to nearest even when the problem asks for a bf16 output.
__device__ __forceinline__ void store_out4(const Problem& p, size_t off, float4 v) {
  if (p.out_bf16) {
    const uint2 u = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + off) = u;
  } else {
    *reinterpret_cast<float4*>(p.out + off) = v;
  }
}
__device__ __forceinline__ void store_out2(const Problem& p, size_t off, float2 v) {
  if (p.out_bf16) *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(p.out) + off) = pack_bf16(v.x, v.y);
  else *reinterpret_cast<float2*>(p.out + off) = v;
}

// Keys of unit-local tile i: block keys for i < blk_tiles, context keys after.
struct TileKeys {
  bool is_blk;
  int first;   // first key index within its source (block position or context position)
  int count;   // valid keys in the tile (>= 1)
};
__device__ __forceinline__ TileKeys tile_keys(const Problem& p, const Unit& x, int i) {
  TileKeys k;
  if (i < p.blk_tiles) {
    k.is_blk = true;
    k.first = i * p.key_tile;
    k.count = min(p.S - k.first, p.key_tile);
  } else {
    k.is_blk = false;
    k.first = (i - p.blk_tiles) * p.key_tile;
    k.count = min(x.L - k.first, p.key_tile);
  }
  return k;
}

// Pool row (of the [num_pages * Hkv * page_size] rows of k_ctx / v_ctx) holding context
// position pos of (n, h) in a paged cache; -1, reported as a device argument error, when
// the page table names a page outside [0, num_pages).
__device__ __forceinline__ int paged_row(const Problem& p, int n, int h, int pos) {
  const int page = __ldg(p.page_table + (size_t)n * p.pages_per_seq + (pos >> p.page_shift));
  if (page < 0 || page >= p.num_pages) {
    raise_error(p.err_word, kErrDeviceArg);
    return -1;
  }
  return ((page * p.Hkv + h) << p.page_shift) + (pos & ((1 << p.page_shift) - 1));
}

}  // namespace tt
