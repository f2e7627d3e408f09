// C ABI of the block attention library: plans, argument checks, launches,
// host-buffer entry, device error word, per-kernel timing hook.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/tt_block_attn.h"
#include "problem.h"
#include "kv_append.h"
#include "attn_bwd.h"
#include "unmask.h"
#include "errbits.h"
#include "sched.cuh"

// Detail text of the last host-side error on this thread (read by tt_last_error_detail).
namespace tt {
thread_local std::string g_detail;
}
using tt::g_detail;

namespace {

tt_status_t fail(tt_status_t st, const std::string& why) {
  g_detail = why;
  return st;
}
tt_status_t cuda_fail(cudaError_t e, const char* where) {
  g_detail = std::string(where) + ": " + cudaGetErrorString(e);
  return TT_ERR_CUDA;
}

// ---------------------------------------------------------- TMA encoding --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor map with `rank` dims (innermost first), 128-byte swizzle.
bool encode_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                 const uint32_t* box) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) s[i] = strides_bytes[i];
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), d, s, b, e,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int kProfMax = 4096;

}  // namespace

struct tt_plan_s {
  tt_block_attn_desc desc;
  int device = 0;
  int sm_count = 0;
  int kernel = TT_KERNEL_MMA_SYNC;
  int C = 1;
  int C_paged = 1;   // ranges of paged calls (differs from C on 2-SM plans)
  int C_decode = 1;  // ranges of contiguous decode calls
  int key_tile = 64;
  int variant = 0;
  int R = 0, g = 1;
  float scale = 0.f;
  // scratch
  void* ws = nullptr;
  size_t ws_bytes = 0;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  tt::SplitRecord* records = nullptr;
  unsigned* err_word = nullptr;
  // fused combine: per-range arrival counts (only growing) of the decode and paged calls
  // (C_decode ranges) and of the block-causal calls (C ranges); each launch kind keeps its own
  // so that every range of a launch has seen the same number of launches
  unsigned* arr_decode = nullptr;
  unsigned* arr_causal = nullptr;
  bool fused_combine = false;   // block-causal calls combine in the attention kernel's tail
  bool fused_decode = false;    // decode and paged calls do
  int* causal_pref = nullptr;
  long long causal_T = 0;
  long long* causal_starts = nullptr;   // weighted range boundaries of block-causal calls, or null
  int causal_NB = 0;
  // host IO staging
  void* stage = nullptr;
  size_t st_q = 0, st_kc = 0, st_kb = 0, st_lens = 0, st_out = 0, st_lse = 0;
  // timing hook
  bool prof_on = false;
  std::vector<cudaEvent_t> prof_ev;      // 2 * kProfMax
  std::vector<int> prof_kid;
  int prof_n = 0;
};

namespace {

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
    else prev = -1;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void prof_mark(tt_plan_t plan, int kid, cudaStream_t s, bool begin) {
  if (!plan->prof_on) return;
  if (plan->prof_n >= kProfMax) return;
  // in a stream being captured into a graph, the record must become a graph node of its own
  // (cudaEventRecordExternal) for its timestamp to be readable after the graph has run
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  const unsigned flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  if (begin) {
    cudaEventRecordWithFlags(plan->prof_ev[2 * plan->prof_n], s, flags);
    plan->prof_kid[plan->prof_n] = kid;
  } else {
    cudaEventRecordWithFlags(plan->prof_ev[2 * plan->prof_n + 1], s, flags);
    plan->prof_n++;
  }
}

tt::Problem base_problem(tt_plan_t plan) {
  tt::Problem p{};
  const tt_block_attn_desc& d = plan->desc;
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.g = plan->g;
  p.D = d.head_dim;
  p.S = d.block_size;
  p.R = plan->R;
  p.scale_log2 = plan->scale * 1.4426950408889634f;
  p.C = plan->C;
  p.key_tile = plan->key_tile;
  p.blk_tiles = tt::ceil_div(d.block_size, plan->key_tile);
  p.part_o = plan->part_o;
  p.part_lse = plan->part_lse;
  p.records = plan->records;
  p.err_word = plan->err_word;
  p.wait_limit_ns = (unsigned long long)(d.wait_timeout_us > 0 ? d.wait_timeout_us : 1000000) * 1000ull;
  p.variant = plan->variant;
  p.arrivals = nullptr;
  p.out_bf16 = (d.flags & TT_PLAN_OUT_BF16) ? 1 : 0;
  return p;
}

tt_status_t launch_all(tt_plan_t plan, const tt::Problem& p, cudaStream_t s) {
  cudaError_t e;
  prof_mark(plan, 0, s, true);
  if (plan->kernel == TT_KERNEL_TCGEN05 && p.variant == 3) {
    e = tt::launch_attn_2sm(p, s);
  } else if (plan->kernel == TT_KERNEL_TCGEN05) {
    tt::TmaMaps maps;
    memset(&maps, 0, sizeof(maps));
    const uint64_t D = p.D;
    const uint32_t g = p.g, S = p.S, kt = p.key_tile;
    // q viewed as [tokens][Hq][D]; box = one unit's rows (S tokens x g heads x 64 dims)
    {
      uint64_t dims[3] = {D, (uint64_t)p.Hq, (uint64_t)p.B * p.NB * p.S};
      uint64_t str[2] = {D * 2, (uint64_t)p.Hq * D * 2};
      uint32_t box[3] = {64, g, S};
      if (!encode_bf16(&maps.q, p.q, 3, dims, str, box)) return fail(TT_ERR_CUDA, "tensor map (q) encode failed");
    }
    // k_blk / v_blk viewed as [tokens][Hkv][D]; box = min(S, key_tile) tokens of one head
    {
      uint64_t dims[3] = {D, (uint64_t)p.Hkv, (uint64_t)p.B * p.NB * p.S};
      uint64_t str[2] = {D * 2, (uint64_t)p.Hkv * D * 2};
      uint32_t box[3] = {64, 1, std::min(S, kt)};
      if (!encode_bf16(&maps.k_blk, p.k_blk, 3, dims, str, box) ||
          !encode_bf16(&maps.v_blk, p.v_blk, 3, dims, str, box))
        return fail(TT_ERR_CUDA, "tensor map (block kv) encode failed");
    }
    // paged: k_ctx / v_ctx are pools viewed as [num_pages*Hkv*page_size rows][D]; box =
    // min(page_size, key_tile) rows x 64 dims (one page's slice of a tile)
    if (p.page_table && (uint64_t)p.num_pages * p.Hkv * p.ctx_stride > 0) {
      uint64_t dims[2] = {D, ((uint64_t)p.num_pages * p.Hkv) << p.page_shift};
      uint64_t str[1] = {D * 2};
      uint32_t box[2] = {64, std::min(1u << p.page_shift, kt)};
      if (!encode_bf16(&maps.k_ctx, p.k_ctx, 2, dims, str, box) ||
          !encode_bf16(&maps.v_ctx, p.v_ctx, 2, dims, str, box))
        return fail(TT_ERR_CUDA, "tensor map (paged context kv) encode failed");
    } else if (p.page_table) {
      maps.k_ctx = maps.k_blk;  // never read: no context tiles exist
      maps.v_ctx = maps.v_blk;
    } else if ((uint64_t)p.B * p.Hkv * p.ctx_stride > 0) {
      // k_ctx / v_ctx viewed as [B*Hkv*stride rows][D]; box = key_tile rows x 64 dims
      uint64_t dims[2] = {D, (uint64_t)p.B * p.Hkv * p.ctx_stride};
      uint64_t str[1] = {D * 2};
      uint32_t box[2] = {64, kt};
      if (!encode_bf16(&maps.k_ctx, p.k_ctx, 2, dims, str, box) ||
          !encode_bf16(&maps.v_ctx, p.v_ctx, 2, dims, str, box))
        return fail(TT_ERR_CUDA, "tensor map (context kv) encode failed");
    } else {
      maps.k_ctx = maps.k_blk;  // never read: no context tiles exist
      maps.v_ctx = maps.v_blk;
    }
    e = tt::launch_attn_tcgen05(p, maps, s);
  } else {
    e = tt::launch_attn_mma_sync(p, s);
  }
  prof_mark(plan, 0, s, false);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  if (p.C > 1 && p.arrivals == nullptr) {
    prof_mark(plan, 1, s, true);
    e = tt::launch_combine(p, s);
    prof_mark(plan, 1, s, false);
    if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
  }
  return TT_OK;
}

// Range boundaries of the block-causal calls of the default tcgen05 kernel, weighted so that
// every range carries the same modelled time: a unit costs its key tiles plus a fixed cost of
// kCausalUnitCost tiles, half before its first tile (the Q load and the pipeline's restart) and
// half after its last (the output epilogue).  The boundaries split that weighted sequence
// evenly; one that falls in a unit's fixed cost moves to the unit's edge (no cut), one that
// falls among its tiles cuts the unit there.  With the uniform split the first ranges of each
// (n, h), which hold many short units, ran up to 1.7 x the mean range's time; a fixed cost of
// about 8 tiles per unit of two M-tiles reproduces that spread.  TT_CAUSAL_UNIT_COST overrides
// the cost (0: the uniform split, no table).
constexpr int kCausalUnitCost = 8;

// The table for `pairs` (n, h) pairs of NB units each, pref the tile prefix over b (NB + 1
// entries), C ranges and a unit cost of H tiles: min(C, T) + 1 entries, or none when the
// uniform split applies (H = 0 or a single range).
std::vector<long long> weighted_causal_starts(const std::vector<int>& pref, long long pairs, int C, long long H) {
  std::vector<long long> tab;
  if (pref.size() < 2 || pairs <= 0) return tab;
  const int NB = (int)pref.size() - 1;
  const long long T = pairs * pref[NB];
  const int Ce = tt::used_ranges(T, C);
  if (H <= 0 || Ce <= 1) return tab;
  const long long U = pairs * NB;
  const long long H0 = H / 2;          // weight before a unit's first tile
  const long long V = T + H * U;       // weighted length
  tab.assign(Ce + 1, 0);
  tab[Ce] = T;
  long long u = 0, vbase = 0, base = 0;  // unit, its weighted and its tile offset
  for (int c = 1; c < Ce; ++c) {
    const long long v = (long long)((__int128)c * V / Ce);
    for (; u < U; ++u) {
      const int b = (int)(u % NB);
      const long long t = pref[b + 1] - pref[b];
      if (vbase + t + H > v) break;
      vbase += t + H;
      base += t;
    }
    if (u >= U) {
      tab[c] = T;
    } else {
      const int b = (int)(u % NB);
      const long long t = pref[b + 1] - pref[b];
      tab[c] = base + std::min(std::max(v - vbase - H0, 0LL), t);
    }
  }
  // strictly increasing: every range holds at least one tile
  for (int c = 1; c < Ce; ++c) tab[c] = std::max(tab[c], tab[c - 1] + 1);
  for (int c = Ce - 1; c >= 1; --c) tab[c] = std::min(tab[c], tab[c + 1] - 1);
  return tab;
}

std::vector<long long> causal_range_table(const tt_plan_s* P, const std::vector<int>& pref,
                                          const tt_block_attn_desc& d) {
  if (pref.empty() || P->kernel != TT_KERNEL_TCGEN05 || P->variant != 0) return {};
  long long H = kCausalUnitCost;
  if (const char* s = std::getenv("TT_CAUSAL_UNIT_COST")) H = std::max(0, std::atoi(s));
  return weighted_causal_starts(pref, (long long)d.batch * d.num_kv_heads, P->C, H);
}

}  // namespace

extern "C" {

const char* tt_status_string(tt_status_t s) {
  switch (s) {
    case TT_OK: return "ok";
    case TT_ERR_INVALID_ARG: return "invalid argument";
    case TT_ERR_UNSUPPORTED: return "unsupported configuration";
    case TT_ERR_CUDA: return "CUDA error";
    case TT_ERR_DEVICE_ARG: return "device-side argument error (ctx_lens out of range)";
    case TT_ERR_TIMEOUT: return "device-side pipeline wait timed out";
  }
  return "unknown status";
}

const char* tt_last_error_detail(void) { return g_detail.c_str(); }

tt_status_t tt_block_attn_plan(const tt_block_attn_desc* desc, int device, tt_plan_t* out_plan) {
  g_detail.clear();
  if (!desc || !out_plan) return fail(TT_ERR_INVALID_ARG, "null descriptor or output pointer");
  const tt_block_attn_desc d = *desc;
  if (d.batch < 0 || d.num_q_heads < 1 || d.num_kv_heads < 1 || d.block_size < 1 || d.ctx_capacity < 0 ||
      d.seq_len < 0 || d.num_ctas < 0 || d.wait_timeout_us < 0)
    return fail(TT_ERR_INVALID_ARG, "negative or zero size in descriptor");
  if (d.num_q_heads % d.num_kv_heads) return fail(TT_ERR_INVALID_ARG, "num_q_heads % num_kv_heads != 0");
  if (!(d.scale >= 0.f) || std::isinf(d.scale)) return fail(TT_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (d.seq_len % d.block_size) return fail(TT_ERR_INVALID_ARG, "seq_len % block_size != 0");
  if (d.kernel < TT_KERNEL_AUTO || d.kernel > TT_KERNEL_MMA_SYNC) return fail(TT_ERR_INVALID_ARG, "unknown kernel");
  if (d.flags & ~(TT_PLAN_HOST_IO | TT_PLAN_OUT_BF16)) return fail(TT_ERR_INVALID_ARG, "unknown flag bits");
  if (d.head_dim != 64 && d.head_dim != 128) return fail(TT_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  const int g = d.num_q_heads / d.num_kv_heads;
  if ((long long)d.block_size * g > 256) return fail(TT_ERR_UNSUPPORTED, "block_size * (Hq/Hkv) must be <= 256");
  const long long tok = (long long)d.batch * std::max(d.seq_len, d.block_size);
  if ((long long)d.batch * d.num_kv_heads * std::max(d.ctx_capacity, d.seq_len) > (1ll << 31) - 1 ||
      tok * d.num_q_heads > (1ll << 31) - 1)
    return fail(TT_ERR_UNSUPPORTED, "tensor too large (rows beyond 2^31)");

  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
  if (device < 0 || device >= ndev) return fail(TT_ERR_INVALID_ARG, "bad device ordinal");
  DeviceGuard guard(device);
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");

  tt_plan_s* P = new tt_plan_s();
  P->desc = d;
  P->device = device;
  P->sm_count = prop.multiProcessorCount;
  P->g = g;
  P->R = d.block_size * g;
  P->scale = d.scale > 0.f ? d.scale : 1.0f / std::sqrt((float)d.head_dim);
  P->kernel = d.kernel == TT_KERNEL_AUTO ? TT_KERNEL_TCGEN05 : d.kernel;
  if (P->kernel == TT_KERNEL_TCGEN05 && prop.major != 10) P->kernel = TT_KERNEL_MMA_SYNC;
  if (P->kernel == TT_KERNEL_TCGEN05) {
    P->key_tile = tt::kTcgen05KeyTile;
    // tuning knobs: TT_TCGEN05_KEY_TILE=128 selects the one-buffer 128-key pipeline;
    // TT_TCGEN05_VARIANT=2 selects the transposed-PV kernel for head_dim 128,
    // TT_TCGEN05_VARIANT=3 the 2-SM kernel (head_dim 128, 128 % g == 0); both run 128-key
    // tiles, which they select unless a key tile is given
    if (const char* kv = std::getenv("TT_TCGEN05_VARIANT")) {
      const int v = std::atoi(kv);
      P->variant = (v == 2 || v == 3) ? v : 0;
      if (P->variant != 0) P->key_tile = 128;
    }
    if (const char* kt = std::getenv("TT_TCGEN05_KEY_TILE")) {
      const int v = std::atoi(kt);
      if (tt::tcgen05_key_tile_supported(v)) P->key_tile = v;
    }
    if (P->variant == 3 && (!tt::attn_2sm_supported(d.head_dim, g) || P->key_tile != 128)) P->variant = 0;
    // the bf16 output is written by the default kernel's epilogue (and the combine): the
    // transposed-PV and 2-SM forms, selectable for fp32 output only, fall back to it
    if ((d.flags & TT_PLAN_OUT_BF16) && P->variant != 0) {
      P->variant = 0;
      P->key_tile = tt::kTcgen05KeyTile;
    }
    P->C = d.num_ctas > 0 ? d.num_ctas : P->sm_count;
    if (P->variant == 3) {
      // one range per cluster of two CTAs; by default as many as can be resident at once
      const int clusters = tt::attn_2sm_max_clusters();
      if (clusters <= 0) P->variant = 0;
      else if (d.num_ctas <= 0) P->C = clusters;
    }
  } else {
    P->key_tile = tt::kMmaSyncKeyTile;
    const int rb = (P->R + 63) / 64;
    P->C = d.num_ctas > 0 ? d.num_ctas : std::max(1, (4 * P->sm_count) / rb);
  }

  // block-causal tile prefix over block index b (identical for every (n, h))
  std::vector<int> pref;
  if (d.seq_len > 0) {
    const int NB = d.seq_len / d.block_size;
    pref.resize(NB + 1);
    long long acc = 0;
    for (int b = 0; b <= NB; ++b) {
      pref[b] = (int)acc;
      if (b < NB) acc += tt::ceil_div(d.block_size, P->key_tile) + tt::ceil_div(d.block_size * b, P->key_tile);
    }
    if (acc > (1ll << 31) - 1) {
      delete P;
      return fail(TT_ERR_UNSUPPORTED, "sequence too long");
    }
    P->causal_NB = NB;
    P->causal_T = (long long)d.batch * d.num_kv_heads * acc;
  }

  // Decode calls on the default tcgen05 kernel: with U = batch * Hkv units and at least two
  // ranges per unit, U * floor(SMs / U) ranges put every unit boundary on a range boundary when
  // the context lengths are equal, so no range carries a second segment (its extra Q load and
  // partial epilogue) at the cost of fewer than U idle SMs.  Ragged lengths are split as before.
  P->C_decode = P->C;
  bool decode_aligned = false;   // every unit of a decode call gets at least two ranges
  if (P->kernel == TT_KERNEL_TCGEN05 && P->variant == 0 && d.num_ctas <= 0) {
    const long long U = (long long)d.batch * d.num_kv_heads;
    if (U > 0 && P->sm_count / U >= 2) {
      P->C_decode = (int)(U * (P->sm_count / U));
      decode_aligned = true;
    }
  }
  // scratch layout (256-byte aligned pieces).  A 2-SM plan runs one range per SM pair, but
  // its paged calls run on the one-CTA-per-SM kernel: room for one range per SM as well.
  P->C_paged = (P->kernel == TT_KERNEL_TCGEN05 && P->variant == 3 && d.num_ctas <= 0) ? P->sm_count : P->C;
  const int Cmax = std::max(P->C, P->C_paged);
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t b_po = up((size_t)2 * Cmax * P->R * d.head_dim * sizeof(float));
  const size_t b_pl = up((size_t)2 * Cmax * P->R * sizeof(float));
  const size_t b_rec = up((size_t)Cmax * sizeof(tt::SplitRecord));
  const size_t b_err = 256;
  const size_t b_pref = up(pref.size() * sizeof(int));
  const size_t b_arr = up((size_t)2 * Cmax * sizeof(unsigned));
  const std::vector<long long> tab = causal_range_table(P, pref, d);
  const size_t b_tab = up(tab.size() * sizeof(long long));
  P->ws_bytes = b_po + b_pl + b_rec + b_err + b_pref + b_arr + b_tab;
  e = cudaMalloc(&P->ws, P->ws_bytes);
  if (e != cudaSuccess) {
    delete P;
    return cuda_fail(e, "cudaMalloc(workspace)");
  }
  char* w = static_cast<char*>(P->ws);
  P->part_o = reinterpret_cast<float*>(w);
  P->part_lse = reinterpret_cast<float*>(w + b_po);
  P->records = reinterpret_cast<tt::SplitRecord*>(w + b_po + b_pl);
  P->err_word = reinterpret_cast<unsigned*>(w + b_po + b_pl + b_rec);
  P->arr_decode = reinterpret_cast<unsigned*>(w + b_po + b_pl + b_rec + b_err + b_pref);
  P->arr_causal = P->arr_decode + Cmax;
  // The fused combine: the default tcgen05 kernel combines the cut units itself, in a
  // cooperative launch (all CTAs resident, one per SM) in which the ranges of each cut unit
  // wait for one another and share its rows, so a call is one launch.  It is the default for
  // decode and paged calls when every unit gets at least two ranges (the aligned split above)
  // and a range holds at most 32 key tiles at the plan's (non-zero) context capacity: there the
  // combine's fixed cost is a large share of a short step (L = 4096: step 36.0 -> 33.3 us).
  // With long ranges the step gains little (L = 131072: 154.9 -> 153.5 us) while the
  // attention kernel's own time grows by the combine's work; with fewer ranges per unit
  // (ragged batches: 213 vs 225 us at B = 64) and for block-causal calls the separate combine
  // kernel measured faster.  TT_FUSED_COMBINE=1 fuses every call of the plan, =0 none.
  {
    const char* fc = std::getenv("TT_FUSED_COMBINE");
    const int force = fc ? std::atoi(fc) : -1;
    const bool can = P->kernel == TT_KERNEL_TCGEN05 && P->variant == 0 && P->C > 1 && P->C <= P->sm_count;
    P->fused_combine = can && force == 1;
    const long long unit_tiles = 1 + (long long)tt::ceil_div(d.ctx_capacity, P->key_tile);
    // (a plan without a context capacity serves paged calls, whose lengths it cannot bound)
    const bool short_ranges = decode_aligned && d.ctx_capacity > 0 &&
                              unit_tiles * d.batch * d.num_kv_heads <= 32LL * std::max(P->C_decode, 1);
    P->fused_decode = can && P->C_decode <= P->sm_count && (force == 1 || (force != 0 && short_ranges));
  }
  P->causal_pref = pref.empty() ? nullptr : reinterpret_cast<int*>(w + b_po + b_pl + b_rec + b_err);
  P->causal_starts = tab.empty() ? nullptr : reinterpret_cast<long long*>(w + b_po + b_pl + b_rec + b_err + b_pref + b_arr);
  e = cudaMemset(P->err_word, 0, b_err);
  if (e == cudaSuccess) e = cudaMemset(P->arr_decode, 0, b_arr);
  if (e == cudaSuccess && !pref.empty())
    e = cudaMemcpy(P->causal_pref, pref.data(), pref.size() * sizeof(int), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && !tab.empty())
    e = cudaMemcpy(P->causal_starts, tab.data(), tab.size() * sizeof(long long), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(P->ws);
    delete P;
    return cuda_fail(e, "workspace init");
  }

  if (d.flags & TT_PLAN_HOST_IO) {
    const size_t B = d.batch, S = d.block_size, Hq = d.num_q_heads, Hkv = d.num_kv_heads, D = d.head_dim;
    P->st_q = up(B * S * Hq * D * 2);
    P->st_kc = up(B * Hkv * (size_t)d.ctx_capacity * D * 2);
    P->st_kb = up(B * S * Hkv * D * 2);
    P->st_lens = up(B * 4);
    P->st_out = up(B * S * Hq * D * ((d.flags & TT_PLAN_OUT_BF16) ? 2 : 4));
    P->st_lse = up(B * Hq * S * 4);
    const size_t tot = P->st_q + 2 * P->st_kc + 2 * P->st_kb + P->st_lens + P->st_out + P->st_lse;
    e = cudaMalloc(&P->stage, std::max<size_t>(tot, 256));
    if (e != cudaSuccess) {
      cudaFree(P->ws);
      delete P;
      return cuda_fail(e, "cudaMalloc(host-io staging)");
    }
  }
  *out_plan = P;
  return TT_OK;
}

void tt_block_attn_plan_destroy(tt_plan_t plan) {
  if (!plan) return;
  DeviceGuard guard(plan->device);
  for (cudaEvent_t ev : plan->prof_ev) cudaEventDestroy(ev);
  if (plan->ws) cudaFree(plan->ws);
  if (plan->stage) cudaFree(plan->stage);
  delete plan;
}

tt_status_t tt_block_attn_plan_get_info(tt_plan_t plan, tt_plan_info* info) {
  if (!plan || !info) return fail(TT_ERR_INVALID_ARG, "null plan or info");
  info->kernel = plan->kernel;
  info->num_ctas = plan->C;
  info->key_tile = plan->key_tile;
  info->rows_per_unit = plan->R;
  info->workspace_bytes = plan->ws_bytes;
  info->sm_count = plan->sm_count;
  info->variant = plan->kernel == TT_KERNEL_TCGEN05 ? plan->variant : 0;
  info->fused_combine = plan->fused_decode ? 1 : 0;
  return TT_OK;
}

tt_status_t tt_block_attn(tt_plan_t plan, const void* q, const void* k_ctx, const void* v_ctx, const void* k_blk,
                          const void* v_blk, const int32_t* ctx_lens, float* out, float* lse, tt_stream_t stream) {
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  const tt_block_attn_desc& d = plan->desc;
  if (d.batch == 0) return TT_OK;
  if (!q || !k_blk || !v_blk || !ctx_lens || !out) return fail(TT_ERR_INVALID_ARG, "null tensor pointer");
  if (d.ctx_capacity > 0 && (!k_ctx || !v_ctx)) return fail(TT_ERR_INVALID_ARG, "null context pointer");
  if (!aligned16(q) || !aligned16(k_ctx) || !aligned16(v_ctx) || !aligned16(k_blk) || !aligned16(v_blk) ||
      !aligned16(out) || !aligned16(lse) || (reinterpret_cast<uintptr_t>(ctx_lens) & 3u))
    return fail(TT_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  DeviceGuard guard(plan->device);
  tt::Problem p = base_problem(plan);
  p.C = plan->C_decode;
  p.arrivals = plan->fused_decode ? plan->arr_decode : nullptr;
  p.mode = tt::kDecode;
  p.NB = 1;
  p.ctx_stride = d.ctx_capacity;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_ctx = static_cast<const __nv_bfloat16*>(k_ctx);
  p.v_ctx = static_cast<const __nv_bfloat16*>(v_ctx);
  p.k_blk = static_cast<const __nv_bfloat16*>(k_blk);
  p.v_blk = static_cast<const __nv_bfloat16*>(v_blk);
  p.ctx_lens = ctx_lens;
  p.out = out;
  p.lse = lse;
  return launch_all(plan, p, reinterpret_cast<cudaStream_t>(stream));
}

tt_status_t tt_block_attn_paged(tt_plan_t plan, const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* page_table, int32_t num_pages, int32_t page_size,
                                int32_t pages_per_seq, const void* k_blk, const void* v_blk, const int32_t* ctx_lens,
                                float* out, float* lse, tt_stream_t stream) {
  if (page_size < 16 || page_size > (1 << 16) || (page_size & (page_size - 1)))
    return fail(TT_ERR_INVALID_ARG, "page_size must be a power of two in [16, 65536]");
  if (num_pages < 0 || pages_per_seq < 0) return fail(TT_ERR_INVALID_ARG, "negative num_pages or pages_per_seq");
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  const tt_block_attn_desc& d = plan->desc;
  if ((long long)pages_per_seq * page_size > (1ll << 31) - 1 ||
      (long long)num_pages * d.num_kv_heads * page_size > (1ll << 31) - 1)
    return fail(TT_ERR_UNSUPPORTED, "page pool or page table too large (rows beyond 2^31)");
  if (d.batch == 0) return TT_OK;
  if (!q || !k_blk || !v_blk || !ctx_lens || !out) return fail(TT_ERR_INVALID_ARG, "null tensor pointer");
  if (pages_per_seq > 0 && (!page_table || !k_pages || !v_pages || num_pages < 1))
    return fail(TT_ERR_INVALID_ARG, "pages_per_seq > 0 needs a page table and non-empty pools");
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(k_blk) || !aligned16(v_blk) ||
      !aligned16(out) || !aligned16(lse) || (reinterpret_cast<uintptr_t>(ctx_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u))
    return fail(TT_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  DeviceGuard guard(plan->device);
  tt::Problem p = base_problem(plan);
  p.mode = tt::kDecode;
  p.NB = 1;
  p.variant = 0;  // the paged loads live in the default tcgen05 kernel (and the mma.sync one)
  p.C = plan->variant == 3 ? plan->C_paged : plan->C_decode;
  p.arrivals = plan->fused_decode ? plan->arr_decode : nullptr;
  p.ctx_stride = pages_per_seq * page_size;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  p.page_shift = shift;
  p.pages_per_seq = pages_per_seq;
  p.num_pages = num_pages;
  p.page_table = pages_per_seq > 0 ? page_table : nullptr;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_ctx = static_cast<const __nv_bfloat16*>(k_pages);
  p.v_ctx = static_cast<const __nv_bfloat16*>(v_pages);
  p.k_blk = static_cast<const __nv_bfloat16*>(k_blk);
  p.v_blk = static_cast<const __nv_bfloat16*>(v_blk);
  p.ctx_lens = ctx_lens;
  p.out = out;
  p.lse = lse;
  return launch_all(plan, p, reinterpret_cast<cudaStream_t>(stream));
}

tt_status_t tt_block_attn_block_causal(tt_plan_t plan, const void* q, const void* k_ctx, const void* v_ctx,
                                       const void* k_blk, const void* v_blk, float* out, float* lse,
                                       tt_stream_t stream) {
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  const tt_block_attn_desc& d = plan->desc;
  if (d.seq_len == 0) return fail(TT_ERR_INVALID_ARG, "plan has seq_len == 0 (decode-only)");
  if (d.batch == 0) return TT_OK;
  if (!q || !k_ctx || !v_ctx || !k_blk || !v_blk || !out) return fail(TT_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k_ctx) || !aligned16(v_ctx) || !aligned16(k_blk) || !aligned16(v_blk) ||
      !aligned16(out) || !aligned16(lse))
    return fail(TT_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  DeviceGuard guard(plan->device);
  tt::Problem p = base_problem(plan);
  p.mode = tt::kBlockCausal;
  p.NB = plan->causal_NB;
  p.arrivals = plan->fused_combine ? plan->arr_causal : nullptr;
  p.ctx_stride = d.seq_len;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_ctx = static_cast<const __nv_bfloat16*>(k_ctx);
  p.v_ctx = static_cast<const __nv_bfloat16*>(v_ctx);
  p.k_blk = static_cast<const __nv_bfloat16*>(k_blk);
  p.v_blk = static_cast<const __nv_bfloat16*>(v_blk);
  p.ctx_lens = nullptr;
  p.out = out;
  p.lse = lse;
  p.T_causal = plan->causal_T;
  p.causal_pref = plan->causal_pref;
  p.causal_starts = plan->causal_starts;
  return launch_all(plan, p, reinterpret_cast<cudaStream_t>(stream));
}

tt_status_t tt_block_attn_host(tt_plan_t plan, const void* q, const void* k_ctx, const void* v_ctx, const void* k_blk,
                               const void* v_blk, const int32_t* ctx_lens, float* out, float* lse,
                               tt_stream_t stream) {
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  if (!plan->stage) return fail(TT_ERR_INVALID_ARG, "plan was created without TT_PLAN_HOST_IO");
  const tt_block_attn_desc& d = plan->desc;
  if (d.batch == 0) return TT_OK;
  if (!q || !k_blk || !v_blk || !ctx_lens || !out || (d.ctx_capacity > 0 && (!k_ctx || !v_ctx)))
    return fail(TT_ERR_INVALID_ARG, "null host pointer");
  DeviceGuard guard(plan->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* st = static_cast<char*>(plan->stage);
  const size_t B = d.batch, S = d.block_size, Hq = d.num_q_heads, Hkv = d.num_kv_heads, D = d.head_dim;
  char* dq = st;
  char* dkc = dq + plan->st_q;
  char* dvc = dkc + plan->st_kc;
  char* dkb = dvc + plan->st_kc;
  char* dvb = dkb + plan->st_kb;
  char* dl = dvb + plan->st_kb;
  char* dout = dl + plan->st_lens;
  char* dlse = dout + plan->st_out;
  const size_t nq = B * S * Hq * D * 2, nkc = B * Hkv * (size_t)d.ctx_capacity * D * 2, nkb = B * S * Hkv * D * 2;
  cudaError_t e = cudaSuccess;
  // one cudaMemcpyAsync per buffer
  if (e == cudaSuccess) e = cudaMemcpyAsync(dq, q, nq, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && nkc) e = cudaMemcpyAsync(dkc, k_ctx, nkc, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && nkc) e = cudaMemcpyAsync(dvc, v_ctx, nkc, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dkb, k_blk, nkb, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dvb, v_blk, nkb, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dl, ctx_lens, B * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
  tt_status_t r = tt_block_attn(plan, dq, nkc ? dkc : nullptr, nkc ? dvc : nullptr, dkb, dvb,
                                reinterpret_cast<const int32_t*>(dl), reinterpret_cast<float*>(dout),
                                lse ? reinterpret_cast<float*>(dlse) : nullptr, stream);
  if (r != TT_OK) return r;
  e = cudaMemcpyAsync(out, dout, B * S * Hq * D * ((d.flags & TT_PLAN_OUT_BF16) ? 2 : 4), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && lse) e = cudaMemcpyAsync(lse, dlse, B * Hq * S * 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  return TT_OK;
}

tt_status_t tt_block_attn_block_causal_backward(tt_plan_t plan, const void* q, const void* k_ctx, const void* v_ctx,
                                                const void* k_blk, const void* v_blk, const float* out,
                                                const float* lse, const void* dout, float* dq, float* dk_blk,
                                                float* dv_blk, tt_stream_t stream) {
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  const tt_block_attn_desc& d = plan->desc;
  if (d.seq_len == 0) return fail(TT_ERR_INVALID_ARG, "plan has seq_len == 0 (decode-only)");
  if (d.flags & TT_PLAN_OUT_BF16)
    return fail(TT_ERR_UNSUPPORTED, "the backward takes the fp32 forward output: use a plan without TT_PLAN_OUT_BF16");
  if (d.batch == 0) return TT_OK;
  if (!q || !k_ctx || !v_ctx || !k_blk || !v_blk || !out || !lse || !dout || !dq || !dk_blk || !dv_blk)
    return fail(TT_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k_ctx) || !aligned16(v_ctx) || !aligned16(k_blk) || !aligned16(v_blk) ||
      !aligned16(out) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk_blk) || !aligned16(dv_blk) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(TT_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  DeviceGuard guard(plan->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  tt::BwdProblem p{};
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.g = plan->g;
  p.D = d.head_dim;
  p.S = d.block_size;
  p.R = plan->R;
  p.N = d.seq_len;
  p.NB = d.seq_len / d.block_size;
  p.scale = plan->scale;
  p.scale_log2 = plan->scale * 1.4426950408889634f;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_ctx = static_cast<const __nv_bfloat16*>(k_ctx);
  p.v_ctx = static_cast<const __nv_bfloat16*>(v_ctx);
  p.k_blk = static_cast<const __nv_bfloat16*>(k_blk);
  p.v_blk = static_cast<const __nv_bfloat16*>(v_blk);
  p.out = out;
  p.lse = lse;
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.dq = dq;
  p.dk_blk = dk_blk;
  p.dv_blk = dv_blk;
  const size_t kv_bytes = (size_t)d.batch * d.seq_len * d.num_kv_heads * d.head_dim * sizeof(float);
  cudaError_t e = cudaMemsetAsync(dk_blk, 0, kv_bytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dv_blk, 0, kv_bytes, s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing dk_blk / dv_blk");
  p.err_word = plan->err_word;
  p.wait_limit_ns = (unsigned long long)(d.wait_timeout_us > 0 ? d.wait_timeout_us : 1000000) * 1000ull;
  // tcgen05 backward on sm_100 plans whose shape it covers (TT_BWD_KERNEL=mma_sync selects
  // the warp-level kernel); the warp-level kernel takes every other shape
  bool use_tc = plan->kernel == TT_KERNEL_TCGEN05 && tt::attn_bwd_tc_supported(p);
  if (const char* bk = std::getenv("TT_BWD_KERNEL")) use_tc = use_tc && std::strcmp(bk, "mma_sync") != 0;
  tt::BwdMaps maps;
  if (use_tc) {
    memset(&maps, 0, sizeof(maps));
    const uint64_t D = p.D;
    const uint32_t tpm = p.R > 128 ? 128u / (uint32_t)p.g : (uint32_t)p.S;   // tokens of one M-tile
    uint64_t qd[3] = {D, (uint64_t)p.Hq, (uint64_t)p.B * p.N};
    uint64_t qs[2] = {D * 2, (uint64_t)p.Hq * D * 2};
    uint32_t qb[3] = {64, (uint32_t)p.g, tpm};
    uint64_t cd[2] = {D, (uint64_t)p.B * p.Hkv * p.N};
    uint64_t cs[1] = {D * 2};
    uint32_t cb[2] = {64, 64};
    uint64_t bd[3] = {D, (uint64_t)p.Hkv, (uint64_t)p.B * p.N};
    uint64_t bs[2] = {D * 2, (uint64_t)p.Hkv * D * 2};
    uint32_t bb[3] = {64, 1, (uint32_t)std::min(p.S, 64)};
    if (!encode_bf16(&maps.q, p.q, 3, qd, qs, qb) || !encode_bf16(&maps.dout, p.dout, 3, qd, qs, qb) ||
        !encode_bf16(&maps.k_ctx, p.k_ctx, 2, cd, cs, cb) || !encode_bf16(&maps.v_ctx, p.v_ctx, 2, cd, cs, cb) ||
        !encode_bf16(&maps.k_blk, p.k_blk, 3, bd, bs, bb) || !encode_bf16(&maps.v_blk, p.v_blk, 3, bd, bs, bb))
      return fail(TT_ERR_CUDA, "tensor map (backward) encode failed");
  }
  prof_mark(plan, 2, s, true);
  e = use_tc ? tt::launch_attn_bwd_tc(p, maps, plan->sm_count, s) : tt::launch_attn_bwd(p, s);
  prof_mark(plan, 2, s, false);
  if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
  return TT_OK;
}

tt_status_t tt_confidence_unmask(const void* logits, int batch, int block, int vocab, float gamma, int min_one,
                                 int32_t* tokens, uint8_t* masked, float* p_max, int32_t* argmax, int32_t* n_committed,
                                 tt_stream_t stream) {
  if (batch < 0 || block < 1 || block > 1024 || vocab < 1)
    return fail(TT_ERR_INVALID_ARG, "need batch >= 0, 1 <= block <= 1024, vocab >= 1");
  if (batch == 0) return TT_OK;
  if (!logits || !tokens || !masked || !p_max || !argmax) return fail(TT_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(logits) || (reinterpret_cast<uintptr_t>(tokens) & 3u) || (reinterpret_cast<uintptr_t>(p_max) & 3u) ||
      (reinterpret_cast<uintptr_t>(argmax) & 3u) || (reinterpret_cast<uintptr_t>(n_committed) & 3u))
    return fail(TT_ERR_INVALID_ARG, "logits must be 16-byte aligned, the int/float arrays 4-byte aligned");
  cudaError_t e = tt::launch_confidence_unmask(logits, batch, block, vocab, gamma, min_one ? 1 : 0, tokens, masked,
                                               p_max, argmax, n_committed, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "confidence unmask launch");
  return TT_OK;
}

tt_status_t tt_kv_append(tt_plan_t plan, const void* k_new, const void* v_new, void* k_ctx, void* v_ctx,
                         int32_t* ctx_lens, int advance, tt_stream_t stream) {
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  const tt_block_attn_desc& d = plan->desc;
  if (d.batch == 0) return TT_OK;
  if (d.ctx_capacity < d.block_size) return fail(TT_ERR_INVALID_ARG, "plan's ctx_capacity has no room for a block");
  if (!k_new || !v_new || !k_ctx || !v_ctx || !ctx_lens) return fail(TT_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_ctx) || !aligned16(v_ctx) ||
      (reinterpret_cast<uintptr_t>(ctx_lens) & 3u))
    return fail(TT_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  DeviceGuard guard(plan->device);
  cudaError_t e = tt::launch_kv_append(k_new, v_new, k_ctx, v_ctx, ctx_lens, d.batch, d.block_size, d.num_kv_heads,
                                       d.head_dim, d.ctx_capacity, advance ? 1 : 0, plan->err_word,
                                       reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kv_append launch");
  return TT_OK;
}

tt_status_t tt_block_attn_check(tt_plan_t plan, tt_stream_t stream) {
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  DeviceGuard guard(plan->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned w = 0;
  e = cudaMemcpy(&w, plan->err_word, sizeof(w), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(plan->err_word, 0, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (w & tt::kErrInternal) return fail(TT_ERR_CUDA, "a kernel found its launch unusable (internal error)");
  if (w & tt::kErrTimeout) return fail(TT_ERR_TIMEOUT, "an in-kernel wait timed out");
  if (w & tt::kErrDeviceArg)
    return fail(TT_ERR_DEVICE_ARG,
                "ctx_lens value out of range (attention: [0, ctx_capacity]; kv append: [0, ctx_capacity - block])");
  return TT_OK;
}

tt_status_t tt_block_attn_profile(tt_plan_t plan, int enable) {
  if (!plan) return fail(TT_ERR_INVALID_ARG, "null plan");
  DeviceGuard guard(plan->device);
  if (enable && plan->prof_ev.empty()) {
    plan->prof_ev.resize(2 * kProfMax);
    plan->prof_kid.resize(kProfMax);
    for (auto& ev : plan->prof_ev) {
      cudaError_t e = cudaEventCreate(&ev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
    }
  }
  plan->prof_on = enable != 0;
  plan->prof_n = 0;
  return TT_OK;
}

tt_status_t tt_block_attn_profile_read(tt_plan_t plan, int kernel_id, int* launches, double* total_ms) {
  if (!plan || !launches || !total_ms) return fail(TT_ERR_INVALID_ARG, "null argument");
  DeviceGuard guard(plan->device);
  int n = 0;
  double tot = 0.0;
  for (int i = 0; i < plan->prof_n; ++i) {
    if (plan->prof_kid[i] != kernel_id) continue;
    cudaError_t e = cudaEventSynchronize(plan->prof_ev[2 * i + 1]);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, plan->prof_ev[2 * i], plan->prof_ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "reading profile events");
    tot += ms;
    ++n;
  }
  *launches = n;
  *total_ms = tot;
  return TT_OK;
}

tt_status_t tt_selftest_wait_timeout(int device, int timeout_us, tt_stream_t stream) {
  if (timeout_us <= 0) return fail(TT_ERR_INVALID_ARG, "timeout_us must be > 0");
  DeviceGuard guard(device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned* w = nullptr;
  cudaError_t e = cudaMalloc(&w, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc");
  e = cudaMemsetAsync(w, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = tt::launch_wait_selftest(w, (unsigned long long)timeout_us * 1000ull, s);
  unsigned h = 0;
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&h, w, sizeof(h), cudaMemcpyDeviceToHost);
  cudaFree(w);
  if (e != cudaSuccess) return cuda_fail(e, "wait self test");
  if (h & 0x80000000u) return fail(TT_ERR_INVALID_ARG, "self test: a wait on a barrier nothing arrives at returned");
  if (h & tt::kErrTimeout) return TT_ERR_TIMEOUT;
  return TT_OK;
}

tt_status_t tt_selftest_exp2(int device, const float* x, float* y, int n) {
  if (n < 0 || (n > 0 && (!x || !y))) return fail(TT_ERR_INVALID_ARG, "bad arguments");
  if (n == 0) return TT_OK;
  DeviceGuard guard(device);
  float* d = nullptr;
  cudaError_t e = cudaMalloc(&d, sizeof(float) * 2 * (size_t)n);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc");
  e = cudaMemcpy(d, x, sizeof(float) * n, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = tt::launch_exp2_selftest(d, d + n, n, 0);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(y, d + n, sizeof(float) * n, cudaMemcpyDeviceToHost);
  cudaFree(d);
  if (e != cudaSuccess) return cuda_fail(e, "exp2 self test");
  return TT_OK;
}

tt_status_t tt_debug_work_split(int num_units, const int* tiles_per_unit, int num_ctas, long long* range_start,
                                int* unit_first, int* unit_last) {
  if (num_units < 0 || num_ctas < 1 || (num_units > 0 && (!tiles_per_unit || !unit_first || !unit_last)) ||
      !range_start)
    return fail(TT_ERR_INVALID_ARG, "bad arguments");
  long long T = 0;
  for (int u = 0; u < num_units; ++u) {
    if (tiles_per_unit[u] < 1) return fail(TT_ERR_INVALID_ARG, "every unit has at least one tile");
    T += tiles_per_unit[u];
  }
  const int Ce = tt::used_ranges(T, num_ctas);
  for (int c = 0; c <= num_ctas; ++c) range_start[c] = c <= Ce ? tt::range_start(T, Ce, c) : T;
  long long Tu = 0;
  for (int u = 0; u < num_units; ++u) {
    unit_first[u] = tt::range_of_tile(T, Ce, Tu);
    unit_last[u] = tt::range_of_tile(T, Ce, Tu + tiles_per_unit[u] - 1);
    Tu += tiles_per_unit[u];
  }
  return TT_OK;
}

tt_status_t tt_debug_causal_split(int batch, int num_kv_heads, int seq_len, int block_size, int key_tile,
                                  int num_ctas, int unit_cost, long long* range_start) {
  if (batch < 1 || num_kv_heads < 1 || block_size < 1 || seq_len < block_size || seq_len % block_size != 0 ||
      key_tile < 1 || num_ctas < 1 || !range_start)
    return fail(TT_ERR_INVALID_ARG, "bad arguments");
  const int NB = seq_len / block_size;
  std::vector<int> pref(NB + 1);
  long long acc = 0;
  for (int b = 0; b <= NB; ++b) {
    pref[b] = (int)acc;
    if (b < NB) acc += tt::ceil_div(block_size, key_tile) + tt::ceil_div(block_size * b, key_tile);
    if (acc > (1ll << 31) - 1) return fail(TT_ERR_UNSUPPORTED, "sequence too long");
  }
  const long long T = (long long)batch * num_kv_heads * acc;
  const std::vector<long long> tab =
      weighted_causal_starts(pref, (long long)batch * num_kv_heads, num_ctas, unit_cost < 0 ? kCausalUnitCost : unit_cost);
  const int Ce = tt::used_ranges(T, num_ctas);
  for (int c = 0; c <= num_ctas; ++c)
    range_start[c] = c > Ce ? T : tab.empty() ? tt::range_start(T, Ce, c) : tab[c];
  return TT_OK;
}

}  // extern "C"
