// Block-causal backward pass on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The method (paperfeed.app review of arXiv 2606.26493, section "Training and
// sampling"): the loss of block b is conditioned on the noisy block and the frozen
// context-tower caches c_{<b}; the context tower runs without gradients.  For the rows
// r of block b and the keys k of its key set (context positions < S*b, then the block's
// own S positions):
//     p = exp(scale q.k - lse),  dp = dO.v,  ds = p (dp - Delta),  Delta = dO.out
//     dq = scale sum_k ds k,  dk_blk += scale ds q,  dv_blk += p dO   (block keys only)
//
// Work item = (sequence, KV head, block, 128-row M-tile of the unit's S*g packed rows).
// Persistent CTAs (one per SM) take items round-robin in order of decreasing block
// index, i.e. heaviest first.  Roles (384 threads):
//   warp 0       TMA producer: Q and dO of the item, then K and V of its key tiles
//                (tile 0 = the block's own keys, tiles 1.. = its visible context, 64
//                keys each) into a ring of shared-memory slots (128-byte swizzle)
//   warp 1       TMEM owner and MMA issuer (one elected lane issues):
//                  S(j) = Q K(j)^T and dP(j) = dO V(j)^T into TMEM buffer j % 2 with Q
//                  and dO read from TMEM (A operands), K and V from shared memory,
//                  dQ += dS(j) K(j) with dS read from TMEM as a bf16 pair hi + lo
//   warps 2, 3   block reducer: dK = scale dS^T Q and dV = P^T dO over the item's rows
//                for the block's own keys (fp32 FMAs on the staged P and dS), added to
//                dk_blk / dv_blk with fp32 atomics (the unit's M-tiles and the g query
//                heads of a KV head all contribute)
//   warps 4..7   softmax warpgroup of the even tiles, warps 8..11 of the odd tiles
//                (thread = TMEM lane = row): p, ds, dS hi + lo back over the S buffer
// TMEM columns: S(b) = [64b, 64b+64), dP(b) = [128+64b, ...) for two buffers b,
// dQ = [256, 256+D), Q = [384, 384+D/2), dO = [448, 448+D/2) (bf16 pairs).  Q and dO
// in TMEM leave each S and dP MMA reading only its K or V slice from shared memory.
// At the start of an item warpgroup 0 copies the item's Q rows and warpgroup 1 its
// dO rows from the TMA-loaded shared tiles into TMEM.
//
// dS enters dQ as hi + lo so dq carries only the rounding of the bf16 inputs; the block
// reducer takes P and dS in fp32.  Every wait is bounded (ptx.cuh: mbar_wait); on a
// timeout the CTA raises the error word, drains what it issued, frees TMEM and returns.
#include <type_traits>

#include "attn_bwd.h"

#include "errbits.h"
#include "ptx.cuh"
#include "sched.cuh"

namespace tt {
namespace {

constexpr int kThreads = 384;
constexpr int kNK = 64;          // keys per tile
constexpr int kRowBytes = 128;   // one 64-element bf16 row of a swizzled half
constexpr int kStages = 8;       // ring slots (one K or one V tile each)
constexpr int kMaxBlk = 32;      // block keys handled by the reducer (S <= 32 on this path)
constexpr int kStageLd = kMaxBlk + 1;   // staged row stride (floats): rows fall in different banks

template <int D>
struct BwdCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kQBytes = 128 * kRowBytes * kHalves;        // one 128-row operand
  static constexpr int kSlotBytes = kNK * kRowBytes * kHalves;     // one K or V tile
  static constexpr int kQOff = 0, kOOff = kQBytes;
  static constexpr int kRingOff = 2 * kQBytes;
  static constexpr int kStageOff = kRingOff + kStages * kSlotBytes;   // P, dS of the block tile
  static constexpr int kStageBytes = 2 * 128 * kStageLd * 4;
  static constexpr int kBarOff = kStageOff + kStageBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct BwdBars {
  uint64_t q_full, q_empty, qo_full, qo_empty, dq_full, dq_empty, blk_full, blk_empty, drain;
  uint64_t sd_full[2], ds_full[2];
  uint64_t kv_full[kStages], kv_empty[kStages];
};

struct BwdShared {
  uint32_t tmem_base;
  int abort_flag;
};

// Geometry of one work item.
struct Item {
  int n, h, b, m;     // sequence, KV head, block, M-tile
  int tok0;           // first token of the block
  int rows;           // valid packed rows of the M-tile
  int tiles;          // key tiles: 1 (block keys) + ceil(S*b / 64) context tiles
};

__device__ __forceinline__ Item item_of(const BwdProblem& p, int idx, int MT) {
  Item it;
  const int per_b = p.B * p.Hkv * MT;
  const int bi = idx / per_b, rem = idx - bi * per_b;
  it.b = p.NB - 1 - bi;   // heaviest blocks first
  it.m = rem % MT;
  const int nh = rem / MT;
  it.n = nh / p.Hkv;
  it.h = nh - it.n * p.Hkv;
  it.tok0 = it.b * p.S;
  it.rows = min(128, p.R - 128 * it.m);
  it.tiles = 1 + ceil_div(p.S * it.b, kNK);
  return it;
}

// Keys of item-local tile i: the block's keys (i = 0) or context positions.
__device__ __forceinline__ void tile_range(const BwdProblem& p, const Item& it, int i, int& first, int& count) {
  if (i == 0) {
    first = 0;
    count = p.S;
  } else {
    first = (i - 1) * kNK;
    count = min(kNK, it.tok0 - first);
  }
}

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_tc_kernel(const BwdProblem p, const __grid_constant__ BwdMaps maps) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + C::kQOff, o_s = sbase + C::kOOff, kv_s = sbase + C::kRingOff;
  float* stage_p = reinterpret_cast<float*>(smem + C::kStageOff);   // [128][kStageLd]
  float* stage_ds = stage_p + 128 * kStageLd;
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::kBarOff);
  BwdShared* sh = reinterpret_cast<BwdShared*>(smem + C::kBarOff + sizeof(BwdBars));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int MT = p.R > 128 ? 2 : 1;
  const int n_items = p.B * p.Hkv * p.NB * MT;
  const int tpm = p.R > 128 ? 128 / p.g : p.S;   // tokens of one M-tile

  // rows that no TMA box covers (single M-tile units with R < 128) stay zero
  for (int i = tid; i < 2 * C::kQBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 64 + 256);   // the reducer and the two TMEM copies read it
    mbar_init(smem_u32(&bars->qo_full), 256);         // Q and dO rows written to TMEM
    mbar_init(smem_u32(&bars->qo_empty), 1);          // the item's last S and dP have read them
    mbar_init(smem_u32(&bars->dq_full), 1);
    mbar_init(smem_u32(&bars->dq_empty), 256);  // both softmax warpgroups read their half
    mbar_init(smem_u32(&bars->blk_full), 128);
    mbar_init(smem_u32(&bars->blk_empty), 64);
    mbar_init(smem_u32(&bars->drain), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->sd_full[b]), 1);
      mbar_init(smem_u32(&bars->ds_full[b]), 128);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    sh->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.dout);
    tma_prefetch_desc(&maps.k_ctx);
    tma_prefetch_desc(&maps.v_ctx);
    tma_prefetch_desc(&maps.k_blk);
    tma_prefetch_desc(&maps.v_blk);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const WaitCtx wc{&sh->abort_flag, p.err_word, p.wait_limit_ns};

  if (warp == 0) {
    // ============================================================ producer ==
    uint32_t it_kv = 0, q_it = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
      const Item x = item_of(p, idx, MT);
      ok = mbar_wait(smem_u32(&bars->q_empty), (q_it & 1) ^ 1, wc);
      if (!ok) break;
      if (lane == 0) {
        const uint32_t bar = smem_u32(&bars->q_full);
        // full boxes: g heads x tpm tokens of Q and of dO (rows past the M-tile's valid ones
        // belong to the next block or are zero fill; they are masked)
        mbar_arrive_expect_tx(bar, (uint32_t)(2 * p.g * tpm * kRowBytes * C::kHalves));
        const int tz = p.NB * p.S * x.n + x.tok0 + x.m * tpm;   // first token row of the M-tile
        for (int hf = 0; hf < C::kHalves; ++hf) {
          tma_load_3d(q_s + hf * (128 * kRowBytes), &maps.q, bar, hf * 64, x.h * p.g, tz);
          tma_load_3d(o_s + hf * (128 * kRowBytes), &maps.dout, bar, hf * 64, x.h * p.g, tz);
        }
      }
      ++q_it;
      const int ctx_row0 = (x.n * p.Hkv + x.h) * p.N;
      for (int i = 0; i < x.tiles && ok; ++i) {
        int first, count;
        tile_range(p, x, i, first, count);
        const int box_rows = i == 0 ? min(p.S, kNK) : kNK;
        const uint32_t bytes = (uint32_t)(box_rows * kRowBytes * C::kHalves);
        for (int kv = 0; kv < 2 && ok; ++kv, ++it_kv) {
          const int s = it_kv % kStages;
          ok = mbar_wait(smem_u32(&bars->kv_empty[s]), ((it_kv / kStages) & 1) ^ 1, wc);
          if (!ok) break;
          const uint32_t slot = kv_s + s * C::kSlotBytes;
          if (lane == 0) {
            const uint32_t bar = smem_u32(&bars->kv_full[s]);
            mbar_arrive_expect_tx(bar, bytes);
            for (int hf = 0; hf < C::kHalves; ++hf) {
              const uint32_t dst = slot + hf * (kNK * kRowBytes);
              if (i == 0) {
                tma_load_3d(dst, kv ? &maps.v_blk : &maps.k_blk, bar, hf * 64, x.h, p.NB * p.S * x.n + x.tok0);
              } else {
                tma_load_2d(dst, kv ? &maps.v_ctx : &maps.k_ctx, bar, hf * 64, ctx_row0 + first);
              }
            }
          }
          // K rows [count, round16(count)) feed the last dQ k-step: clear them once landed
          if (kv == 0 && (count & 15) != 0) {
            ok = mbar_wait(smem_u32(&bars->kv_full[s]), (it_kv / kStages) & 1, wc);
            if (!ok) break;
            const int r0 = count, r1 = round16(count);
            const int n16 = (r1 - r0) * 8 * C::kHalves;
            for (int e = lane; e < n16; e += 32) {
              const int hf = e / ((r1 - r0) * 8);
              const int rem = e - hf * (r1 - r0) * 8;
              const int row = r0 + rem / 8, ch = rem % 8;
              uint4* dst = reinterpret_cast<uint4*>(smem + C::kRingOff + s * C::kSlotBytes + hf * (kNK * kRowBytes) +
                                                    row * kRowBytes + ch * 16);
              *dst = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
        }
      }
    }
    if (!ok) {
      int dummy = 0;
      WaitCtx dw{&dummy, nullptr, 2000000ull};
      for (uint32_t j = (it_kv > (uint32_t)kStages ? it_kv - kStages : 0); j < it_kv; ++j)
        mbar_wait(smem_u32(&bars->kv_full[j % kStages]), (j / kStages) & 1, dw);
      if (q_it) mbar_wait(smem_u32(&bars->q_full), (q_it - 1) & 1, dw);
    }
  } else if (warp == 1) {
    // ============================================================= MMA warp ==
    // The whole warp runs the control flow (waits and descriptors stay warp-uniform); one
    // elected lane issues each burst of MMAs and its commits.
    uint32_t it_kv = 0, q_it = 0, G = 0, item_cnt = 0;
    bool ok = true;
    const uint32_t q_tmem = tmem + 384, o_tmem = tmem + 448;
    const uint64_t kdesc0 = smem_desc_sw128(kv_s, 16, 1024);              // K-major (S, dP)
    const uint64_t kmn0 = smem_desc_sw128(kv_s, kNK * kRowBytes, 1024);   // MN-major (dQ)
    const uint32_t idesc_sd0 = idesc_bf16_f32(128, 0, 0, 0);   // A (Q, dO) from TMEM, K-major B
    const uint32_t idesc_dq = idesc_bf16_f32(128, D, 0, 1);
    const uint32_t dq_tmem = tmem + 256;
    // S = Q K^T and dP = dO V^T of tile j into buffer b (K, V = ring entries ek, ek + 1), then
    // the commits: S and dP ready, V read
    auto issue_sd = [&](int b, uint32_t ek, int nk) {
      const uint32_t idesc = idesc_sd0 | ((uint32_t)(nk >> 3) << 17);
      const uint64_t kd = kdesc0 + (uint64_t)(((ek % kStages) * C::kSlotBytes) >> 4);
      const uint64_t vd = kdesc0 + (uint64_t)((((ek + 1) % kStages) * C::kSlotBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * (kNK * kRowBytes) + (kk & 3) * 32;
          tc_mma_ts(tmem + 64 * b, q_tmem + kk * 8, kd + (koff >> 4), idesc, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * (kNK * kRowBytes) + (kk & 3) * 32;
          tc_mma_ts(tmem + 128 + 64 * b, o_tmem + kk * 8, vd + (koff >> 4), idesc, kk > 0);
        }
        tc_commit(smem_u32(&bars->sd_full[b]));
        tc_commit(smem_u32(&bars->kv_empty[(ek + 1) % kStages]));   // V read by dP
      }
      __syncwarp();
    };
    auto kv_wait = [&](uint32_t e) {
      return mbar_wait_warp(smem_u32(&bars->kv_full[e % kStages]), (e / kStages) & 1, wc);
    };
    for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x, ++item_cnt) {
      const Item x = item_of(p, idx, MT);
      const int n = x.tiles;
      ok = mbar_wait_warp(smem_u32(&bars->qo_full), q_it & 1, wc);
      ++q_it;
      if (!ok) break;
      tc_fence_after();
      // prologue: S and dP of the first two tiles
      for (int j = 0; j < 2 && j < n && ok; ++j) {
        const uint32_t ek = it_kv + 2 * j;
        ok = kv_wait(ek) && kv_wait(ek + 1);
        if (!ok) break;
        tc_fence_after();
        int first, count;
        tile_range(p, x, j, first, count);
        issue_sd((G + j) & 1, ek, round16(count));
      }
      // the previous item's dQ must have been read out before this item overwrites it
      if (ok && item_cnt > 0) ok = mbar_wait_warp(smem_u32(&bars->dq_empty), (item_cnt - 1) & 1, wc);
      for (int j = 0; j < n && ok; ++j, ++G) {
        const int b = G & 1;
        ok = mbar_wait_warp(smem_u32(&bars->ds_full[b]), (G >> 1) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        int first, count;
        tile_range(p, x, j, first, count);
        const int ksteps = round16(count) / 16;
        const uint32_t ek = it_kv + 2 * j;
        const uint64_t kb = kmn0 + (uint64_t)(((ek % kStages) * C::kSlotBytes) >> 4);
        const uint32_t hi = tmem + 64 * b, lo = hi + 32;
        if (elect_one()) {
          if (ksteps == kNK / 16) {
#pragma unroll
            for (int kk = 0; kk < kNK / 16; ++kk) {
              const uint64_t bd = kb + (uint64_t)((kk * 16 * kRowBytes) >> 4);
              tc_mma_ts(dq_tmem, hi + kk * 8, bd, idesc_dq, (j > 0 || kk > 0) ? 1u : 0u);
              tc_mma_ts(dq_tmem, lo + kk * 8, bd, idesc_dq, 1u);
            }
          } else {
            for (int kk = 0; kk < ksteps; ++kk) {
              const uint64_t bd = kb + (uint64_t)((kk * 16 * kRowBytes) >> 4);
              tc_mma_ts(dq_tmem, hi + kk * 8, bd, idesc_dq, (j > 0 || kk > 0) ? 1u : 0u);
              tc_mma_ts(dq_tmem, lo + kk * 8, bd, idesc_dq, 1u);
            }
          }
          tc_commit(smem_u32(&bars->kv_empty[ek % kStages]));   // K read by S and dQ
        }
        __syncwarp();
        if (j + 2 < n) {
          // S and dP of tile j + 2 into buffer b, after dQ(j) has read dS(j) from it
          const uint32_t e2 = it_kv + 2 * (j + 2);
          ok = kv_wait(e2) && kv_wait(e2 + 1);
          if (!ok) break;
          tc_fence_after();
          int f2, c2;
          tile_range(p, x, j + 2, f2, c2);
          issue_sd(b, e2, round16(c2));
        }
      }
      if (!ok) break;
      it_kv += 2 * n;
      if (elect_one()) {
        tc_commit(smem_u32(&bars->dq_full));
        tc_commit(smem_u32(&bars->qo_empty));
      }
      __syncwarp();
    }
    if (elect_one()) tc_commit(smem_u32(&bars->drain));
    __syncwarp();
    int dummy = 0;
    WaitCtx dw{&dummy, nullptr, 2000000ull};
    mbar_wait(smem_u32(&bars->drain), 0, dw);
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    // ========================================================= block reducer ==
    // thread t of 64: dims t and t + 64 (D = 128) or dim t (D = 64), every block key
    const int t = tid - 64;
    uint32_t item_cnt = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x, ++item_cnt) {
      const Item x = item_of(p, idx, MT);
      ok = mbar_wait(smem_u32(&bars->blk_full), item_cnt & 1, wc);
      if (!ok) break;
      constexpr int ND = D / 64;
      float dk[ND][kMaxBlk > 16 ? 16 : kMaxBlk], dv[ND][16];
      const int nkey = p.S;   // block keys (<= 64 on this path), in chunks of 16
      for (int k0 = 0; k0 < nkey; k0 += 16) {
#pragma unroll
        for (int e = 0; e < ND; ++e)
#pragma unroll
          for (int k = 0; k < 16; ++k) dk[e][k] = dv[e][k] = 0.f;
        for (int r = 0; r < x.rows; ++r) {
          float qv[ND], ov[ND];
#pragma unroll
          for (int e = 0; e < ND; ++e) {
            // element (row r, dim d) of a 128-byte-swizzled K-major operand
            const int d = t + 64 * e;
            const int hf = d >> 6, c = (d & 63) >> 3;
            const uint32_t off = hf * (128 * kRowBytes) + r * kRowBytes + ((c ^ (r & 7)) << 4) + (d & 7) * 2;
            qv[e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(smem + C::kQOff + off));
            ov[e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(smem + C::kOOff + off));
          }
          const float* ps = stage_p + r * kStageLd + k0;    // same address in every thread
          const float* ds = stage_ds + r * kStageLd + k0;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float pv = ps[k], dsv = ds[k];
#pragma unroll
            for (int e = 0; e < ND; ++e) {
              dk[e][k] += dsv * qv[e];
              dv[e][k] += pv * ov[e];
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int key = k0 + k;
          if (key < nkey) {
            const size_t row = ((size_t)(x.n * p.N + x.tok0 + key) * p.Hkv + x.h) * D;
#pragma unroll
            for (int e = 0; e < ND; ++e) {
              atomicAdd(p.dk_blk + row + t + 64 * e, p.scale * dk[e][k]);
              atomicAdd(p.dv_blk + row + t + 64 * e, dv[e][k]);
            }
          }
        }
      }
      mbar_arrive(smem_u32(&bars->blk_empty));
      mbar_arrive(smem_u32(&bars->q_empty));
    }
  } else {
    // ========================================================= softmax WGs ==
    const int w = (warp - 4) >> 2;        // this warpgroup takes the CTA's tiles of parity w
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;       // row within the M-tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t dq_addr = tmem + lane_off + 256 + (D / 2) * w;
    uint32_t G = 0, item_cnt = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x, ++item_cnt) {
      const Item x = item_of(p, idx, MT);
      const bool valid = row < x.rows;
      const int r = 128 * x.m + row;                     // packed row of the unit
      const int tt = r / p.g, jj = r - (r / p.g) * p.g;  // block token, query head within the group
      float lse2 = 0.f, delta = 0.f;
      size_t qrow = 0;
      if (valid) {
        qrow = ((size_t)(x.n * p.N + x.tok0 + tt) * p.Hq + x.h * p.g + jj) * D;
        lse2 = p.lse[(size_t)(x.n * p.Hq + x.h * p.g + jj) * p.N + x.tok0 + tt] * 1.4426950408889634f;
        const float4* o4 = reinterpret_cast<const float4*>(p.out + qrow);
        const uint2* d4 = reinterpret_cast<const uint2*>(p.dout + qrow);
        float acc = 0.f;
#pragma unroll 4
        for (int c = 0; c < D / 4; ++c) {
          const float4 o = o4[c];
          const uint2 dd = d4[c];
          acc += o.x * __uint_as_float(dd.x << 16) + o.y * __uint_as_float(dd.x & 0xFFFF0000u) +
                 o.z * __uint_as_float(dd.y << 16) + o.w * __uint_as_float(dd.y & 0xFFFF0000u);
        }
        delta = acc;
      }
      const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
      const float2 nl2 = make_float2(-lse2, -lse2), nd2 = make_float2(-delta, -delta);
      // One tile: p = 2^(s c - lse2), ds = p (dp - Delta) for the 64 keys of this row, dS
      // back to TMEM as hi (columns [0, 32)) and lo ([32, 64)) over the consumed scores.
      // A full tile runs without masking; in a partial one, keys past `count` take 0 by
      // selection (their scores and dP come from rows that may hold anything).
      auto tile = [&](auto full_tag, uint32_t s_addr, uint32_t dp_addr, int count, bool blk) {
        constexpr bool kFull = decltype(full_tag)::value;
        uint32_t lo0[16];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t sv[32], dv[32];
          tmem_ld32(s_addr + 32 * ch, sv);
          tmem_ld32(dp_addr + 32 * ch, dv);
          tc_wait_ld();
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int c0 = 32 * ch + 2 * k;
            const float2 xs = __ffma2_rn(make_float2(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])), c2, nl2);
            float2 pp = make_float2(fast_exp2(xs.x), fast_exp2(xs.y));
            float2 dd = __fmul2_rn(pp, __fadd2_rn(make_float2(__uint_as_float(dv[2 * k]), __uint_as_float(dv[2 * k + 1])), nd2));
            if (!kFull) {
              const bool v0 = c0 < count, v1 = c0 + 1 < count;
              pp = make_float2(v0 ? pp.x : 0.f, v1 ? pp.y : 0.f);
              dd = make_float2(v0 ? dd.x : 0.f, v1 ? dd.y : 0.f);
            }
            hi[k] = pack_bf16(dd.x, dd.y);
            const float2 rem = __fadd2_rn(dd, make_float2(-__uint_as_float(hi[k] << 16), -__uint_as_float(hi[k] & 0xFFFF0000u)));
            lo[k] = pack_bf16(rem.x, rem.y);
            if (!kFull && blk && c0 < p.S) {
              stage_p[row * kStageLd + c0] = valid ? pp.x : 0.f;
              stage_ds[row * kStageLd + c0] = valid ? dd.x : 0.f;
              if (c0 + 1 < p.S) {
                stage_p[row * kStageLd + c0 + 1] = valid ? pp.y : 0.f;
                stage_ds[row * kStageLd + c0 + 1] = valid ? dd.y : 0.f;
              }
            }
          }
          // hi of keys [32ch, 32ch+32) -> columns [16ch, 16ch+16): scores already consumed
          tmem_st16(s_addr + 16 * ch, hi);
          if (ch == 0) {
#pragma unroll
            for (int k = 0; k < 16; ++k) lo0[k] = lo[k];
          } else {
            // lo -> columns [32, 64), over scores that are now all consumed
            tmem_st16(s_addr + 32, lo0);
            tmem_st16(s_addr + 48, lo);
          }
        }
      };
      // ---- this item's Q (warpgroup 0) or dO (warpgroup 1) rows into TMEM ----
      ok = mbar_wait(smem_u32(&bars->q_full), item_cnt & 1, wc);
      if (ok && item_cnt > 0) ok = mbar_wait(smem_u32(&bars->qo_empty), (item_cnt - 1) & 1, wc);
      if (!ok) break;
      tc_fence_after();
      {
        const uint8_t* src = smem + (w == 0 ? C::kQOff : C::kOOff);
        const uint32_t dst = tmem + lane_off + (w == 0 ? 384 : 448);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf) {
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            // chunk c (dims 8c..8c+7 of this half) of row `row` of a 128-byte-swizzled tile
            const uint4 u = *reinterpret_cast<const uint4*>(src + hf * (128 * kRowBytes) + row * kRowBytes +
                                                            ((c ^ (row & 7)) << 4));
            v[4 * c] = u.x;
            v[4 * c + 1] = u.y;
            v[4 * c + 2] = u.z;
            v[4 * c + 3] = u.w;
          }
          tmem_st32(dst + 32 * hf, v);
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->qo_full));
        mbar_arrive(smem_u32(&bars->q_empty));   // this warpgroup is done with the shared tile
      }
      // item tile j is the CTA's tile G + j, in TMEM buffer (G + j) % 2
      for (int j = (w ^ (int)(G & 1u)) & 1; j < x.tiles; j += 2) {
        const uint32_t Gj = G + (uint32_t)j;
        const int b = (int)(Gj & 1u);
        ok = mbar_wait(smem_u32(&bars->sd_full[b]), (Gj >> 1) & 1u, wc);
        if (!ok) break;
        tc_fence_after();
        int first, count;
        tile_range(p, x, j, first, count);
        const bool blk = j == 0;
        if (blk && item_cnt > 0) {
          // the reducer must be done with the previous item's staged block tile
          ok = mbar_wait(smem_u32(&bars->blk_empty), (item_cnt - 1) & 1, wc);
          if (!ok) break;
        }
        const uint32_t s_addr = tmem + lane_off + 64 * b, dp_addr = tmem + lane_off + 128 + 64 * b;
        // the block tile (<= 32 keys) always takes the masked path, which also stages P and dS
        if (count == kNK && !blk)
          tile(std::true_type{}, s_addr, dp_addr, count, false);
        else
          tile(std::false_type{}, s_addr, dp_addr, count, blk);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->ds_full[b]));
        if (blk) {
          __threadfence_block();
          mbar_arrive(smem_u32(&bars->blk_full));
        }
      }
      if (!ok) break;
      G += (uint32_t)x.tiles;
      // ---- dq rows: this warpgroup's half of the dQ columns ----
      ok = mbar_wait(smem_u32(&bars->dq_full), item_cnt & 1, wc);
      if (!ok) break;
      tc_fence_after();
      float* dst = p.dq + qrow + (D / 2) * w;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t o[32];
        tmem_ld32(dq_addr + 32 * cc, o);
        tc_wait_ld();
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(dst + 32 * cc)[q] =
                make_float4(p.scale * __uint_as_float(o[4 * q]), p.scale * __uint_as_float(o[4 * q + 1]),
                            p.scale * __uint_as_float(o[4 * q + 2]), p.scale * __uint_as_float(o[4 * q + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->dq_empty));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

bool attn_bwd_tc_supported(const BwdProblem& p) {
  if (p.D != 64 && p.D != 128) return false;
  if (p.S > kMaxBlk) return false;
  if (p.R > 128 && (128 % p.g != 0 || p.R > 256)) return false;
  return true;
}

size_t attn_bwd_tc_smem_bytes(int D) { return D == 128 ? BwdCfg<128>::kSmemBytes : BwdCfg<64>::kSmemBytes; }

cudaError_t launch_attn_bwd_tc(const BwdProblem& p, const BwdMaps& maps, int num_ctas, cudaStream_t stream) {
  static const bool attr_done = [] {
    cudaFuncSetAttribute(attn_bwd_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         BwdCfg<128>::kSmemBytes);
    cudaFuncSetAttribute(attn_bwd_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         BwdCfg<64>::kSmemBytes);
    return true;
  }();
  (void)attr_done;
  const int MT = p.R > 128 ? 2 : 1;
  const long long items = (long long)p.B * p.Hkv * p.NB * MT;
  const int grid = (int)(items < num_ctas ? items : num_ctas);
  if (grid <= 0) return cudaSuccess;
  if (p.D == 128)
    attn_bwd_tc_kernel<128><<<grid, kThreads, BwdCfg<128>::kSmemBytes, stream>>>(p, maps);
  else
    attn_bwd_tc_kernel<64><<<grid, kThreads, BwdCfg<64>::kSmemBytes, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace tt
