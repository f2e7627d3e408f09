// Block attention on a pair of SMs (tcgen05 cta_group::2, M = 256) for head_dim 128.
//
// The method (paperfeed.app review of arXiv 2606.26493, "Nemotron-Labs-
// TwoTower", section "The idea: freeze the reader, train the writer"): the S
// noisy block queries of denoiser layer i attend, in one softmax, to the
// frozen context tower's layer-i cache followed by the block's own keys.
//
// A cluster of two CTAs works on one range of key tiles (sched.cuh).  The up
// to 256 packed query rows of a unit are split by rows: the even CTA owns rows
// 0..127, the odd CTA rows 128..255.  Every MMA is a 2-SM instruction issued by
// the even CTA:
//   S = Q K^T   A = Q (each CTA its 128 rows), B = K tile split by keys
//               (each CTA holds half of the tile's keys, all 128 dims);
//   O += P V    A = P (each CTA its rows, shared memory), B = V tile split by
//               dims (each CTA holds 64 of the 128 dims, all keys).
// So each SM reads from HBM and from its shared memory only half of every K/V
// tile, and one instruction does the work of two 1-SM instructions.
//
// Each CTA runs two softmax warpgroups that take alternate key tiles; each
// has its own S buffer and O accumulator in TMEM (S_0 | S_1 | O_0 | O_1, 4 x 128
// columns), two P buffers in shared memory, its own running maximum and sum.
// The scores of tile j + 2 are computed as soon as tile j's scores have been
// read into registers, so a warpgroup finds its next S ready when it finishes
// a tile; with two P buffers it writes P(j) while P(j - 2) V may still run, and
// waits for that product only when O must be rescaled.  The two partial
// softmax states of a row are merged exactly in the epilogue.
//
// The MMA warp issues S(j+2) interleaved, instruction by instruction, with P(j-1) V
// (the other warpgroup's product), so that two independent accumulator chains are in
// flight (the ring order below follows).
//
// Synchronisation across the pair: the even CTA's MMA warp commits with
// multicast to barriers in both CTAs.  The odd CTA's TMA completions and softmax
// arrivals land on its own barriers and are forwarded to the even CTA's by
// otherwise idle warps (remote mbarrier arrive), so no softmax warp pays for a
// cluster-scope release.  No TMA multicast is used.  Every wait is bounded
// (ptx.cuh); on a timeout the CTA raises the error word and both CTAs still
// meet at the final cluster barrier before TMEM is released.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "problem.h"
#include "ptx.cuh"
#include "tc_common.cuh"
#include "walker.cuh"

namespace tt {
namespace {

constexpr int kThreads = 384;
constexpr int kD = 128;
constexpr int kNK = 128;                       // keys per tile
constexpr int kRowBytes = 128;                 // one 64-element bf16 half-row (swizzle atom width)
constexpr int kHalf = 128 * kRowBytes;         // 16 KB: 128 rows x 64 elements
constexpr int kQOff = 0;                       // Q: [2 d-halves][128 rows][128 B]      32 KB
constexpr int kPOff = 2 * kHalf;               // P[w][b]: [2 key-halves][128 rows][128 B]  4 x 32 KB
constexpr int kPBytes = 2 * kHalf;
constexpr int kRingOff = kPOff + 4 * kPBytes;  // K/V ring
constexpr int kEntryBytes = 16384;             // K: [2 d-halves][64 keys][128 B]; V: [128 keys][128 B]
constexpr int kStages = 4;
constexpr int kMiscOff = kRingOff + kStages * kEntryBytes;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kCtrlRegs = 80, kSoftmaxRegs = 200;
static_assert(4 * 32 * kCtrlRegs + 8 * 32 * kSoftmaxRegs <= kThreads * 168, "register split");

struct Bars {
  uint64_t q_full, q_ready, q_empty, tail, drain, epi, epi_done;
  uint64_t kv_full[kStages], kv_ready[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2][2];   // pv_done[warpgroup][P buffer]
  uint64_t o_full, o_empty;
  uint64_t o_done[2];   // odd CTA: its warpgroup w has read O (forwarded to the even CTA's o_empty)
};

struct Misc {
  Bars bars;
  uint32_t tmem_base;
  int abort_flag;
  long long T, start, end;
  Unit first;
  float ml[2][2][128];      // [warpgroup][m or l][row]: epilogue exchange
};

constexpr int kSmemBytes = kMiscOff + (int)sizeof(Misc);
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ uint64_t add16(uint64_t desc, uint32_t byte_off) { return desc + (uint64_t)(byte_off >> 4); }

// Ring entries of a segment with n tiles, in the order the MMA consumes them.  The MMA
// thread issues S(j+2) interleaved, instruction by instruction, with P(j-1) V (the other
// warpgroup's product), so that two independent accumulator chains are always in flight:
// K0, K1, K2, (K3 V0), (K4 V1), ..., (K(n-1) V(n-4)), V(n-3), V(n-2), V(n-1)
__device__ __forceinline__ void entry_to_tile(int e, int n, int& j, int& kv) {
  if (e < min(n, 3)) { j = e; kv = 0; }
  else if (n >= 3 && e <= 2 * n - 4) {
    if (e & 1) { j = (e + 3) >> 1; kv = 0; }
    else { j = (e - 4) >> 1; kv = 1; }
  } else { j = e - n; kv = 1; }
}
__device__ __forceinline__ uint32_t entry_k(int t) { return t <= 2 ? (uint32_t)t : (uint32_t)(2 * t - 3); }
__device__ __forceinline__ uint32_t entry_v(int i, int n) {
  return i <= n - 4 ? (uint32_t)(2 * i + 4) : (uint32_t)(n + i);
}

// P row of one warp lane to shared memory: weights exp2(s * c - m_ref) of the 128 keys,
// rounded to bf16, written as 16-byte chunks in the 128-byte swizzled K-major layout
// (keys 0..63 in the first 16 KB half, 64..127 in the second).  Returns the sum of the
// rounded weights, so that numerator and denominator see the same values.
template <bool kFull>
__device__ __forceinline__ float exp_to_smem(const uint32_t* v, int count, float c, float m_ref, uint8_t* prow,
                                             int lr) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m_ref, -m_ref);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < kNK / 8; ++q) {
    uint32_t h[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c0 = 8 * q + 2 * t;
      const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[c0]), __uint_as_float(v[c0 + 1])), c2, nm2);
      float a = fast_exp2(x.x), b = fast_exp2(x.y);
      if (!kFull) {
        a = c0 < count ? a : 0.f;
        b = c0 + 1 < count ? b : 0.f;
      }
      h[t] = pack_bf16(a, b);
      acc = __fadd2_rn(acc, make_float2(__uint_as_float(h[t] << 16), __uint_as_float(h[t] & 0xFFFF0000u)));
    }
    const int half = q >> 3, ch = q & 7;
    *reinterpret_cast<uint4*>(prow + half * kHalf + ((ch ^ (lr & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
  }
  return acc.x + acc.y;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_2sm_kernel(const Problem p, const __grid_constant__ TmaMaps maps) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Misc* ms = reinterpret_cast<Misc*>(smem + kMiscOff);
  Bars* bars = &ms->bars;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();     // 0: even CTA (issues the MMAs), 1: odd CTA
  const int c = blockIdx.x >> 1;               // range index = pair index
  const uint32_t sbase = smem_u32(smem);
  const bool aligned = (sbase & 1023u) == 0;   // the swizzled layouts need a 1024-byte aligned base
  const uint32_t q_s = sbase + kQOff, p_s = sbase + kPOff, ring_s = sbase + kRingOff;
  auto bar = [&](const uint64_t& b) { return smem_u32(&b); };
  // Softmax warps arrive on barriers of their own CTA only: a cluster-scope release
  // costs a softmax warp a thousand cycles or more, so the odd CTA's arrivals are
  // forwarded to the even CTA by otherwise idle warps (see the forwarders below).

  // ---------------------------------------------------------------- setup --
  if (tid == 0) {
    mbar_init(bar(bars->q_full), 1);
    mbar_init(bar(bars->q_ready), 2);   // even CTA: own TMA + forwarded odd-CTA TMA
    mbar_init(bar(bars->q_empty), 1);
    mbar_init(bar(bars->tail), 1);
    mbar_init(bar(bars->drain), 1);
    mbar_init(bar(bars->epi), 256);
    mbar_init(bar(bars->epi_done), 256);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(bars->kv_full[s]), 1);
      mbar_init(bar(bars->kv_ready[s]), 2);
      mbar_init(bar(bars->kv_empty[s]), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(bars->s_full[w]), 1);
      // even CTA: its 4 warps + one forwarded arrival for the odd CTA's 4; odd CTA: its 4 warps
      mbar_init(bar(bars->s_free[w]), rank == 0 ? 5 : 4);
      mbar_init(bar(bars->p_full[w]), rank == 0 ? 5 : 4);
      mbar_init(bar(bars->o_done[w]), 4);
      mbar_init(bar(bars->pv_done[w][0]), 1);
      mbar_init(bar(bars->pv_done[w][1]), 1);
    }
    mbar_init(bar(bars->o_full), 1);
    mbar_init(bar(bars->o_empty), 10);      // even CTA: 8 softmax warps + 2 forwarded (odd warpgroups)
    ms->abort_flag = aligned ? 0 : 1;
    if (!aligned) raise_error(p.err_word, kErrInternal);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k_ctx);
    tma_prefetch_desc(&maps.v_ctx);
    tma_prefetch_desc(&maps.k_blk);
    tma_prefetch_desc(&maps.v_blk);
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish2();
  }
  if (warp == 2) {
    long long T = 0, start = 0, end = 0;
    Unit first;
    find_range(p, c, T, start, end, first);
    if (lane == 0) {
      ms->T = T;
      ms->start = start;
      ms->end = end;
      if (start < end) ms->first = first;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();

  const uint32_t tmem = ms->tmem_base;
  const long long T = ms->T, start = ms->start, end = ms->end;
  const WaitCtx wc{&ms->abort_flag, p.err_word, p.wait_limit_ns};
  const bool have_work = start < end && aligned;
  if (have_work && warp < 4) regs_dec<kCtrlRegs>();

  if (warp == 0 && have_work) {
    // ============================================================ producer ==
    uint32_t it = 0, q_it = 0, tail_ph = 0;
    bool ok = true;
    Unit x = ms->first;
    const int rows_tok = 128 / p.g;  // tokens of this CTA's 128 rows
    for (; ok;) {
      const Segment sg = segment_of(x, start, end, c);
      const int n = sg.hi - sg.lo;
      const int ctx_row0 = (x.n * p.Hkv + x.h) * p.ctx_stride;
      ok = mbar_wait(bar(bars->q_empty), (q_it & 1) ^ 1, wc);
      if (!ok) break;
      if (lane == 0) {
        const uint32_t qb = rank == 0 ? bar(bars->q_ready) : bar(bars->q_full);
        mbar_arrive_expect_tx(qb, (uint32_t)(2 * kHalf));
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(q_s + hf * kHalf, &maps.q, qb, hf * 64, x.h * p.g, x.ns * p.S + (int)rank * rows_tok);
      }
      ++q_it;
      for (int e = 0; e < 2 * n && ok; ++e, ++it) {
        int j, kv;
        entry_to_tile(e, n, j, kv);
        const TileKeys tk = tile_keys(p, x, sg.lo + j);
        const int nk = round16(tk.count);
        const int s = it % kStages;
        ok = mbar_wait(bar(bars->kv_empty[s]), ((it / kStages) & 1) ^ 1, wc);
        if (!ok) break;
        const uint32_t slot = ring_s + s * kEntryBytes;
        const bool fix = kv == 1 && (tk.count & 15) != 0;  // V rows [count, nk) are read by the last k-step
        const uint32_t fb = rank == 0 ? bar(bars->kv_ready[s]) : bar(bars->kv_full[s]);
        const uint32_t b = fix ? bar(bars->tail) : fb;
        if (lane == 0) {
          if (kv == 0) {
            // this CTA's half of the keys: [first + rank*nk/2, + nk/2), all 128 dims
            const int k0 = tk.first + (int)rank * (nk >> 1);
            mbar_arrive_expect_tx(b, (uint32_t)(2 * 64 * kRowBytes));
            for (int hf = 0; hf < 2; ++hf) {
              if (tk.is_blk) tma_load_3d(slot + hf * 64 * kRowBytes, &maps.k_blk, b, hf * 64, x.h, x.ns * p.S + k0);
              else tma_load_2d(slot + hf * 64 * kRowBytes, &maps.k_ctx, b, hf * 64, ctx_row0 + k0);
            }
          } else {
            // this CTA's 64 dims of V for all keys of the tile
            const int rows = tk.is_blk ? min(p.S, kNK) : kNK;
            mbar_arrive_expect_tx(b, (uint32_t)(rows * kRowBytes));
            if (tk.is_blk) tma_load_3d(slot, &maps.v_blk, b, (int)rank * 64, x.h, x.ns * p.S + tk.first);
            else tma_load_2d(slot, &maps.v_ctx, b, (int)rank * 64, ctx_row0 + tk.first);
          }
        }
        if (fix) {
          ok = mbar_wait(bar(bars->tail), tail_ph, wc);
          tail_ph ^= 1;
          if (!ok) break;
          for (int q = lane; q < (nk - tk.count) * 8; q += 32) {
            const int row = tk.count + q / 8, ch = q % 8;
            *reinterpret_cast<uint4*>(smem + kRingOff + s * kEntryBytes + row * kRowBytes + ch * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(fb);
        }
      }
      if (!ok || sg.last) break;
      x = make_unit(p, x.u + 1, x.Tu + x.tiles);
    }
    if (!ok) {
      int dummy = 0;
      WaitCtx dw{&dummy, nullptr, 2000000ull};
      for (uint32_t j = (it > (uint32_t)kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait(rank == 0 ? bar(bars->kv_ready[j % kStages]) : bar(bars->kv_full[j % kStages]),
                  (j / kStages) & 1, dw);
    }
  } else if (warp >= 1 && warp <= 3 && rank == 1 && have_work) {
    // ===================================== odd CTA: forward completions to the even CTA ==
    // warp 2: the TMA completions of Q and of every K/V ring entry, in the order the
    // producer issued them; warp 1 (warp 3): the arrivals of softmax warpgroup 0 (1),
    // tile by tile (S read, P written) and O read at the end of each segment.
    if (lane == 0) {
      uint32_t it = 0, q_it = 0, G = 0, seg_cnt = 0;
      const int w = warp == 1 ? 0 : 1;
      bool ok = true;
      Unit x = ms->first;
      for (; ok;) {
        const Segment sg = segment_of(x, start, end, c);
        const int n = sg.hi - sg.lo;
        if (warp == 2) {
          ok = mbar_wait(bar(bars->q_full), q_it & 1, wc);
          if (ok) mbar_arrive_remote(mapa_shared(bar(bars->q_ready), 0));
          ++q_it;
          for (int e = 0; e < 2 * n && ok; ++e, ++it) {
            ok = mbar_wait(bar(bars->kv_full[it % kStages]), (it / kStages) & 1, wc);
            if (ok) mbar_arrive_remote(mapa_shared(bar(bars->kv_ready[it % kStages]), 0));
          }
        } else {
          for (int j = 0; j < n && ok; ++j) {
            const uint32_t g = G + j;
            if ((int)(g & 1) != w) continue;
            ok = mbar_wait(bar(bars->s_free[w]), (g >> 1) & 1, wc);
            if (ok) mbar_arrive_remote(mapa_shared(bar(bars->s_free[w]), 0));
            if (ok) ok = mbar_wait(bar(bars->p_full[w]), (g >> 1) & 1, wc);
            if (ok) mbar_arrive_remote(mapa_shared(bar(bars->p_full[w]), 0));
          }
          if (ok) ok = mbar_wait(bar(bars->o_done[w]), seg_cnt & 1, wc);
          if (ok) mbar_arrive_remote(mapa_shared(bar(bars->o_empty), 0));
          G += n;
          ++seg_cnt;
        }
        if (!ok || sg.last) break;
        x = make_unit(p, x.u + 1, x.Tu + x.tiles);
      }
    }
    __syncwarp();
  } else if (warp == 1 && rank == 0 && have_work) {
    // ============================================= even CTA: 2-SM MMA issue ==
    // The whole warp runs the control flow (waits and descriptors stay warp-uniform); one
    // elected lane issues each burst of MMAs and its commits.
    {
      uint32_t it = 0, q_it = 0, G = 0, seg_cnt = 0;
      bool ok = true;
      Unit x = ms->first;
      const uint64_t qdesc = smem_desc_sw128(q_s, 16, 1024);                 // A of S: K-major
      const uint64_t kdesc = smem_desc_sw128(ring_s, 16, 1024);              // B of S: K-major (keys)
      const uint64_t pdesc = smem_desc_sw128(p_s, 16, 1024);                 // A of PV: K-major (keys)
      const uint64_t vdesc = smem_desc_sw128(ring_s, kEntryBytes, 1024);     // B of PV: MN-major (dims)
      const uint32_t idesc_s0 = idesc_bf16_f32(256, 0, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(256, kD, 0, 1);
      auto ring_wait = [&](uint32_t e) {
        return mbar_wait_cluster_warp(bar(bars->kv_ready[e % kStages]), (e / kStages) & 1, wc);
      };
      // the S buffer of tile g was last used by tile g - 2: its softmax must have read it
      auto s_buffer_free = [&](uint32_t g) {
        if (g < 2) return true;
        return mbar_wait_cluster_warp(bar(bars->s_free[g & 1]), ((g >> 1) & 1) ^ 1, wc);
      };
      for (; ok;) {
        const Segment sg = segment_of(x, start, end, c);
        const int n = sg.hi - sg.lo;
        ok = mbar_wait_cluster_warp(bar(bars->q_ready), q_it & 1, wc);
        ++q_it;
        if (!ok) break;
        // One step: S of tile t (when t < n) and P V of tile i (when 0 <= i), issued
        // interleaved.  Q is released after the segment's last S.
        auto step = [&](int t, int i) -> bool {
          const bool has_s = t < n, has_pv = i >= 0;
          if (!has_s && !has_pv) return true;
          const uint32_t gs = G + t, gp = G + i;
          uint32_t ek = 0, ev = 0;
          // P(i) first: the warpgroup of tile i arrives on p_full once per tile, so this wait
          // must not fall two of its arrivals behind (a parity wait cannot tell them apart);
          // its next P needs S(i + 2), which the previous step issued just before this one
          if (has_pv) {
            if (!mbar_wait_cluster_warp(bar(bars->p_full[gp & 1]), (gp >> 1) & 1, wc)) return false;
            ev = it + entry_v(i, n);
            if (!ring_wait(ev)) return false;
            if (i == 0 && !mbar_wait_cluster_warp(bar(bars->o_empty), (seg_cnt & 1) ^ 1, wc)) return false;
          }
          if (has_s) {
            if (!s_buffer_free(gs)) return false;
            ek = it + entry_k(t);
            if (!ring_wait(ek)) return false;
          }
          tc_fence_after();
          const int nk = has_s ? round16(tile_keys(p, x, sg.lo + t).count) : 0;
          const int npv = has_pv ? round16(tile_keys(p, x, sg.lo + i).count) / 16 : 0;
          const uint32_t idesc_s = idesc_s0 | ((uint32_t)(nk >> 3) << 17);
          const uint64_t kd = add16(kdesc, (ek % kStages) * kEntryBytes);
          const uint64_t pd = add16(pdesc, ((gp & 1) * 2 + ((gp >> 1) & 1)) * kPBytes);   // P[warpgroup][buffer]
          const uint64_t vd = add16(vdesc, (ev % kStages) * kEntryBytes);
          const uint32_t s_acc = tmem + 128 * (gs & 1), o_acc = tmem + 256 + 128 * (gp & 1);
          const uint32_t pv_acc0 = i >= 2 ? 1u : 0u;   // O_w starts at this warpgroup's first tile
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              if (has_s)
                tc_mma2_ss(s_acc, add16(qdesc, (kk >> 2) * kHalf + (kk & 3) * 32),
                           add16(kd, (kk >> 2) * (64 * kRowBytes) + (kk & 3) * 32), idesc_s, kk > 0);
              if (kk < npv)
                tc_mma2_ss(o_acc, add16(pd, (kk >> 2) * kHalf + (kk & 3) * 32), add16(vd, kk * 16 * kRowBytes),
                           idesc_pv, kk > 0 ? 1u : pv_acc0);
            }
            if (has_s) {
              tc_commit2_both(bar(bars->s_full[gs & 1]));
              tc_commit2_both(bar(bars->kv_empty[ek % kStages]));
              if (t == n - 1) tc_commit2_both(bar(bars->q_empty));
            }
            if (has_pv) {
              tc_commit2_both(bar(bars->pv_done[gp & 1][(gp >> 1) & 1]));
              tc_commit2_both(bar(bars->kv_empty[ev % kStages]));
            }
          }
          __syncwarp();
          return true;
        };
        ok = step(0, -1);
        if (ok && n > 1) ok = step(1, -1);
        for (int j = 0; j < n && ok; ++j) ok = step(j + 2, j - 1);
        if (ok) ok = step(n, n - 1);
        if (!ok) break;
        if (elect_one()) tc_commit2_both(bar(bars->o_full));
        __syncwarp();
        it += 2 * n;
        G += n;
        ++seg_cnt;
        if (sg.last) break;
        x = make_unit(p, x.u + 1, x.Tu + x.tiles);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && have_work) {
    // ========================================================= softmax WGs ==
    regs_inc<kSoftmaxRegs>();
    const int w = (warp - 4) >> 2;               // warpgroup: takes tiles with G % 2 == w
    const int q4 = warp & 3;                     // TMEM lane quarter
    const int lr = q4 * 32 + lane;               // row within this CTA
    const int r = (int)rank * 128 + lr;          // packed row of the unit
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + 128 * w;
    const uint32_t o_base = tmem + lane_off + 256;   // O_0 at +0, O_1 at +128
    uint8_t* prow0 = smem + kPOff + 2 * w * kPBytes + lr * kRowBytes;   // P[w][0]; P[w][1] follows
    uint32_t G = 0, seg_cnt = 0;
    bool ok = true;
    Unit x = ms->first;
    for (; ok;) {
      const Segment sg = segment_of(x, start, end, c);
      const int n = sg.hi - sg.lo;
      float m_w = -INFINITY, l_w = 0.f;
      bool first = true;
      for (int j = 0; j < n; ++j) {
        const uint32_t g = G + j;
        if ((int)(g & 1) != w) continue;
        const int count = tile_keys(p, x, sg.lo + j).count;
        const bool full = count == kNK;
        ok = mbar_wait(bar(bars->s_full[w]), (g >> 1) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        uint32_t v[kNK];
#pragma unroll
        for (int ch = 0; ch < kNK / 32; ++ch)
          if (full || 32 * ch < count) tmem_ld32(s_addr + 32 * ch, v + 32 * ch);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->s_free[w]));   // S may be overwritten by tile g + 2
        const float mx = (full ? tile_row_max<kNK, true>(v, count) : tile_row_max<kNK, false>(v, count)) * p.scale_log2;
        const uint32_t b = (g >> 1) & 1;   // P buffer of this tile; tile g - 2 used the other one
        if (first) {
          m_w = mx;  // O_w is overwritten by this warpgroup's first PV of the segment
        } else {
          const bool need = mx > m_w + kRescaleThreshold;
          if (__any_sync(0xffffffffu, need)) {
            // O_w must hold P(g-2) V before it is rescaled
            ok = mbar_wait(bar(bars->pv_done[w][b ^ 1]), ((g - 2) >> 2) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const float alpha = need ? fast_exp2(m_w - mx) : 1.f;
            if (need) {
              m_w = mx;
              l_w *= alpha;
            }
#pragma unroll 1
            for (int cc = 0; cc < kD / 16; ++cc) {
              uint32_t o[16];
              tmem_ld16(o_base + 128 * w + cc * 16, o);
              tc_wait_ld();
#pragma unroll
              for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st16(o_base + 128 * w + cc * 16, o);
            }
            tc_wait_st();
          }
        }
        // P buffer b was last read by the PV of tile g - 4
        if (g >= 4) {
          ok = mbar_wait(bar(bars->pv_done[w][b]), ((g >> 2) & 1) ^ 1, wc);
          if (!ok) break;
          tc_fence_after();
        }
        uint8_t* prow = prow0 + b * kPBytes;
        l_w += full ? exp_to_smem<true>(v, count, p.scale_log2, m_w, prow, lr)
                    : exp_to_smem<false>(v, count, p.scale_log2, m_w, prow, lr);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->p_full[w]));
        first = false;
      }
      if (!ok) break;
      // ---- epilogue: merge the two warpgroups' states, write rows (or partials) ----
      ok = mbar_wait(bar(bars->o_full), seg_cnt & 1, wc);
      if (!ok) break;
      tc_fence_after();
      const int par = seg_cnt & 1;
      // the previous segment's exchange must have been read by every thread of the CTA
      if (seg_cnt > 0) {
        ok = mbar_wait(bar(bars->epi_done), par ^ 1, wc);
        if (!ok) break;
      }
      ms->ml[w][0][lr] = first ? -INFINITY : m_w;
      ms->ml[w][1][lr] = first ? 0.f : l_w;
      mbar_arrive(bar(bars->epi));
      ok = mbar_wait(bar(bars->epi), par, wc);
      if (!ok) break;
      const float mA = ms->ml[0][0][lr], lA = ms->ml[0][1][lr];
      const float mB = ms->ml[1][0][lr], lB = ms->ml[1][1][lr];
      mbar_arrive(bar(bars->epi_done));
      const bool hasA = n >= 1 && ((G & 1) == 0 || n >= 2);   // warpgroup 0 had a tile
      const bool hasB = n >= 1 && ((G & 1) == 1 || n >= 2);   // warpgroup 1 had a tile
      const float m = fmaxf(hasA ? mA : -INFINITY, hasB ? mB : -INFINITY);
      const float fA = hasA ? fast_exp2(mA - m) : 0.f, fB = hasB ? fast_exp2(mB - m) : 0.f;
      const float L = fA * lA + fB * lB;
      const float inv = 1.f / L;
      // warpgroup w writes dims [64w, 64w + 64) of its rows
      const float wA = hasA ? fA * inv : 0.f, wB = hasB ? fB * inv : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        const int col = 64 * w + 16 * cc;
        uint32_t oa[16], ob[16];
        tmem_ld16(o_base + col, oa);
        tmem_ld16(o_base + 128 + col, ob);
        tc_wait_ld();
        if (cc == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(rank == 0 ? bar(bars->o_empty) : bar(bars->o_done[w]));  // O read
        }
        if (r < p.R) {
          float* dst = out_row(p, x, sg, r, kD) + col;
#pragma unroll
          for (int k = 0; k < 16; k += 4) {
            float4 f;
            // an accumulator that received no PV holds stale values: select, never scale by 0
            f.x = (hasA ? wA * __uint_as_float(oa[k]) : 0.f) + (hasB ? wB * __uint_as_float(ob[k]) : 0.f);
            f.y = (hasA ? wA * __uint_as_float(oa[k + 1]) : 0.f) + (hasB ? wB * __uint_as_float(ob[k + 1]) : 0.f);
            f.z = (hasA ? wA * __uint_as_float(oa[k + 2]) : 0.f) + (hasB ? wB * __uint_as_float(ob[k + 2]) : 0.f);
            f.w = (hasA ? wA * __uint_as_float(oa[k + 3]) : 0.f) + (hasB ? wB * __uint_as_float(ob[k + 3]) : 0.f);
            *reinterpret_cast<float4*>(dst + k) = f;
          }
        }
      }
      if (w == 0 && r < p.R) {
        const float lse = (m + __log2f(L)) * 0.6931471805599453f;
        if (sg.full) {
          if (p.lse) {
            const int t = r / p.g, jj = r - (r / p.g) * p.g;
            p.lse[(size_t)(x.n * p.Hq + x.h * p.g + jj) * (p.NB * p.S) + x.b * p.S + t] = lse;
          }
        } else {
          p.part_lse[(size_t)sg.slot * p.R + r] = lse;
        }
      }
      G += n;
      ++seg_cnt;
      if (sg.last) break;
      x = make_unit(p, x.u + 1, x.Tu + x.tiles);
    }
  }

  // record for the combine: the cut unit (if any) that begins in this range
  if (tid == 64 && rank == 0) {
    SplitRecord rec{-1, -1, 0, 0};
    if (have_work) {
      Unit x = ms->first;
      while (x.Tu + x.tiles < end) x = make_unit(p, x.u + 1, x.Tu + x.tiles);
      rec = record_of(x, T, p.C, start, end, range_table(p));
    }
    p.records[c] = rec;
  }

  // drain every 2-SM MMA before either CTA releases TMEM
  if (warp == 1) {
    // the lane that issued the MMAs commits (elect_one picks the same lane of a converged warp)
    if (rank == 0 && elect_one()) tc_commit2_both(bar(bars->drain));
    __syncwarp();
    int dummy = 0;
    WaitCtx dw{&dummy, nullptr, 2000000ull};
    mbar_wait(bar(bars->drain), 0, dw);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc2(tmem, 512);
}

// ---------------------------------------------------------------- host ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  if (!fn) return false;
  cuuint32_t elem[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_2sm_supported(int D, int g) { return D == kD && g >= 1 && 128 % g == 0; }

int attn_2sm_max_clusters() {
  static int cached = -1;
  if (cached >= 0) return cached;
  cudaFuncSetAttribute(attn_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (void*)attn_2sm_kernel, &cfg) != cudaSuccess) n = 0;
  cached = n;
  return n;
}

cudaError_t launch_attn_2sm(const Problem& p, cudaStream_t stream) {
  static const bool attr_done = [] {
    cudaFuncSetAttribute(attn_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    return true;
  }();
  (void)attr_done;
  if (!attn_2sm_supported(p.D, p.g) || p.key_tile != kNK) return cudaErrorInvalidValue;
  TmaMaps maps;
  memset(&maps, 0, sizeof(maps));
  const cuuint64_t D = kD;
  {
    // q as [tokens][Hq][D]; box = the 128 rows of one CTA: 128/g tokens x g heads x 64 dims
    cuuint64_t dims[3] = {D, (cuuint64_t)p.Hq, (cuuint64_t)p.B * p.NB * p.S};
    cuuint64_t str[2] = {D * 2, (cuuint64_t)p.Hq * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)p.g, (cuuint32_t)(128 / p.g)};
    if (!encode(&maps.q, p.q, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    // block keys: 64 tokens of one head (a CTA's half of a 128-key tile at most);
    // block values: all block tokens of the tile, 64 dims
    cuuint64_t dims[3] = {D, (cuuint64_t)p.Hkv, (cuuint64_t)p.B * p.NB * p.S};
    cuuint64_t str[2] = {D * 2, (cuuint64_t)p.Hkv * D * 2};
    cuuint32_t kbox[3] = {64, 1, 64};
    cuuint32_t vbox[3] = {64, 1, (cuuint32_t)std::min(p.S, kNK)};
    if (!encode(&maps.k_blk, p.k_blk, 3, dims, str, kbox) || !encode(&maps.v_blk, p.v_blk, 3, dims, str, vbox))
      return cudaErrorInvalidValue;
  }
  if ((long long)p.B * p.Hkv * p.ctx_stride > 0) {
    cuuint64_t dims[2] = {D, (cuuint64_t)p.B * p.Hkv * p.ctx_stride};
    cuuint64_t str[1] = {D * 2};
    cuuint32_t kbox[2] = {64, 64};
    cuuint32_t vbox[2] = {64, (cuuint32_t)kNK};
    if (!encode(&maps.k_ctx, p.k_ctx, 2, dims, str, kbox) || !encode(&maps.v_ctx, p.v_ctx, 2, dims, str, vbox))
      return cudaErrorInvalidValue;
  } else {
    maps.k_ctx = maps.k_blk;  // never read: no context tiles exist
    maps.v_ctx = maps.v_blk;
  }
  attn_2sm_kernel<<<2 * p.C, kThreads, kSmemBytes, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace tt
