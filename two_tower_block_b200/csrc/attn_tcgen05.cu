// Block attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The method (paperfeed.app review of arXiv 2606.26493, "Nemotron-Labs-
// TwoTower", section "The idea: freeze the reader, train the writer"): the S
// noisy block queries of denoiser layer i attend, in one softmax, to the
// frozen context tower's layer-i cache followed by the block's own keys.
//
// One persistent CTA per SM walks its range of key tiles (sched.cuh).  The
// S*g query rows of a unit (all g query heads that share a KV head, for all S
// block tokens) are packed into one or two 128-row tensor-core tiles, so each
// key tile is read from HBM once and feeds up to 256 query rows.
//
// Roles (384 threads):
//   warp 0       TMA producer of Q (each segment) and of the K tiles, into the K half
//                of a ring of shared-memory slots (128-byte swizzle)
//   warp 3       TMA producer of the V tiles, into the V half of the ring; for a
//                tile whose valid rows are not a multiple of 16 it zeroes the V rows
//                the last MMA k-step would otherwise read
//   warp 1       TMEM owner; issues the MMAs of M-tile 0 (one elected lane): S =
//                Q_0 K^T into TMEM, O_0 += P V with P read from TMEM (aliasing its S
//                buffer)
//   warp 2       issues the MMAs of M-tile 1 (when the unit has two)
//   warps 4..7   softmax warpgroup of M-tile 0 (thread = TMEM lane = row)
//   warps 8..11  softmax warpgroup of M-tile 1
// TMEM columns: M-tile m owns S buffers [128m, 128m+128) (NBUF buffers of NK
// keys), O_0 = [256, 256+D), O_1 = [256+D, 256+2D).
//
// Pipeline per M-tile (tile G of the CTA uses S buffer G % NBUF): the MMA
// thread issues PV(j) as soon as P(j) is ready and then S(j+NBUF) into the
// buffer PV(j) has just consumed; with two buffers the softmax of tile j+1
// finds its S ready while the tensor core works on PV(j).
//
// The softmax keeps a running reference maximum per row and rescales O (in
// TMEM) only when a new maximum exceeds it by more than 2^8; the final
// normalisation divides by the sum of the same bf16-rounded weights the PV
// product used, so the result is exact up to rounding.
//
// Every wait is bounded (ptx.cuh: mbar_wait); on a timeout the CTA raises the
// error word, drains what it issued, frees TMEM and returns.
#include <type_traits>

#include "combine_row.cuh"
#include "problem.h"
#include "ptx.cuh"
#include "tc_common.cuh"
#include "walker.cuh"

namespace tt {
namespace {

constexpr int kThreads = 384;
constexpr int kMaxRows = 256;
constexpr int kRowBytes = 128;              // one 64-element bf16 row of a swizzled half
constexpr float kRescaleThreshold = 8.0f;   // log2 units

template <int D, int NK>
struct Cfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kBufs = 128 / NK;                       // S buffers per M-tile
  static constexpr int kSlotBytes = NK * kRowBytes * kHalves;  // one K or V tile
  static constexpr int kStages = (128 * 1024) / kSlotBytes;    // 128 KB ring
  static constexpr int kQBytes = kMaxRows * kRowBytes * kHalves;
  static constexpr int kStageOff = kQBytes;
  static constexpr int kEpiOff = kStageOff + kStages * kSlotBytes;
  static constexpr int kEpiBytes = 8 * 32 * 32 * 4;  // 8 softmax warps x 32 rows x 32 fp32
  static constexpr int kBarOff = kEpiOff + kEpiBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;  // barriers/flags + alignment slack
  // Register split (launch: 168 per thread = 65536 / 384 rounded down to 8): the
  // 128-key variant keeps a full 128-score row per softmax thread.
  static constexpr bool kSplitRegs = NK == 128;
  static constexpr int kCtrlRegs = 80, kSoftmaxRegs = 200;
  static_assert(4 * 32 * kCtrlRegs + 8 * 32 * kSoftmaxRegs <= kThreads * 168, "register split");
  static_assert(kStages <= 16, "ring too deep");
};

struct Bars {
  uint64_t q_full, q_empty, tail, drain;
  uint64_t s_full[2][2], p_full[2][2];  // [M-tile][S buffer]
  uint64_t pv_done[2], o_full[2], o_empty[2];
  uint64_t kv_full[16], kv_empty[16];
};

struct Shared {
  uint32_t tmem_base;
  int abort_flag;
  long long T, start, end;
  Unit first;
};
static_assert(sizeof(Bars) + sizeof(Shared) <= 512, "barrier block overflows its shared-memory slot");

// Fused split combine (cooperative launch only: every CTA is resident).  Once its segments and
// partials are written, each CTA adds one to its range's arrival count; every range does so
// exactly once per launch, so all counts of a launch are equal.  For each cut unit with a
// segment in this range (at most two: the unit holding the range's first tile and the one
// holding its last), the CTA waits until every range of that unit has reached its own count,
// then combines its share of the unit's rows: rows [i R / n, (i + 1) R / n) for the i-th of the
// unit's n ranges, one warp per row.  No CTA waits for ranges outside its units.  The waits
// are bounded; a CTA that gave up (or whose pipeline aborted) combines nothing and the error
// word says so.
template <int D>
__device__ __forceinline__ void fused_combine(const Problem& p, long long T, long long start, long long end,
                                              const Unit& first, bool aborted) {
  __shared__ unsigned s_k;
  __shared__ int s_ok;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  __syncthreads();  // every write of this CTA precedes its arrival
  if (tid == 0) {
    __threadfence();
    s_k = atomicAdd(p.arrivals + c, 1u) + 1u;
  }
  __syncthreads();
  if (start >= end || aborted) return;
  const unsigned k = s_k;
  const int Ce = used_ranges(T, p.C);
  Unit last = first;
  while (last.Tu + last.tiles < end) last = make_unit(p, last.u + 1, last.Tu + last.tiles);
  for (int which = 0; which < 2; ++which) {
    const Unit x = which == 0 ? first : last;
    if (which == 1 && last.u == first.u) break;
    if (x.Tu >= start && x.Tu + x.tiles <= end) continue;  // whole in this range: not cut
    const long long* tab = range_table(p);
    const int c0 = range_of_tile_tab(tab, T, Ce, x.Tu), c1 = range_of_tile_tab(tab, T, Ce, x.Tu + x.tiles - 1);
    if (warp == 0) {
      bool ok = true;
      const unsigned long long t0 = globaltimer_ns();
      for (int cc = c0 + lane; cc <= c1 && ok; cc += 32) {
        while (ld_acquire_gpu_u32(p.arrivals + cc) < k) {
          if (globaltimer_ns() - t0 > p.wait_limit_ns) {
            raise_error(p.err_word, kErrTimeout);
            ok = false;
            break;
          }
          __nanosleep(32);
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) s_ok = ok;
    }
    __syncthreads();
    if (!s_ok) return;
    const int n = c1 - c0 + 1, i = c - c0;
    const SplitRecord rec{x.u, c1, x.Tu == range_start_tab(tab, T, Ce, c0) ? 0 : 1, 0};
    const int r0 = (int)((long long)i * p.R / n), r1 = (int)((long long)(i + 1) * p.R / n);
    for (int r = r0 + warp; r < r1; r += kThreads / 32) combine_row<D, 16>(p, c0, rec, r, lane);
  }
}

template <int D, int NK>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tcgen05_kernel(const Problem p, const __grid_constant__ TmaMaps maps) {
  using C = Cfg<D, NK>;
  constexpr int NBUF = C::kBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase;
  const uint32_t kv_s = sbase + C::kStageOff;
  float* epi = reinterpret_cast<float*>(smem + C::kEpiOff);
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kBarOff);
  Shared* sh = reinterpret_cast<Shared*>(smem + C::kBarOff + sizeof(Bars));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int MT = p.R > 128 ? 2 : 1;
  // a dependent combine launch may be scheduled now; it waits for this grid on the device
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---------------------------------------------------------------- setup --
  {
    // zero Q (rows >= R stay zero for every segment) through the generic proxy; when R
    // fills its M-tiles every row is loaded by TMA and nothing needs clearing
    if (p.R % 128 != 0) {
      uint4* z = reinterpret_cast<uint4*>(smem);
      for (int i = tid; i < C::kQBytes / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
      fence_proxy_async_smem();
    }
  }
  if (tid == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), MT);  // one commit per M-tile issuer
    mbar_init(smem_u32(&bars->tail), 1);
    mbar_init(smem_u32(&bars->drain), MT);
    for (int m = 0; m < 2; ++m) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&bars->s_full[m][b]), 1);
        mbar_init(smem_u32(&bars->p_full[m][b]), 128);
      }
      mbar_init(smem_u32(&bars->pv_done[m]), 1);
      mbar_init(smem_u32(&bars->o_full[m]), 1);
      mbar_init(smem_u32(&bars->o_empty[m]), 128);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), MT);
    }
    sh->abort_flag = 0;
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
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  // launched as a programmatic dependent of the previous kernel on the stream: everything above
  // (barriers, TMEM, descriptor prefetch) overlaps that kernel's tail; nothing below reads or
  // writes global memory before it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (warp == 2) {
    long long T = 0, start = 0, end = 0;
    Unit first;
    find_range(p, c, T, start, end, first);
    if (lane == 0) {
      sh->T = T;
      sh->start = start;
      sh->end = end;
      if (start < end) sh->first = first;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sh->tmem_base;
  const long long T = sh->T, start = sh->start, end = sh->end;
  const WaitCtx wc{&sh->abort_flag, p.err_word, p.wait_limit_ns};
  const bool have_work = start < end;
  if constexpr (C::kSplitRegs) {
    if (have_work && warp < 4) regs_dec<C::kCtrlRegs>();
  }

  if ((warp == 0 || warp == 3) && have_work) {
    // =========================================================== producers ==
    // Warp 0 loads Q of each segment and the K tiles, warp 3 the V tiles, each into its own
    // half of the ring: K(t) of the CTA's t-th tile in stage t % H, V(t) in stage H + t % H
    // (H = half the stages).  A K slot frees as soon as both M-tiles' S MMAs have read it, long
    // before P V frees the V slot of the same tile, so K loads run further ahead than they
    // could behind V loads in one ring.
    constexpr int H = C::kStages / 2;
    const int kv = warp == 0 ? 0 : 1;
    uint32_t t = 0, q_it = 0, tail_ph = 0;
    bool ok = true;
    Unit x = sh->first;
    for (; ok;) {
      const Segment sg = segment_of(x, start, end, c);
      if (kv == 0) {
        ok = mbar_wait(smem_u32(&bars->q_empty), (q_it & 1) ^ 1, wc);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t bar = smem_u32(&bars->q_full);
          mbar_arrive_expect_tx(bar, (uint32_t)(p.R * kRowBytes * C::kHalves));
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_3d(q_s + hf * (kMaxRows * kRowBytes), &maps.q, bar, hf * 64, x.h * p.g, x.ns * p.S);
        }
        ++q_it;
      }
      const int ctx_row0 = (x.n * p.Hkv + x.h) * p.ctx_stride;
      // paged cache: a context tile is loaded in slices of psub rows, one per page (pages of
      // at least NK keys hold whole tiles); slices past the tile's last key are not loaded
      const int psub = p.page_table ? min(1 << p.page_shift, NK) : NK;
      // paged context: lane s looks up the pool row of slice s of a tile (one table read per
      // lane, all in flight together), one tile ahead of the loads that use it
      auto slice_row = [&](int i) -> int {
        const TileKeys tk = tile_keys(p, x, i);
        if (!p.page_table || tk.is_blk || lane * psub >= tk.count) return 0;
        const int row = paged_row(p, x.n, x.h, tk.first + lane * psub);
        return row < 0 ? (p.num_pages * p.Hkv) << p.page_shift : row;  // a bad page reads as zeros
      };
      int cur_row = slice_row(sg.lo);
      for (int i = sg.lo; i < sg.hi && ok; ++i, ++t) {
        const TileKeys tk = tile_keys(p, x, i);
        const int box_rows = tk.is_blk ? min(p.S, NK) : (p.page_table ? ceil_div(tk.count, psub) * psub : NK);
        const uint32_t bytes = (uint32_t)(box_rows * kRowBytes * C::kHalves);
        const int nsl = p.page_table && !tk.is_blk ? box_rows / psub : 0;   // slices of a paged tile
        const int row_i = cur_row;
        if (i + 1 < sg.hi) cur_row = slice_row(i + 1);
        const int s = kv * H + (int)(t % H);
        ok = mbar_wait(smem_u32(&bars->kv_empty[s]), ((t / H) & 1) ^ 1, wc);
        if (!ok) break;
        const uint32_t slot = kv_s + s * C::kSlotBytes;
        const CUtensorMap* m = tk.is_blk ? (kv ? &maps.v_blk : &maps.k_blk) : (kv ? &maps.v_ctx : &maps.k_ctx);
        // V rows [count, round16(count)) are read by the last PV k-step: zero them.
        const bool fix = kv == 1 && (tk.count & 15) != 0;
        const uint32_t bar = fix ? smem_u32(&bars->tail) : smem_u32(&bars->kv_full[s]);
        if (lane == 0) mbar_arrive_expect_tx(bar, bytes);
        if (nsl > 0) {
          // each slice lands at its row offset in the stage (a multiple of 2 KB: the swizzle
          // pattern stays aligned); issued after the expected byte count is set
          __syncwarp();
          if (lane < nsl)
            for (int hf = 0; hf < C::kHalves; ++hf)
              tma_load_2d(slot + hf * (NK * kRowBytes) + lane * psub * kRowBytes, m, bar, hf * 64, row_i);
        } else if (lane == 0) {
          for (int hf = 0; hf < C::kHalves; ++hf) {
            const uint32_t dst = slot + hf * (NK * kRowBytes);
            if (tk.is_blk) tma_load_3d(dst, m, bar, hf * 64, x.h, x.ns * p.S + tk.first);
            else tma_load_2d(dst, m, bar, hf * 64, ctx_row0 + tk.first);
          }
        }
        if (fix) {
          ok = mbar_wait(smem_u32(&bars->tail), tail_ph, wc);
          tail_ph ^= 1;
          if (!ok) break;
          const int r0 = tk.count, r1 = round16(tk.count);
          const int n16 = (r1 - r0) * 8 * C::kHalves;  // 16-byte chunks to clear
          for (int e = lane; e < n16; e += 32) {
            const int hf = e / ((r1 - r0) * 8);
            const int rem = e - hf * (r1 - r0) * 8;
            const int row = r0 + rem / 8, ch = rem % 8;
            uint4* dst = reinterpret_cast<uint4*>(smem + C::kStageOff + s * C::kSlotBytes +
                                                  hf * (NK * kRowBytes) + row * kRowBytes + ch * 16);
            *dst = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->kv_full[s]));
        }
      }
      if (!ok || sg.last) break;
      x = make_unit(p, x.u + 1, x.Tu + x.tiles);
    }
    if (!ok) {
      // drain: wait (briefly) for loads that may still be landing in shared memory
      int dummy = 0;
      WaitCtx dw{&dummy, nullptr, 2000000ull};
      for (uint32_t j = (t > (uint32_t)H ? t - H : 0); j < t; ++j)
        mbar_wait(smem_u32(&bars->kv_full[kv * H + j % H]), (j / H) & 1, dw);
      if (q_it) mbar_wait(smem_u32(&bars->q_full), (q_it - 1) & 1, dw);
    }
  } else if ((warp == 1 || (warp == 2 && MT == 2)) && have_work) {
    // ====================================================== MMA issuers ==
    // One warp per M-tile (warp 1: M-tile 0, warp 2: M-tile 1), so an M-tile whose P is not
    // ready never holds back the other's MMAs; the tensor core interleaves the two instruction
    // streams.  The whole warp runs the control flow (waits, tile bookkeeping, descriptors stay
    // warp-uniform) and one elected lane issues each burst of MMAs and its commits.  Each warp
    // commits its own reads of a ring slot and of Q, and those barriers expect one commit per
    // M-tile.
    const int m = warp - 1;
    constexpr int H = C::kStages / 2;   // K tiles in stages [0, H), V tiles in [H, 2H)
    uint32_t tb = 0, q_it = 0, G = 0, seg_cnt = 0;   // tb: the CTA's tile count before this segment
    bool ok = true;
    Unit x = sh->first;
    // descriptors: a start-address offset is added in 16-byte units to the low field
    const uint64_t qdesc = smem_desc_sw128(q_s + m * 128 * kRowBytes, 16, 1024);
    const uint64_t kdesc0 = smem_desc_sw128(kv_s, 16, 1024);
    const uint64_t vdesc0 = smem_desc_sw128(kv_s, NK * kRowBytes, 1024);
    const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    const uint32_t idesc_s0 = idesc_bf16_f32(128, 0, 0, 0);
    const uint32_t s_tmem = tmem + m * 128, o_tmem = tmem + 256 + m * D;
    // S = Q K^T of one tile into buffer `buf` (K in ring slot `slot`), then its commits
    auto issue_s = [&](int buf, uint32_t slot, int n_mma) {
      const uint32_t idesc = idesc_s0 | ((uint32_t)(n_mma >> 3) << 17);
      const uint64_t kd = kdesc0 + (uint64_t)((slot * C::kSlotBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kMaxRows * kRowBytes) + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * (NK * kRowBytes) + (kk & 3) * 32;
          tc_mma_ss(s_tmem + buf * NK, qdesc + (off >> 4), kd + (koff >> 4), idesc, kk > 0);
        }
        tc_commit(smem_u32(&bars->s_full[m][buf]));
        tc_commit(smem_u32(&bars->kv_empty[slot]));
      }
      __syncwarp();
    };
    // K (kv = 0) or V (kv = 1) of the CTA's tile t
    auto kv_wait = [&](uint32_t t, int kv) {
      return mbar_wait_warp(smem_u32(&bars->kv_full[kv * H + t % H]), (t / H) & 1, wc);
    };
    for (; ok;) {
      const Segment sg = segment_of(x, start, end, c);
      const int n = sg.hi - sg.lo;
      ok = mbar_wait_warp(smem_u32(&bars->q_full), q_it & 1, wc);
      ++q_it;
      if (!ok) break;
      tc_fence_after();
      // prologue: S of the segment's first NBUF tiles
      for (int j = 0; j < NBUF && j < n && ok; ++j) {
        ok = kv_wait(tb + j, 0);
        if (!ok) break;
        tc_fence_after();
        issue_s((G + j) % NBUF, (tb + j) % H, round16(tile_keys(p, x, sg.lo + j).count));
      }
      for (int j = 0; j < n && ok; ++j, ++G) {
        const int b = G % NBUF;
        const uint32_t ev = H + (tb + j) % H;  // stage of V of tile j
        ok = kv_wait(tb + j, 1);
        if (ok) ok = mbar_wait_warp(smem_u32(&bars->p_full[m][b]), (G / NBUF) & 1, wc);
        if (ok && j == 0) ok = mbar_wait_warp(smem_u32(&bars->o_empty[m]), (seg_cnt & 1) ^ 1, wc);
        if (!ok) break;
        tc_fence_after();
        const int nv = round16(tile_keys(p, x, sg.lo + j).count);
        const uint64_t vd = vdesc0 + (uint64_t)((ev * C::kSlotBytes) >> 4);
        const uint32_t pa = s_tmem + b * NK;
        if (elect_one()) {
          if (nv == NK) {
#pragma unroll
            for (int kk = 0; kk < NK / 16; ++kk)
              tc_mma_ts(o_tmem, pa + kk * 8, vd + (uint64_t)(kk * 16 * kRowBytes >> 4), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
          } else {
            for (int kk = 0; kk < nv / 16; ++kk)
              tc_mma_ts(o_tmem, pa + kk * 8, vd + (uint64_t)(kk * 16 * kRowBytes >> 4), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&bars->pv_done[m]));
          tc_commit(smem_u32(&bars->kv_empty[ev]));
        }
        __syncwarp();
        if (j + NBUF < n) {
          // S of tile j + NBUF into buffer b, after P V(j) has read P(j) from it (in issue order)
          ok = kv_wait(tb + j + NBUF, 0);
          if (!ok) break;
          tc_fence_after();
          issue_s(b, (tb + j + NBUF) % H, round16(tile_keys(p, x, sg.lo + j + NBUF).count));
        }
      }
      if (!ok) break;
      tb += n;
      if (elect_one()) {
        tc_commit(smem_u32(&bars->o_full[m]));
        tc_commit(smem_u32(&bars->q_empty));
      }
      __syncwarp();
      ++seg_cnt;
      if (sg.last) break;
      x = make_unit(p, x.u + 1, x.Tu + x.tiles);
    }
    // drain every MMA this warp issued before TMEM can be released
    if (elect_one()) tc_commit(smem_u32(&bars->drain));
    __syncwarp();
    int dummy = 0;
    WaitCtx dw{&dummy, nullptr, 2000000ull};
    mbar_wait(smem_u32(&bars->drain), 0, dw);
    __syncwarp();
  } else if (warp >= 4 && have_work) {
    // ========================================================= softmax WGs ==
    if constexpr (C::kSplitRegs) regs_inc<C::kSoftmaxRegs>();
    const int m = (warp - 4) >> 2;
    const int q4 = warp & 3;             // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;      // row within the M-tile
    const int r = m * 128 + row;         // packed row of the unit
    if (m < MT) {
      const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
      const uint32_t s_base = tmem + lane_off + m * 128;  // + buffer * NK
      const uint32_t o_addr = tmem + lane_off + 256 + m * D;
      float* stage = epi + (warp - 4) * 32 * 32;
      uint32_t G = 0, seg_cnt = 0;
      bool ok = true;
      Unit x = sh->first;
      for (; ok;) {
        const Segment sg = segment_of(x, start, end, c);
        float m_ref = -INFINITY, l = 0.f;
        // One tile of the softmax: its S row in registers, the row maximum in log2 units, the
        // lazy rescale of O, then P (bf16) over the S buffer.  Full tiles and the masked last
        // tile of a unit run separate code: folding them into one path would make every full
        // tile pay for the masking.
        auto tile = [&](auto full_tag, int count, uint32_t s_addr, bool first) -> bool {
          constexpr bool kFull = decltype(full_tag)::value;
          uint32_t v[NK];
#pragma unroll
          for (int ch = 0; ch < NK / 32; ++ch)
            if (kFull || 32 * ch < count) tmem_ld32(s_addr + 32 * ch, v + 32 * ch);
          tc_wait_ld();
          const float mx = tile_row_max<NK, kFull>(v, count) * p.scale_log2;
          if (first) {
            m_ref = mx;  // O is overwritten by the first PV of the segment
          } else {
            const bool need = mx > m_ref + kRescaleThreshold;
            if (__any_sync(0xffffffffu, need)) {
              // O must hold every earlier PV of this segment before it is rescaled
              if (!mbar_wait(smem_u32(&bars->pv_done[m]), (G - 1) & 1, wc)) return false;
              tc_fence_after();
              const float alpha = need ? fast_exp2(m_ref - mx) : 1.f;
              if (need) {
                m_ref = mx;
                l *= alpha;
              }
#pragma unroll 1
              for (int cc = 0; cc < D / 16; ++cc) {
                uint32_t o[16];
                tmem_ld16(o_addr + cc * 16, o);
                tc_wait_ld();
#pragma unroll
                for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                tmem_st16(o_addr + cc * 16, o);
              }
            }
          }
          l += tile_exp_store<NK, kFull>(v, count, p.scale_log2, m_ref, s_addr);
          return true;
        };
        for (int i = sg.lo; i < sg.hi; ++i, ++G) {
          const int count = tile_keys(p, x, i).count;
          const int b = G % NBUF;
          const uint32_t s_addr = s_base + b * NK;
          ok = mbar_wait(smem_u32(&bars->s_full[m][b]), (G / NBUF) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          // (128-key tiles keep a single masked path: a second copy of their 128-register body
          // would not fit the register budget)
          if constexpr (NK == 128)
            ok = tile(std::false_type{}, count, s_addr, i == sg.lo);
          else
            ok = count == NK ? tile(std::true_type{}, count, s_addr, i == sg.lo)
                             : tile(std::false_type{}, count, s_addr, i == sg.lo);
          if (!ok) break;
          tc_wait_st();
          tc_fence_before();
          mbar_arrive(smem_u32(&bars->p_full[m][b]));
        }
        if (!ok) break;
        // ---- epilogue: O / l to the output (or the segment's partial) ----
        ok = mbar_wait(smem_u32(&bars->o_full[m]), seg_cnt & 1, wc);
        if (!ok) break;
        tc_fence_after();
        const float inv = 1.f / l;
        const int rbase = m * 128 + q4 * 32;  // first packed row of this warp
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(o_addr + cc * 32, o);
          tc_wait_ld();
          if (cc == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->o_empty[m]));  // O fully read: the next segment may overwrite it
          }
          // stage the 32x32 block (16-byte chunks XOR-swizzled by row) for coalesced stores
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float4 f = make_float4(__uint_as_float(o[4 * q]) * inv, __uint_as_float(o[4 * q + 1]) * inv,
                                   __uint_as_float(o[4 * q + 2]) * inv, __uint_as_float(o[4 * q + 3]) * inv);
            reinterpret_cast<float4*>(stage + lane * 32)[q ^ (lane & 7)] = f;
          }
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int rr = k * 4 + (lane >> 3);  // row within the warp's 32
            const int q = lane & 7;
            const int gr = rbase + rr;
            if (gr < p.R) {
              float4 f = reinterpret_cast<const float4*>(stage + rr * 32)[q ^ (rr & 7)];
              if (sg.full) store_out4(p, out_offset(p, x, gr, D) + cc * 32 + q * 4, f);
              else *reinterpret_cast<float4*>(out_row(p, x, sg, gr, D) + cc * 32 + q * 4) = f;
            }
          }
          __syncwarp();
        }
        if (r < p.R) {
          const float lse = (m_ref + __log2f(l)) * 0.6931471805599453f;
          if (sg.full) {
            if (p.lse) {
              const int t = r / p.g, j = r - (r / p.g) * p.g;
              p.lse[(size_t)(x.n * p.Hq + x.h * p.g + j) * (p.NB * p.S) + x.b * p.S + t] = lse;
            }
          } else {
            p.part_lse[(size_t)sg.slot * p.R + r] = lse;
          }
        }
        ++seg_cnt;
        if (sg.last) break;
        x = make_unit(p, x.u + 1, x.Tu + x.tiles);
      }
    }
  }

  // record for the combine: the cut unit (if any) that begins in this range
  if (tid == 64) {
    SplitRecord rec{-1, -1, 0, 0};
    if (have_work) {
      Unit x = sh->first;
      while (x.Tu + x.tiles < end) x = make_unit(p, x.u + 1, x.Tu + x.tiles);
      rec = record_of(x, T, p.C, start, end, range_table(p));
    }
    p.records[c] = rec;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
  if (p.arrivals != nullptr)
    fused_combine<D>(p, T, start, end, sh->first, *(volatile int*)&sh->abort_flag != 0);
}

template <int D, int NK>
void set_smem_attr() {
  cudaFuncSetAttribute(attn_tcgen05_kernel<D, NK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       Cfg<D, NK>::kSmemBytes);
}

template <int D, int NK>
cudaError_t launch(const Problem& p, const TmaMaps& maps, cudaStream_t stream) {
  // a programmatic dependent of the previous kernel on the stream (its setup overlaps that
  // kernel's tail), and cooperative when the fused combine needs every CTA resident at once
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg<D, NK>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.arrivals != nullptr ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, attn_tcgen05_kernel<D, NK>, p, maps);
}

}  // namespace

bool tcgen05_key_tile_supported(int key_tile) { return key_tile == 64 || key_tile == 128; }

cudaError_t launch_attn_tcgen05(const Problem& p, const TmaMaps& maps, cudaStream_t stream) {
  static const bool attr_done = [] {
    set_smem_attr<128, 128>();
    set_smem_attr<128, 64>();
    set_smem_attr<64, 128>();
    set_smem_attr<64, 64>();
    return true;
  }();
  (void)attr_done;
  if (!tcgen05_key_tile_supported(p.key_tile)) return cudaErrorInvalidValue;
  // variant 2: head_dim 128 with 128-key tiles on the transposed-PV kernel (attn_tcgen05_pt.cu)
  if (p.D == 128 && p.key_tile == 128 && p.variant == 2) return launch_attn_pt(p, maps, stream);
  if (p.D == 128) return p.key_tile == 128 ? launch<128, 128>(p, maps, stream) : launch<128, 64>(p, maps, stream);
  return p.key_tile == 128 ? launch<64, 128>(p, maps, stream) : launch<64, 64>(p, maps, stream);
}

}  // namespace tt
