// Block attention on tcgen05 for head_dim 128 with the PV product transposed.
//
// The method (paperfeed.app review of arXiv 2606.26493, "Nemotron-Labs-
// TwoTower", section "The idea: freeze the reader, train the writer"): the S
// noisy block queries of denoiser layer i attend, in one softmax, to the
// frozen context tower's layer-i cache followed by the block's own keys.
//
// Why transposed.  Both M-tiles (the up to 256 packed query rows of a unit)
// share every key tile.  O^T = V^T P^T computes all 256 rows with one N=256
// instruction per 16 keys (the tensor core's most efficient shape), and S_0,
// S_1 = Q_m K^T are issued k-step by k-step into two accumulators so their
// instructions overlap.  P goes to shared memory (B operand of the PV
// product), so S(j+1) no longer has to wait for P(j) to be consumed: the
// tensor core computes S(j+1) while the softmax works on tile j.
//
// Roles (384 threads):
//   warp 0       TMA producer: Q per segment; K and V tiles into a 3-slot ring,
//                with the context tiles further ahead prefetched into L2.
//   warp 1       TMEM owner, MMA issuer (one thread).
//   warps 4..7   softmax of rows 0..127   (thread = TMEM lane of S_0 = row)
//   warps 8..11  softmax of rows 128..255 (thread = TMEM lane of S_1 = row)
// TMEM columns: S_0 [0,128), S_1 [128,256), O^T [256,512) (lane = d, column =
// packed row).  Shared memory: Q 64 KB | P 64 KB | ring 96 KB | barriers.
//
// Softmax per tile: load the S row, release S (the MMA may overwrite it),
// row maximum, lazy reference update (O is rescaled only when the maximum
// grows by more than 2^8), p = 2^(s*c - m) rounded to bf16, row sum of the
// rounded weights, P row to shared memory once the previous PV has read it.
// A row whose reference moved leaves its factor in shared memory; after
// both warpgroups have written P, warpgroup 0 (lanes = d) rescales the O^T
// columns of those rows, then releases the PV product.
//
// Every wait is bounded (ptx.cuh: mbar_wait); on a timeout the CTA raises the
// error word and returns.
#include "problem.h"
#include "ptx.cuh"
#include "tc_common.cuh"
#include "walker.cuh"

namespace tt {
namespace {

constexpr int kThreads = 384;
constexpr int kD = 128;                  // head dim of this kernel
constexpr int kNK = 128;                 // keys per tile
constexpr int kRows = 256;               // two 128-row M-tiles
constexpr int kRowBytes = 128;           // one 64-element bf16 half-row (128-byte swizzle atom width)
constexpr int kHalfBytes = kRows * kRowBytes;     // 32 KB
constexpr int kQOff = 0;                          // Q: [2 d-halves][256 rows][128 B]
constexpr int kPOff = 2 * kHalfBytes;             // P: [2 key-halves][256 rows][128 B]
constexpr int kRingOff = 4 * kHalfBytes;          // K/V ring
constexpr int kSlotBytes = kNK * kRowBytes * 2;   // 32 KB: one K or V tile
constexpr int kStages = 3;
constexpr int kMiscOff = kRingOff + kStages * kSlotBytes;
constexpr int kPrefetchAhead = 3;        // context tiles prefetched into L2 ahead of the ring
constexpr float kRescaleThreshold = 8.0f;
constexpr int kCtrlRegs = 72, kSoftmaxRegs = 208;
static_assert(4 * 32 * kCtrlRegs + 8 * 32 * kSoftmaxRegs <= kThreads * 168, "register split");

struct Bars {
  uint64_t q_full, q_empty, tail, drain;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, s_free, p_half, p_ready, pv_done, o_full, o_empty, epi_a, epi_b;
};

struct Misc {
  Bars bars;
  uint32_t tmem_base;
  int abort_flag;
  int resc[3];              // rows whose reference moved, per tile (mod 3)
  int pad;
  long long T, start, end;
  Unit first;
  float alpha[2][kRows];    // per-row O^T rescale factors, per tile (mod 2)
};

constexpr int kSmemBytes = kMiscOff + (int)sizeof(Misc);
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ uint64_t add16(uint64_t desc, uint32_t byte_off) { return desc + (uint64_t)(byte_off >> 4); }

__global__ void __launch_bounds__(kThreads, 1)
    attn_pt_kernel(const Problem p, const __grid_constant__ TmaMaps maps) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Misc* ms = reinterpret_cast<Misc*>(smem + kMiscOff);
  Bars* bars = &ms->bars;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled layouts need a 1024-byte aligned base
    if (tid == 0) {
      raise_error(p.err_word, kErrInternal);
      p.records[c] = SplitRecord{-1, -1, 0, 0};
    }
    return;
  }
  const uint32_t q_s = sbase + kQOff, p_s = sbase + kPOff, ring_s = sbase + kRingOff;

  // ---------------------------------------------------------------- setup --
  {
    uint4* z = reinterpret_cast<uint4*>(smem + kQOff);  // Q rows >= R stay zero
    for (int i = tid; i < 2 * kHalfBytes / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (tid == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 1);
    mbar_init(smem_u32(&bars->tail), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->s_free), 256);
    mbar_init(smem_u32(&bars->p_half), 256);
    mbar_init(smem_u32(&bars->p_ready), 128);
    mbar_init(smem_u32(&bars->pv_done), 1);
    mbar_init(smem_u32(&bars->o_full), 1);
    mbar_init(smem_u32(&bars->o_empty), 256);
    mbar_init(smem_u32(&bars->epi_a), 256);
    mbar_init(smem_u32(&bars->epi_b), 256);
    ms->abort_flag = 0;
    ms->resc[0] = ms->resc[1] = ms->resc[2] = 0;
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
    tmem_alloc(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish();
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
  tc_fence_after();

  const uint32_t tmem = ms->tmem_base;
  const long long T = ms->T, start = ms->start, end = ms->end;
  const WaitCtx wc{&ms->abort_flag, p.err_word, p.wait_limit_ns};
  const bool have_work = start < end;
  if (have_work && warp < 4) regs_dec<kCtrlRegs>();

  if (warp == 0 && have_work) {
    // ============================================================ producer ==
    uint32_t it = 0, q_it = 0, tail_ph = 0;
    bool ok = true;
    Unit x = ms->first;
    for (; ok;) {
      const Segment sg = segment_of(x, start, end, c);
      const int ctx_row0 = (x.n * p.Hkv + x.h) * p.ctx_stride;
      auto prefetch = [&](int i) {  // context tile i of this segment into L2
        if (i >= sg.hi || i < p.blk_tiles) return;
        const TileKeys tk = tile_keys(p, x, i);
        for (int hf = 0; hf < 2; ++hf) {
          tma_prefetch_l2_2d(&maps.k_ctx, hf * 64, ctx_row0 + tk.first);
          tma_prefetch_l2_2d(&maps.v_ctx, hf * 64, ctx_row0 + tk.first);
        }
      };
      if (lane == 0)
        for (int i = sg.lo + 1; i < sg.lo + kPrefetchAhead; ++i) prefetch(i);
      ok = mbar_wait(smem_u32(&bars->q_empty), (q_it & 1) ^ 1, wc);
      if (!ok) break;
      if (lane == 0) {
        const uint32_t bar = smem_u32(&bars->q_full);
        mbar_arrive_expect_tx(bar, (uint32_t)(p.R * kRowBytes * 2));
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(q_s + hf * kHalfBytes, &maps.q, bar, hf * 64, x.h * p.g, x.ns * p.S);
      }
      ++q_it;
      // ring entries in the order the MMA consumes them: K0, K1, V0, K2, V1, ..., V(n-1)
      const int n = sg.hi - sg.lo;
      for (int e = 0; e < 2 * n && ok; ++e, ++it) {
        int j, kv;
        if (e == 0) { j = 0; kv = 0; }
        else if (e == 2 * n - 1) { j = n - 1; kv = 1; }
        else if (e & 1) { j = (e + 1) >> 1; kv = 0; }
        else { j = (e >> 1) - 1; kv = 1; }
        const int i = sg.lo + j;
        if (kv == 0 && lane == 0) prefetch(i + kPrefetchAhead);
        const TileKeys tk = tile_keys(p, x, i);
        const int box_rows = tk.is_blk ? min(p.S, kNK) : kNK;
        const uint32_t bytes = (uint32_t)(box_rows * kRowBytes * 2);
        {
          const int s = it % kStages;
          ok = mbar_wait(smem_u32(&bars->kv_empty[s]), ((it / kStages) & 1) ^ 1, wc);
          if (!ok) break;
          const uint32_t slot = ring_s + s * kSlotBytes;
          const CUtensorMap* m = tk.is_blk ? (kv ? &maps.v_blk : &maps.k_blk) : (kv ? &maps.v_ctx : &maps.k_ctx);
          // V rows [count, round16(count)) are read by the last PV k-step: zero them.
          const bool fix = kv == 1 && (tk.count & 15) != 0;
          const uint32_t bar = fix ? smem_u32(&bars->tail) : smem_u32(&bars->kv_full[s]);
          if (lane == 0) {
            mbar_arrive_expect_tx(bar, bytes);
            for (int hf = 0; hf < 2; ++hf) {
              const uint32_t dst = slot + hf * (kNK * kRowBytes);
              if (tk.is_blk) tma_load_3d(dst, m, bar, hf * 64, x.h, x.ns * p.S + tk.first);
              else tma_load_2d(dst, m, bar, hf * 64, ctx_row0 + tk.first);
            }
          }
          if (fix) {
            ok = mbar_wait(smem_u32(&bars->tail), tail_ph, wc);
            tail_ph ^= 1;
            if (!ok) break;
            const int r0 = tk.count, r1 = round16(tk.count);
            const int n16 = (r1 - r0) * 8 * 2;  // 16-byte chunks to clear
            for (int q = lane; q < n16; q += 32) {
              const int hf = q / ((r1 - r0) * 8);
              const int rem = q - hf * (r1 - r0) * 8;
              const int row = r0 + rem / 8, ch = rem % 8;
              uint4* dst = reinterpret_cast<uint4*>(smem + kRingOff + s * kSlotBytes + hf * (kNK * kRowBytes) +
                                                    row * kRowBytes + ch * 16);
              *dst = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->kv_full[s]));
          }
        }
      }
      if (!ok || sg.last) break;
      x = make_unit(p, x.u + 1, x.Tu + x.tiles);
    }
    if (!ok) {
      // drain: wait (briefly) for loads that may still be landing in shared memory
      int dummy = 0;
      WaitCtx dw{&dummy, nullptr, 2000000ull};
      for (uint32_t j = (it > (uint32_t)kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait(smem_u32(&bars->kv_full[j % kStages]), (j / kStages) & 1, dw);
      if (q_it) mbar_wait(smem_u32(&bars->q_full), (q_it - 1) & 1, dw);
    }
  } else if (warp == 1 && have_work) {
    // ============================================================= MMA warp ==
    if (lane == 0) {
      uint32_t it = 0, q_it = 0, G = 0, seg_cnt = 0;
      bool ok = true;
      Unit x = ms->first;
      const uint64_t qdesc = smem_desc_sw128(q_s, 16, 1024);           // A of S: K-major
      const uint64_t kdesc = smem_desc_sw128(ring_s, 16, 1024);        // B of S: K-major
      const uint64_t vdesc = smem_desc_sw128(ring_s, kNK * kRowBytes, 1024);  // A of O^T: MN-major (d)
      const uint64_t pdesc = smem_desc_sw128(p_s, 16, 1024);           // B of O^T: K-major (keys)
      const uint32_t idesc_s0 = idesc_bf16_f32(128, 0, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, kRows, 1, 0);
      auto kv_wait = [&](uint32_t e) {
        return mbar_wait(smem_u32(&bars->kv_full[e % kStages]), (e / kStages) & 1, wc);
      };
      // S_0 and S_1 of one key tile, k-steps interleaved over the two accumulators
      auto issue_s = [&](uint32_t e, int n_mma) {
        const uint32_t idesc = idesc_s0 | ((uint32_t)(n_mma >> 3) << 17);
        const uint64_t kd = add16(kdesc, (e % kStages) * kSlotBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          const uint32_t ko = (kk >> 2) * (kNK * kRowBytes) + (kk & 3) * 32;
          tc_mma_ss(tmem + 0, add16(qdesc, qo), add16(kd, ko), idesc, kk > 0);
          tc_mma_ss(tmem + 128, add16(qdesc, qo + 128 * kRowBytes), add16(kd, ko), idesc, kk > 0);
        }
        tc_commit(smem_u32(&bars->s_full));
        tc_commit(smem_u32(&bars->kv_empty[e % kStages]));
      };
      for (; ok;) {
        const Segment sg = segment_of(x, start, end, c);
        const int n = sg.hi - sg.lo;
        ok = mbar_wait(smem_u32(&bars->q_full), q_it & 1, wc);
        ++q_it;
        if (!ok) break;
        // S of the segment's first tile, once the softmax has released the previous S
        // ring entries of this segment: K(0) = 0, K(j) = 2j - 1, V(j) = 2j + 2 (last V: 2n - 1)
        auto ek = [&](int j) { return it + (j == 0 ? 0u : (uint32_t)(2 * j - 1)); };
        auto ev_of = [&](int j) { return it + (j == n - 1 ? (uint32_t)(2 * n - 1) : (uint32_t)(2 * j + 2)); };
        if (G > 0) ok = mbar_wait(smem_u32(&bars->s_free), (G - 1) & 1, wc);
        if (ok) ok = kv_wait(it);
        if (!ok) break;
        tc_fence_after();
        issue_s(it, round16(tile_keys(p, x, sg.lo).count));
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t g = G + j;
          if (j + 1 < n) {
            ok = mbar_wait(smem_u32(&bars->s_free), g & 1, wc);
            if (ok) ok = kv_wait(ek(j + 1));
            if (!ok) break;
            tc_fence_after();
            issue_s(ek(j + 1), round16(tile_keys(p, x, sg.lo + j + 1).count));
          }
          const uint32_t ev = ev_of(j);  // V of tile j
          ok = kv_wait(ev);
          if (ok) ok = mbar_wait(smem_u32(&bars->p_ready), g & 1, wc);
          if (ok && j == 0) ok = mbar_wait(smem_u32(&bars->o_empty), (seg_cnt & 1) ^ 1, wc);
          if (!ok) break;
          tc_fence_after();
          const int nv = round16(tile_keys(p, x, sg.lo + j).count);
          const uint64_t vd = add16(vdesc, (ev % kStages) * kSlotBytes);
          for (int kk = 0; kk < nv / 16; ++kk)
            tc_mma_ss(tmem + 256, add16(vd, kk * 16 * kRowBytes), add16(pdesc, (kk >> 2) * kHalfBytes + (kk & 3) * 32),
                      idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(smem_u32(&bars->pv_done));
          tc_commit(smem_u32(&bars->kv_empty[ev % kStages]));
        }
        if (!ok) break;
        tc_commit(smem_u32(&bars->o_full));
        tc_commit(smem_u32(&bars->q_empty));
        it += 2 * n;
        G += n;
        ++seg_cnt;
        if (sg.last) break;
        x = make_unit(p, x.u + 1, x.Tu + x.tiles);
      }
      // drain every MMA this thread issued before TMEM can be released
      tc_commit(smem_u32(&bars->drain));
      int dummy = 0;
      WaitCtx dw{&dummy, nullptr, 2000000ull};
      mbar_wait(smem_u32(&bars->drain), 0, dw);
    }
    __syncwarp();
  } else if (warp >= 4 && have_work) {
    // ========================================================= softmax WGs ==
    regs_inc<kSoftmaxRegs>();
    const int wg = (warp - 4) >> 2;         // M-tile
    const int q4 = warp & 3;                // TMEM lane quarter
    const int r = wg * 128 + q4 * 32 + lane;  // packed row owned by this thread
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + wg * 128;
    const uint32_t ot_addr = tmem + lane_off + 256;   // O^T: this thread's lane is d = q4*32 + lane
    uint8_t* prow = smem + kPOff + r * kRowBytes;     // this row's P (two key-halves, 32 KB apart)
    float* inv_l = reinterpret_cast<float*>(smem + kPOff);  // epilogue only (P is free then)
    uint32_t G = 0, seg_cnt = 0;
    bool ok = true;
    Unit x = ms->first;
    for (; ok;) {
      const Segment sg = segment_of(x, start, end, c);
      float m_ref = -INFINITY, l = 0.f;
      for (int i = sg.lo; i < sg.hi; ++i, ++G) {
        const int count = tile_keys(p, x, i).count;
        const bool full = count == kNK;
        ok = mbar_wait(smem_u32(&bars->s_full), G & 1, wc);
        if (!ok) break;
        tc_fence_after();
        if (tid == 128) ms->resc[(G + 1) % 3] = 0;  // reused two tiles from now
        uint32_t v[kNK];
#pragma unroll
        for (int ch = 0; ch < kNK / 32; ++ch)
          if (full || 32 * ch < count) tmem_ld32(s_addr + 32 * ch, v + 32 * ch);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->s_free));  // S may now be overwritten by the next tile
        const float mx = (full ? tile_row_max<kNK, true>(v, count) : tile_row_max<kNK, false>(v, count)) * p.scale_log2;
        float alpha = 1.f;
        bool need = false;
        if (i == sg.lo) {
          m_ref = mx;  // O^T is overwritten by the segment's first PV
        } else if (mx > m_ref + kRescaleThreshold) {
          need = true;
          alpha = fast_exp2(m_ref - mx);
          m_ref = mx;
          l *= alpha;
        }
        uint32_t pk[kNK / 2];
        l += full ? tile_exp_pack<kNK, true>(v, count, p.scale_log2, m_ref, pk)
                  : tile_exp_pack<kNK, false>(v, count, p.scale_log2, m_ref, pk);
        // the previous PV must have read P before it is overwritten
        if (G > 0) {
          ok = mbar_wait(smem_u32(&bars->pv_done), (G - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint32_t* w = pk + 32 * h + 4 * ch;
            *reinterpret_cast<uint4*>(prow + h * kHalfBytes + ((ch ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        fence_proxy_async_smem();
        ms->alpha[G & 1][r] = alpha;
        if (need) atomicAdd(&ms->resc[G % 3], 1);
        mbar_arrive(smem_u32(&bars->p_half));
        if (wg == 0) {
          // every row's P and factor are in: rescale the moved O^T columns, then release PV
          ok = mbar_wait(smem_u32(&bars->p_half), G & 1, wc);
          if (!ok) break;
          if (i > sg.lo && *reinterpret_cast<volatile int*>(&ms->resc[G % 3]) != 0) {
            const float* al = ms->alpha[G & 1];
#pragma unroll 1
            for (int cc = 0; cc < kRows / 32; ++cc) {
              uint32_t o[32];
              tmem_ld32(ot_addr + 32 * cc, o);
              tc_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * al[32 * cc + k]);
              tmem_st32(ot_addr + 32 * cc, o);
            }
            tc_wait_st();
          }
          tc_fence_before();
          mbar_arrive(smem_u32(&bars->p_ready));
        }
      }
      if (!ok) break;
      // ---- epilogue: O^T / l to the output rows (or the segment's partial) ----
      ok = mbar_wait(smem_u32(&bars->o_full), seg_cnt & 1, wc);
      if (!ok) break;
      tc_fence_after();
      inv_l[r] = 1.f / l;
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
      mbar_arrive(smem_u32(&bars->epi_a));
      ok = mbar_wait(smem_u32(&bars->epi_a), seg_cnt & 1, wc);
      if (!ok) break;
      const int d = q4 * 32 + lane;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        const int col = wg * 128 + cc * 32;  // packed rows col .. col+31
        uint32_t o[32];
        tmem_ld32(ot_addr + col, o);
        tc_wait_ld();
        if (cc == 3) {
          tc_fence_before();
          mbar_arrive(smem_u32(&bars->o_empty));  // O^T read: the next segment may overwrite it
        }
#pragma unroll 4
        for (int k = 0; k < 32; ++k) {
          const int row = col + k;
          if (row < p.R) out_row(p, x, sg, row, kD)[d] = __uint_as_float(o[k]) * inv_l[row];
        }
      }
      mbar_arrive(smem_u32(&bars->epi_b));  // inv_l read by all before P is rewritten
      ok = mbar_wait(smem_u32(&bars->epi_b), seg_cnt & 1, wc);
      if (!ok) break;
      ++seg_cnt;
      if (sg.last) break;
      x = make_unit(p, x.u + 1, x.Tu + x.tiles);
    }
  }

  // record for the combine: the cut unit (if any) that begins in this range
  if (tid == 64) {
    SplitRecord rec{-1, -1, 0, 0};
    if (have_work) {
      Unit x = ms->first;
      while (x.Tu + x.tiles < end) x = make_unit(p, x.u + 1, x.Tu + x.tiles);
      rec = record_of(x, T, p.C, start, end, range_table(p));
    }
    p.records[c] = rec;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

size_t attn_pt_smem_bytes() { return kSmemBytes; }

cudaError_t launch_attn_pt(const Problem& p, const TmaMaps& maps, cudaStream_t stream) {
  static const bool attr_done = [] {
    cudaFuncSetAttribute(attn_pt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    return true;
  }();
  (void)attr_done;
  if (p.D != kD) return cudaErrorInvalidValue;
  attn_pt_kernel<<<p.C, kThreads, kSmemBytes, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace tt
