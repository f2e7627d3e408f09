// Warp-level baseline of the block attention: mma.sync.m16n8k16 (bf16 -> fp32),
// cp.async double-buffered key/value tiles, register online softmax.
//
// CTA = (work range c, 64 packed query rows).  Each of its 4 warps owns 16
// rows; a range is walked segment by segment (see sched.cuh), and every
// segment streams its key tiles (block keys first, then the visible context)
// through one online softmax -- the single joint softmax over [context ;
// block] of the method (paperfeed.app review of arXiv 2606.26493, "The idea:
// freeze the reader, train the writer").
#include "problem.h"
#include "ptx.cuh"
#include "walker.cuh"

namespace tt {
namespace {

constexpr int kRows = 64;   // packed query rows per CTA
constexpr int kKeys = kMmaSyncKeyTile;  // keys per tile
constexpr int kThreads = 128;

template <int D>
__global__ void __launch_bounds__(kThreads) attn_mma_sync_kernel(const Problem p) {
  constexpr int LDS = D + 8;   // padded smem row (elements): ldmatrix rows hit distinct banks
  constexpr int CH = D / 8;    // 16-byte chunks per row
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sK = sQ + kRows * LDS;     // [2][kKeys][LDS]
  __nv_bfloat16* sV = sK + 2 * kKeys * LDS; // [2][kKeys][LDS]
  __shared__ long long s_T, s_start, s_end;
  __shared__ Unit s_first;

  const int c = blockIdx.x, rb = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, qq = lane & 3;  // mma fragment coordinates

  if (warp == 0) {
    long long T = 0, start = 0, end = 0;
    Unit first;
    find_range(p, c, T, start, end, first);
    if (lane == 0) {
      s_T = T; s_start = start; s_end = end;
      if (start < end) s_first = first;
    }
  }
  __syncthreads();
  const long long T = s_T, start = s_start, end = s_end;
  if (start >= end) {
    if (rb == 0 && tid == 0) p.records[c] = SplitRecord{-1, -1, 0, 0};
    return;
  }
  Unit x = s_first;
  const int row0 = rb * kRows;

  for (;;) {
    const Segment sg = segment_of(x, start, end, c);

    // ---- Q rows [row0, row0 + 64) of this unit (rows >= R are zero) ----
    for (int i = tid; i < kRows * CH; i += kThreads) {
      const int r = i / CH, ch = i - (i / CH) * CH;
      const int row = row0 + r;
      const bool valid = row < p.R;
      const __nv_bfloat16* src = p.q;
      if (valid) {
        const int t = row / p.g, j = row - (row / p.g) * p.g;
        src = p.q + ((size_t)(x.ns * p.S + t) * p.Hq + x.h * p.g + j) * D + ch * 8;
      }
      cp_async_16(smem_u32(sQ + r * LDS + ch * 8), src, valid);
    }
    auto load_tile = [&](int i, int buf) {
      const TileKeys tk = tile_keys(p, x, i);
      for (int e = tid; e < kKeys * CH; e += kThreads) {
        const int r = e / CH, ch = e - (e / CH) * CH;
        bool valid = r < tk.count;
        const __nv_bfloat16* ks = p.k_blk;
        const __nv_bfloat16* vs = p.v_blk;
        if (valid) {
          if (tk.is_blk) {
            const size_t off = ((size_t)(x.ns * p.S + tk.first + r) * p.Hkv + x.h) * D + ch * 8;
            ks = p.k_blk + off;
            vs = p.v_blk + off;
          } else if (!p.page_table) {
            const size_t off = ((size_t)(x.n * p.Hkv + x.h) * p.ctx_stride + tk.first + r) * D + ch * 8;
            ks = p.k_ctx + off;
            vs = p.v_ctx + off;
          } else {
            const int row = paged_row(p, x.n, x.h, tk.first + r);  // -1: page outside the pool
            valid = row >= 0;  // a bad page reads as zeros
            if (valid) {
              ks = p.k_ctx + (size_t)row * D + ch * 8;
              vs = p.v_ctx + (size_t)row * D + ch * 8;
            }
          }
        }
        cp_async_16(smem_u32(sK + (buf * kKeys + r) * LDS + ch * 8), ks, valid);
        cp_async_16(smem_u32(sV + (buf * kKeys + r) * LDS + ch * 8), vs, valid);
      }
    };
    load_tile(sg.lo, 0);
    cp_async_commit();

    uint32_t qa[D / 16][4];
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int i = sg.lo; i < sg.hi; ++i) {
      const int buf = (i - sg.lo) & 1;
      if (i + 1 < sg.hi) {
        load_tile(i + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      if (i == sg.lo) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a = smem_u32(sQ + (warp * 16 + (lane & 15)) * LDS + kk * 16 + (lane >> 4) * 8);
          ldmatrix_x4(a, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
        }
      }
      const int nvalid = tile_keys(p, x, i).count;

      // ---- S = Q K^T for 16 rows x 64 keys ----
      float s[kKeys / 8][4];
#pragma unroll
      for (int nb = 0; nb < kKeys / 8; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
      const __nv_bfloat16* kb = sK + buf * kKeys * LDS;
#pragma unroll
      for (int nb2 = 0; nb2 < kKeys / 16; ++nb2) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t b0, b1, b2, b3;
          const uint32_t a = smem_u32(kb + (nb2 * 16 + (lane & 7) + 8 * (lane >> 4)) * LDS + kk * 16 +
                                      8 * ((lane >> 3) & 1));
          ldmatrix_x4(a, b0, b1, b2, b3);
          mma_bf16_16816(s[2 * nb2], qa[kk], b0, b1);
          mma_bf16_16816(s[2 * nb2 + 1], qa[kk], b2, b3);
        }
      }

      // ---- online softmax in the log2 domain ----
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nb = 0; nb < kKeys / 8; ++nb) {
        const int col = nb * 8 + 2 * qq;
        s[nb][0] = col < nvalid ? s[nb][0] * p.scale_log2 : -INFINITY;
        s[nb][1] = col + 1 < nvalid ? s[nb][1] * p.scale_log2 : -INFINITY;
        s[nb][2] = col < nvalid ? s[nb][2] * p.scale_log2 : -INFINITY;
        s[nb][3] = col + 1 < nvalid ? s[nb][3] * p.scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, fmaxf(s[nb][0], s[nb][1]));
        mx1 = fmaxf(mx1, fmaxf(s[nb][2], s[nb][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);  // 0 on the first tile
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int nb = 0; nb < kKeys / 8; ++nb) {
        // weights rounded to bf16 here, so the row sum uses what the PV product uses
        s[nb][0] = __bfloat162float(__float2bfloat16_rn(fast_exp2(s[nb][0] - mn0)));
        s[nb][1] = __bfloat162float(__float2bfloat16_rn(fast_exp2(s[nb][1] - mn0)));
        s[nb][2] = __bfloat162float(__float2bfloat16_rn(fast_exp2(s[nb][2] - mn1)));
        s[nb][3] = __bfloat162float(__float2bfloat16_rn(fast_exp2(s[nb][3] - mn1)));
        rs0 += s[nb][0] + s[nb][1];
        rs1 += s[nb][2] + s[nb][3];
      }
      l0 = l0 * al0 + rs0;
      l1 = l1 * al1 + rs1;
#pragma unroll
      for (int db = 0; db < D / 8; ++db) {
        o[db][0] *= al0; o[db][1] *= al0;
        o[db][2] *= al1; o[db][3] *= al1;
      }

      // ---- O += P V ----
      const __nv_bfloat16* vb = sV + buf * kKeys * LDS;
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int db2 = 0; db2 < D / 16; ++db2) {
          uint32_t b0, b1, b2, b3;
          const uint32_t a = smem_u32(vb + (kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1)) * LDS +
                                      db2 * 16 + 8 * (lane >> 4));
          ldmatrix_x4_trans(a, b0, b1, b2, b3);
          mma_bf16_16816(o[2 * db2], pa, b0, b1);
          mma_bf16_16816(o[2 * db2 + 1], pa, b2, b3);
        }
      }
      __syncthreads();  // every warp is done with `buf` before it is refilled
    }

    // ---- epilogue: normalise, write final rows or the segment's partial ----
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = row0 + warp * 16 + gq + 8 * half;
      if (r >= p.R) continue;
      const float l = half ? l1 : l0;
      const float inv = 1.f / l;
      const float lse = ((half ? m1 : m0) + __log2f(l)) * 0.6931471805599453f;
      const int t = r / p.g, j = r - (r / p.g) * p.g;
      const size_t off = out_offset(p, x, r, D);
      float* part = p.part_o + ((size_t)sg.slot * p.R + r) * D;
#pragma unroll
      for (int db = 0; db < D / 8; ++db) {
        float2 v = make_float2(o[db][2 * half] * inv, o[db][2 * half + 1] * inv);
        if (sg.full) store_out2(p, off + db * 8 + 2 * qq, v);
        else *reinterpret_cast<float2*>(part + db * 8 + 2 * qq) = v;
      }
      if (qq == 0) {
        if (sg.full) {
          if (p.lse)
            p.lse[(size_t)(x.n * p.Hq + x.h * p.g + j) * (p.NB * p.S) + x.b * p.S + t] = lse;
        } else {
          p.part_lse[(size_t)sg.slot * p.R + r] = lse;
        }
      }
    }

    if (sg.last) {
      if (rb == 0 && tid == 0) p.records[c] = record_of(x, T, p.C, start, end, range_table(p));
      break;
    }
    x = make_unit(p, x.u + 1, x.Tu + x.tiles);
  }
}

}  // namespace

size_t attn_mma_sync_smem_bytes(int D) { return (size_t)(kRows + 4 * kKeys) * (D + 8) * 2; }

cudaError_t launch_attn_mma_sync(const Problem& p, cudaStream_t stream) {
  const size_t smem = attn_mma_sync_smem_bytes(p.D);
  dim3 grid(p.C, (p.R + kRows - 1) / kRows);
  // The opt-in shared-memory size is set once per process (not during a graph capture).
  static const bool attr_done = [] {
    cudaFuncSetAttribute(attn_mma_sync_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_mma_sync_smem_bytes(128));
    cudaFuncSetAttribute(attn_mma_sync_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_mma_sync_smem_bytes(64));
    return true;
  }();
  (void)attr_done;
  if (p.D == 128) attn_mma_sync_kernel<128><<<grid, kThreads, smem, stream>>>(p);
  else attn_mma_sync_kernel<64><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace tt
