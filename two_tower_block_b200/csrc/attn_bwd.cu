// Block-causal backward pass: gradients of the training loss with respect to the
// denoiser's queries and its own block keys and values.
//
// The method (paperfeed.app review of arXiv 2606.26493, section "Training and
// sampling"): the loss of block b is conditioned on the noisy block and the frozen
// context-tower caches c_{<b}; the context tower runs without gradients.  So, for
// the rows r of block b and the keys k of its key set (context positions < S*b, then
// the block's own S positions):
//     p = exp(scale q.k - lse),  dp = dO.v,  ds = p (dp - Delta),  Delta = dO.out
//     dq = scale sum_k ds k,  dk_blk += scale ds q,  dv_blk += p dO   (block keys only)
//
// Warp-level tensor cores (mma.sync m16n8k16, bf16 operands, fp32 accumulation).
// CTA = (unit (sequence, KV head, block), 64 packed query rows); each of its 4 warps
// owns 16 rows.  Per key tile of 64 keys: S = Q K^T, p from the forward's lse,
// dP = dO V^T, dS, dQ += dS K (dQ stays in registers for the whole key list).  On the
// block's own tiles, P and dS go through shared memory and every warp forms
// dK = dS^T Q and dV = P^T dO for 16 of the keys, added with fp32 atomics (the CTAs
// of a unit's row chunks and the g query heads of a KV head all contribute).  dS and
// P enter these products as bf16 pairs hi + lo, so the gradients carry only the
// rounding of the bf16 inputs.
#include "attn_bwd.h"

#include "errbits.h"
#include "ptx.cuh"

namespace tt {
namespace {

constexpr int kRows = 64;
constexpr int kKeys = 64;
constexpr int kThreads = 128;
constexpr int kLdt = kKeys + 8;  // padded row of the staged P / dS tiles (elements)

template <int D>
__global__ void __launch_bounds__(kThreads) attn_bwd_kernel(const BwdProblem p) {
  constexpr int LDS = D + 8;  // padded smem row (elements)
  constexpr int CH = D / 8;   // 16-byte chunks of a bf16 row
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sO = sQ + kRows * LDS;   // dO
  __nv_bfloat16* sK = sO + kRows * LDS;
  __nv_bfloat16* sV = sK + kKeys * LDS;
  // staged P and dS of a block tile, each as a bf16 pair hi + lo (hi = bf16(x), lo =
  // bf16(x - hi)), so that dK and dV do not inherit a bf16 rounding of dS or P
  __nv_bfloat16* sP = sV + kKeys * LDS;   // [2][kRows][kLdt]: P hi, P lo
  __nv_bfloat16* sS = sP + 2 * kRows * kLdt;  // [2][kRows][kLdt]: dS hi, dS lo
  __shared__ float s_delta[kRows], s_lse2[kRows];

  const int u = blockIdx.x, row0 = blockIdx.y * kRows;
  const int b = u % p.NB, h = (u / p.NB) % p.Hkv, n = u / (p.NB * p.Hkv);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, qq = lane & 3;
  const int tok0 = b * p.S;  // first token of the block
  const float log2e = 1.4426950408889634f;

  // ---- Q and dO rows (bf16, cp.async, zero beyond R); Delta = dO . out; lse ----
  for (int i = tid; i < kRows * CH; i += kThreads) {
    const int r = i / CH, ch = i - (i / CH) * CH, row = row0 + r;
    const bool valid = row < p.R;
    size_t off = 0;
    if (valid) {
      const int t = row / p.g, j = row - (row / p.g) * p.g;
      off = ((size_t)(n * p.N + tok0 + t) * p.Hq + h * p.g + j) * D + ch * 8;
    }
    cp_async_16(smem_u32(sQ + r * LDS + ch * 8), p.q + off, valid);
    cp_async_16(smem_u32(sO + r * LDS + ch * 8), p.dout + off, valid);
  }
  cp_async_commit();
  {
    constexpr int LPR = D / 4;          // lanes per row (one float4 each)
    constexpr int RPW = 32 / LPR;       // rows per warp step
    const int sub = lane / LPR, c4 = lane - sub * LPR;
    for (int r = warp * RPW + sub; r < kRows; r += 4 * RPW) {
      const int row = row0 + r;
      float4 d4 = make_float4(0.f, 0.f, 0.f, 0.f), o4 = d4;
      float lse = 0.f;
      if (row < p.R) {
        const int t = row / p.g, j = row - (row / p.g) * p.g;
        const size_t off = ((size_t)(n * p.N + tok0 + t) * p.Hq + h * p.g + j) * D + c4 * 4;
        const uint2 dr = *reinterpret_cast<const uint2*>(p.dout + off);   // four bf16
        d4 = make_float4(__uint_as_float(dr.x << 16), __uint_as_float(dr.x & 0xFFFF0000u),
                         __uint_as_float(dr.y << 16), __uint_as_float(dr.y & 0xFFFF0000u));
        o4 = *reinterpret_cast<const float4*>(p.out + off);
        lse = p.lse[(size_t)(n * p.Hq + h * p.g + j) * p.N + tok0 + t];
      }
      float dot = d4.x * o4.x + d4.y * o4.y + d4.z * o4.z + d4.w * o4.w;
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (c4 == 0) {
        s_delta[r] = dot;
        s_lse2[r] = lse * log2e;
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  uint32_t qa[D / 16][4], da[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t aq = smem_u32(sQ + (warp * 16 + (lane & 15)) * LDS + kk * 16 + (lane >> 4) * 8);
    ldmatrix_x4(aq, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
    const uint32_t ad = smem_u32(sO + (warp * 16 + (lane & 15)) * LDS + kk * 16 + (lane >> 4) * 8);
    ldmatrix_x4(ad, da[kk][0], da[kk][1], da[kk][2], da[kk][3]);
  }
  const int ra = warp * 16 + gq, rb = ra + 8;   // this thread's two rows within the CTA
  const float lse_a = s_lse2[ra], lse_b = s_lse2[rb];
  const float del_a = s_delta[ra], del_b = s_delta[rb];
  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;

  const int L = tok0;                               // visible context of block b
  const int n_ctx = (L + kKeys - 1) / kKeys, n_blk = (p.S + kKeys - 1) / kKeys;
  for (int it = 0; it < n_ctx + n_blk; ++it) {
    const bool is_blk = it >= n_ctx;
    const int first = is_blk ? (it - n_ctx) * kKeys : it * kKeys;
    const int nvalid = min(kKeys, (is_blk ? p.S : L) - first);
    // ---- K, V tile (zero beyond nvalid) ----
    for (int e = tid; e < kKeys * CH; e += kThreads) {
      const int r = e / CH, ch = e - (e / CH) * CH;
      const bool valid = r < nvalid;
      const __nv_bfloat16* ks = p.k_blk;
      const __nv_bfloat16* vs = p.v_blk;
      if (valid) {
        if (is_blk) {
          const size_t off = ((size_t)(n * p.N + tok0 + first + r) * p.Hkv + h) * D + ch * 8;
          ks = p.k_blk + off;
          vs = p.v_blk + off;
        } else {
          const size_t off = ((size_t)(n * p.Hkv + h) * p.N + first + r) * D + ch * 8;
          ks = p.k_ctx + off;
          vs = p.v_ctx + off;
        }
      }
      cp_async_16(smem_u32(sK + r * LDS + ch * 8), ks, valid);
      cp_async_16(smem_u32(sV + r * LDS + ch * 8), vs, valid);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    // ---- S = Q K^T and dP = dO V^T, 16 rows x 64 keys per warp ----
    float s[kKeys / 8][4], dp[kKeys / 8][4];
#pragma unroll
    for (int nb = 0; nb < kKeys / 8; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nb][e] = dp[nb][e] = 0.f;
#pragma unroll
    for (int nb2 = 0; nb2 < kKeys / 16; ++nb2) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int koff = (nb2 * 16 + (lane & 7) + 8 * (lane >> 4)) * LDS + kk * 16 + 8 * ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(smem_u32(sK + koff), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * nb2], qa[kk], b0, b1);
        mma_bf16_16816(s[2 * nb2 + 1], qa[kk], b2, b3);
        ldmatrix_x4(smem_u32(sV + koff), b0, b1, b2, b3);
        mma_bf16_16816(dp[2 * nb2], da[kk], b0, b1);
        mma_bf16_16816(dp[2 * nb2 + 1], da[kk], b2, b3);
      }
    }
    // ---- p = 2^(s scale log2e - lse log2e) (0 beyond nvalid); ds = p (dp - Delta) ----
#pragma unroll
    for (int nb = 0; nb < kKeys / 8; ++nb) {
      const int col = nb * 8 + 2 * qq;
      const float p0 = col < nvalid ? fast_exp2(s[nb][0] * p.scale_log2 - lse_a) : 0.f;
      const float p1 = col + 1 < nvalid ? fast_exp2(s[nb][1] * p.scale_log2 - lse_a) : 0.f;
      const float p2 = col < nvalid ? fast_exp2(s[nb][2] * p.scale_log2 - lse_b) : 0.f;
      const float p3 = col + 1 < nvalid ? fast_exp2(s[nb][3] * p.scale_log2 - lse_b) : 0.f;
      s[nb][0] = p0;
      s[nb][1] = p1;
      s[nb][2] = p2;
      s[nb][3] = p3;
      dp[nb][0] = p0 * (dp[nb][0] - del_a);
      dp[nb][1] = p1 * (dp[nb][1] - del_a);
      dp[nb][2] = p2 * (dp[nb][2] - del_b);
      dp[nb][3] = p3 * (dp[nb][3] - del_b);
    }
    // ---- dQ += dS K  (A = dS from registers as a bf16 pair hi + lo, B = K rows via
    //      transposed loads): dq does not inherit a bf16 rounding of dS ----
    auto split = [](float x0, float x1, uint32_t& hi, uint32_t& lo) {
      hi = pack_bf16(x0, x1);
      lo = pack_bf16(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xFFFF0000u));
    };
#pragma unroll
    for (int kk = 0; kk < kKeys / 16; ++kk) {
      uint32_t pa[4], pl[4];
      split(dp[2 * kk][0], dp[2 * kk][1], pa[0], pl[0]);
      split(dp[2 * kk][2], dp[2 * kk][3], pa[1], pl[1]);
      split(dp[2 * kk + 1][0], dp[2 * kk + 1][1], pa[2], pl[2]);
      split(dp[2 * kk + 1][2], dp[2 * kk + 1][3], pa[3], pl[3]);
#pragma unroll
      for (int db2 = 0; db2 < D / 16; ++db2) {
        uint32_t b0, b1, b2, b3;
        const uint32_t a = smem_u32(sK + (kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1)) * LDS + db2 * 16 +
                                    8 * (lane >> 4));
        ldmatrix_x4_trans(a, b0, b1, b2, b3);
        mma_bf16_16816(dq[2 * db2], pa, b0, b1);
        mma_bf16_16816(dq[2 * db2 + 1], pa, b2, b3);
        mma_bf16_16816(dq[2 * db2], pl, b0, b1);
        mma_bf16_16816(dq[2 * db2 + 1], pl, b2, b3);
      }
    }

    if (is_blk) {
      // ---- stage P and dS of the block's keys; dK = dS^T Q, dV = P^T dO over this CTA's rows ----
      auto stage = [&](__nv_bfloat16* dst, int r, float x0, float x1) {
        const uint32_t hi = pack_bf16(x0, x1);
        const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
        *reinterpret_cast<uint32_t*>(dst + r * kLdt) = hi;
        *reinterpret_cast<uint32_t*>(dst + (kRows + r) * kLdt) = pack_bf16(x0 - h0, x1 - h1);
      };
#pragma unroll
      for (int nb = 0; nb < kKeys / 8; ++nb) {
        const int col = nb * 8 + 2 * qq;
        stage(sP + col, ra, s[nb][0], s[nb][1]);
        stage(sP + col, rb, s[nb][2], s[nb][3]);
        stage(sS + col, ra, dp[nb][0], dp[nb][1]);
        stage(sS + col, rb, dp[nb][2], dp[nb][3]);
      }
      __syncthreads();
      const int mb = warp;  // this warp's 16 keys
      if (mb * 16 < nvalid) {
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {   // 0: dK from dS and Q; 1: dV from P and dO
          const __nv_bfloat16* sA = which ? sP : sS;
          const __nv_bfloat16* sB = which ? sO : sQ;
          float acc[D / 8][4];
#pragma unroll
          for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
          for (int ks = 0; ks < kRows / 16; ++ks) {
            uint32_t a[4], al[4];
            const int aoff = (ks * 16 + (lane & 7) + 8 * (lane >> 4)) * kLdt + mb * 16 + 8 * ((lane >> 3) & 1);
            ldmatrix_x4_trans(smem_u32(sA + aoff), a[0], a[1], a[2], a[3]);
            ldmatrix_x4_trans(smem_u32(sA + kRows * kLdt + aoff), al[0], al[1], al[2], al[3]);
#pragma unroll
            for (int db2 = 0; db2 < D / 16; ++db2) {
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4_trans(smem_u32(sB + (ks * 16 + (lane & 7) + 8 * ((lane >> 3) & 1)) * LDS + db2 * 16 +
                                         8 * (lane >> 4)),
                                b0, b1, b2, b3);
              mma_bf16_16816(acc[2 * db2], a, b0, b1);
              mma_bf16_16816(acc[2 * db2 + 1], a, b2, b3);
              mma_bf16_16816(acc[2 * db2], al, b0, b1);
              mma_bf16_16816(acc[2 * db2 + 1], al, b2, b3);
            }
          }
          float* dst = which ? p.dv_blk : p.dk_blk;
          const float f = which ? 1.f : p.scale;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int key = mb * 16 + gq + 8 * half;
            if (key < nvalid) {
              float* row = dst + ((size_t)(n * p.N + tok0 + first + key) * p.Hkv + h) * D;
#pragma unroll
              for (int db = 0; db < D / 8; ++db) {
                atomicAdd(row + db * 8 + 2 * qq, f * acc[db][2 * half]);
                atomicAdd(row + db * 8 + 2 * qq + 1, f * acc[db][2 * half + 1]);
              }
            }
          }
        }
      }
    }
    __syncthreads();  // the tile buffers are refilled next
  }

  // ---- dq rows of this CTA ----
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = row0 + (half ? rb : ra);
    if (row >= p.R) continue;
    const int t = row / p.g, j = row - (row / p.g) * p.g;
    float* dst = p.dq + ((size_t)(n * p.N + tok0 + t) * p.Hq + h * p.g + j) * D;
#pragma unroll
    for (int db = 0; db < D / 8; ++db)
      *reinterpret_cast<float2*>(dst + db * 8 + 2 * qq) =
          make_float2(p.scale * dq[db][2 * half], p.scale * dq[db][2 * half + 1]);
  }
}

template <int D>
constexpr size_t smem_bytes() {
  return (size_t)(2 * kRows + 2 * kKeys) * (D + 8) * 2 + (size_t)4 * kRows * kLdt * 2;
}

}  // namespace

cudaError_t launch_attn_bwd(const BwdProblem& p, cudaStream_t stream) {
  static const bool attr_done = [] {
    cudaFuncSetAttribute(attn_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes<128>());
    cudaFuncSetAttribute(attn_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes<64>());
    return true;
  }();
  (void)attr_done;
  const dim3 grid(p.B * p.Hkv * p.NB, (p.R + kRows - 1) / kRows);
  if (p.D == 128) attn_bwd_kernel<128><<<grid, kThreads, smem_bytes<128>(), stream>>>(p);
  else attn_bwd_kernel<64><<<grid, kThreads, smem_bytes<64>(), stream>>>(p);
  return cudaGetLastError();
}

}  // namespace tt
