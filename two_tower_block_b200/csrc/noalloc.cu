// Decode entry point that allocates no device memory.
//
// Some callers cannot call cudaMalloc: inference engines and framework
// plugins that reserve all device memory up front and own the allocator, or
// latency-critical serving loops where an allocation may implicitly
// synchronise the device.  For them, tt_block_attn_noalloc runs the same
// decode kernels as tt_block_attn without a plan: its scratch (split partials,
// per-range records, error word) lives in one file-scope device array of
// fixed size, reserved on every GPU that loads this library until the process
// exits.  The caller passes inputs and outputs as usual.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/tt_block_attn.h"
#include "problem.h"
#include "sched.cuh"

namespace tt {
extern thread_local std::string g_detail;  // shared with the other entry points (api.cpp)
}

namespace {

// 40 MiB per device: room for one range per SM (148) at S*g = 256 rows and head_dim 128
constexpr size_t kScratchBytes = size_t(40) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct DeviceSetup {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_scratch on this device
  int sm_count = 0;
  int major = 0;
};
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mutex;

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch bytes the split needs for C ranges of R rows x D columns.
size_t scratch_need(int C, int R, int D) {
  return up256(size_t(2) * C * R * D * sizeof(float)) + up256(size_t(2) * C * R * sizeof(float)) +
         up256(size_t(C) * sizeof(tt::SplitRecord)) + 256;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!fn) return false;
  cuuint32_t elem[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

tt_status_t reject(tt_status_t st, const std::string& why) {
  tt::g_detail = why;
  return st;
}

// Once per device, with that device current: resolve the array's device address.
tt_status_t setup_device(int dev, DeviceSetup** out) {
  if (dev < 0 || dev >= kMaxDevices) return reject(TT_ERR_UNSUPPORTED, "device ordinal beyond 64");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceSetup& s = g_setup[dev];
  if (!s.ready) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_scratch);
    if (e != cudaSuccess) return reject(TT_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    e = cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&s.major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return reject(TT_ERR_CUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
    s.scratch = static_cast<unsigned char*>(ptr);
    s.ready = true;
  }
  *out = &s;
  return TT_OK;
}

}  // namespace

extern "C" TT_API tt_status_t tt_block_attn_noalloc(const tt_block_attn_desc* desc, const void* q, const void* k_ctx,
                                                    const void* v_ctx, const void* k_blk, const void* v_blk,
                                                    const int32_t* ctx_lens, float* out, float* lse,
                                                    uint32_t* status, tt_stream_t stream) {
  tt::g_detail.clear();
  if (!desc) return reject(TT_ERR_INVALID_ARG, "null descriptor");
  const tt_block_attn_desc d = *desc;
  if (d.batch < 0 || d.num_q_heads < 1 || d.num_kv_heads < 1 || d.block_size < 1 || d.ctx_capacity < 0 ||
      d.num_ctas < 0 || d.wait_timeout_us < 0 || d.num_q_heads % d.num_kv_heads)
    return reject(TT_ERR_INVALID_ARG, "malformed descriptor");
  if (d.seq_len != 0 || d.flags != 0) return reject(TT_ERR_INVALID_ARG, "decode only: seq_len and flags must be 0");
  if (!(d.scale >= 0.f) || std::isinf(d.scale)) return reject(TT_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (d.kernel < TT_KERNEL_AUTO || d.kernel > TT_KERNEL_MMA_SYNC) return reject(TT_ERR_INVALID_ARG, "unknown kernel");
  if (d.head_dim != 64 && d.head_dim != 128) return reject(TT_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  const int g = d.num_q_heads / d.num_kv_heads;
  const int R = d.block_size * g;
  if (R > 256) return reject(TT_ERR_UNSUPPORTED, "block_size * (Hq/Hkv) must be <= 256");
  if ((long long)d.batch * d.num_kv_heads * d.ctx_capacity > (1ll << 31) - 1)
    return reject(TT_ERR_UNSUPPORTED, "context cache rows beyond 2^31");
  if (d.num_ctas > 0 && scratch_need(d.num_ctas, R, d.head_dim) > kScratchBytes)
    return reject(TT_ERR_INVALID_ARG, "num_ctas needs " + std::to_string(scratch_need(d.num_ctas, R, d.head_dim)) +
                                          " scratch bytes; the no-allocation scratch holds " +
                                          std::to_string(kScratchBytes));
  if (d.batch == 0) return TT_OK;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!q || !k_blk || !v_blk || !ctx_lens || !out || (d.ctx_capacity > 0 && (!k_ctx || !v_ctx)))
    return reject(TT_ERR_INVALID_ARG, "null tensor pointer");
  if (!a16(q) || !a16(k_ctx) || !a16(v_ctx) || !a16(k_blk) || !a16(v_blk) || !a16(out) || !a16(lse) ||
      (reinterpret_cast<uintptr_t>(ctx_lens) & 3u) || (reinterpret_cast<uintptr_t>(status) & 3u))
    return reject(TT_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return reject(TT_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  DeviceSetup* ds = nullptr;
  tt_status_t st = setup_device(dev, &ds);
  if (st != TT_OK) return st;

  const int kernel = (d.kernel == TT_KERNEL_MMA_SYNC || ds->major != 10) ? TT_KERNEL_MMA_SYNC : TT_KERNEL_TCGEN05;
  const int key_tile = kernel == TT_KERNEL_TCGEN05 ? tt::kTcgen05KeyTile : tt::kMmaSyncKeyTile;
  int C = d.num_ctas;
  if (C == 0) {
    C = kernel == TT_KERNEL_TCGEN05 ? ds->sm_count : std::max(1, (4 * ds->sm_count) / ((R + 63) / 64));
    while (C > 1 && scratch_need(C, R, d.head_dim) > kScratchBytes) --C;
  }

  tt::Problem p{};
  p.mode = tt::kDecode;
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.g = g;
  p.D = d.head_dim;
  p.S = d.block_size;
  p.R = R;
  p.NB = 1;
  p.ctx_stride = d.ctx_capacity;
  const float scale = d.scale > 0.f ? d.scale : 1.0f / std::sqrt((float)d.head_dim);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_ctx = static_cast<const __nv_bfloat16*>(k_ctx);
  p.v_ctx = static_cast<const __nv_bfloat16*>(v_ctx);
  p.k_blk = static_cast<const __nv_bfloat16*>(k_blk);
  p.v_blk = static_cast<const __nv_bfloat16*>(v_blk);
  p.ctx_lens = ctx_lens;
  p.out = out;
  p.lse = lse;
  p.C = C;
  p.key_tile = key_tile;
  p.blk_tiles = tt::ceil_div(d.block_size, key_tile);
  unsigned char* w = ds->scratch;
  const size_t b_po = up256(size_t(2) * C * R * d.head_dim * sizeof(float));
  const size_t b_pl = up256(size_t(2) * C * R * sizeof(float));
  const size_t b_rec = up256(size_t(C) * sizeof(tt::SplitRecord));
  p.part_o = reinterpret_cast<float*>(w);
  p.part_lse = reinterpret_cast<float*>(w + b_po);
  p.records = reinterpret_cast<tt::SplitRecord*>(w + b_po + b_pl);
  p.err_word = status ? reinterpret_cast<unsigned*>(status) : reinterpret_cast<unsigned*>(w + b_po + b_pl + b_rec);
  p.wait_limit_ns = (unsigned long long)(d.wait_timeout_us > 0 ? d.wait_timeout_us : 1000000) * 1000ull;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The error word must start at zero; partials and records are written before they are read.
  e = cudaMemsetAsync(p.err_word, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return reject(TT_ERR_CUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));

  if (kernel == TT_KERNEL_TCGEN05) {
    tt::TmaMaps maps;
    memset(&maps, 0, sizeof(maps));
    const cuuint64_t D = d.head_dim;
    {
      cuuint64_t dims[3] = {D, (cuuint64_t)p.Hq, (cuuint64_t)p.B * p.S};
      cuuint64_t str[2] = {D * 2, (cuuint64_t)p.Hq * D * 2};
      cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)p.S};
      if (!encode(&maps.q, q, 3, dims, str, box)) return reject(TT_ERR_CUDA, "tensor map (q) encode failed");
    }
    {
      cuuint64_t dims[3] = {D, (cuuint64_t)p.Hkv, (cuuint64_t)p.B * p.S};
      cuuint64_t str[2] = {D * 2, (cuuint64_t)p.Hkv * D * 2};
      cuuint32_t box[3] = {64, 1, (cuuint32_t)std::min(p.S, key_tile)};
      if (!encode(&maps.k_blk, k_blk, 3, dims, str, box) || !encode(&maps.v_blk, v_blk, 3, dims, str, box))
        return reject(TT_ERR_CUDA, "tensor map (block kv) encode failed");
    }
    if ((long long)p.B * p.Hkv * p.ctx_stride > 0) {
      cuuint64_t dims[2] = {D, (cuuint64_t)p.B * p.Hkv * p.ctx_stride};
      cuuint64_t str[1] = {D * 2};
      cuuint32_t box[2] = {64, (cuuint32_t)key_tile};
      if (!encode(&maps.k_ctx, k_ctx, 2, dims, str, box) || !encode(&maps.v_ctx, v_ctx, 2, dims, str, box))
        return reject(TT_ERR_CUDA, "tensor map (context kv) encode failed");
    } else {
      maps.k_ctx = maps.k_blk;
      maps.v_ctx = maps.v_blk;
    }
    e = tt::launch_attn_tcgen05(p, maps, s);
  } else {
    e = tt::launch_attn_mma_sync(p, s);
  }
  if (e != cudaSuccess) return reject(TT_ERR_CUDA, std::string("attention kernel launch: ") + cudaGetErrorString(e));
  if (C > 1) {
    e = tt::launch_combine(p, s);
    if (e != cudaSuccess) return reject(TT_ERR_CUDA, std::string("combine kernel launch: ") + cudaGetErrorString(e));
  }
  return TT_OK;
}
