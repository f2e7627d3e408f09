// Log-sum-exp combine of the units that a range boundary cut into segments
// (combine_row.cuh: one warp per row), and the bounded-wait self test.
#include "combine_row.cuh"
#include "problem.h"
#include "ptx.cuh"
#include "walker.cuh"

namespace tt {
namespace {

constexpr int kRowsPerBlock = 8;   // one warp per row
constexpr int kThreads = 256;

template <int D>
__global__ void __launch_bounds__(kThreads) combine_kernel(const Problem p) {
  // launched as a programmatic dependent of the attention kernel: wait until its grid has
  // completed and its partials are visible; the next call's attention kernel may be scheduled
  // meanwhile and waits for this grid itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int c = blockIdx.x;
  const SplitRecord rec = p.records[c];
  if (rec.unit < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * kRowsPerBlock + warp;
  if (r >= p.R) return;
  combine_row<D>(p, c, rec, r, lane);
}

// One thread waits on a barrier that nothing arrives at; the bounded wait must
// give up, raise kErrTimeout and return.
__global__ void wait_selftest_kernel(unsigned* err_word, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx w{&abort_flag, err_word, limit_ns};
    if (mbar_wait(smem_u32(&bar), 0, w)) atomicOr(err_word, 0x80000000u);  // must not happen
  }
  __syncthreads();
}

// The FMA-pipe exp2 of the softmax (ptx.cuh: exp2_poly2) on n arguments.
__global__ void exp2_selftest_kernel(const float* x, float* y, int n) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
  if (i + 1 < n) {
    const float2 e = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = e.x;
    y[i + 1] = e.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

}  // namespace

cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t stream) {
  exp2_selftest_kernel<<<(n + 511) / 512, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_combine(const Problem& p, cudaStream_t stream) {
  // a programmatic dependent launch: the launch overlaps the attention kernel's tail and the
  // kernel waits for the attention grid on the device
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.C, (p.R + kRowsPerBlock - 1) / kRowsPerBlock, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.D == 128) return cudaLaunchKernelEx(&cfg, combine_kernel<128>, p);
  return cudaLaunchKernelEx(&cfg, combine_kernel<64>, p);
}

cudaError_t launch_wait_selftest(unsigned* err_word, unsigned long long limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(err_word, limit_ns);
  return cudaGetLastError();
}

}  // namespace tt
