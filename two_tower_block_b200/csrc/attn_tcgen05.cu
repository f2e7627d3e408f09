// placeholder until the tcgen05 kernel lands
#include "problem.h"
namespace tt {
size_t attn_tcgen05_smem_bytes(int) { return 0; }
cudaError_t launch_attn_tcgen05(const Problem&, const TmaMaps&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace tt
