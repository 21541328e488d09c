// Sparse GQA attention on the tcgen05 tensor cores (placeholder until the kernel lands).
#include "kernels.h"

namespace quoka {

cudaError_t launch_attn_tc(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace quoka
