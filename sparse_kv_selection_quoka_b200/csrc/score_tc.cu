// Key scoring on the tcgen05 tensor cores (placeholder until the kernel lands).
#include "kernels.h"

namespace quoka {

cudaError_t launch_score_tc(int, Strided, int, int, int64_t, const uint16_t*, int, float*, int*,
                            cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace quoka
