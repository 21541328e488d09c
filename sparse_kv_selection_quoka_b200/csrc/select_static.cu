// quoka_select_static: the key-selection step for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain scratch memory: a plugin hosted by a
// framework whose own allocator owns all device memory and forbids raw
// cudaMalloc, or code on a latency-critical path where cudaMalloc (which can
// synchronise the device) is not acceptable. This entry point runs the same
// kernels as quoka_select but takes its scratch from a fixed, file-scope
// device array instead of a caller-supplied workspace, so the caller passes
// only inputs and outputs and nothing is allocated per call.
//
// The array is QUOKA_STATIC_SCRATCH_BYTES (8 MiB) per device; every GPU that
// loads this library keeps it until the process exits. All calls on a device
// share it, so calls that overlap on the GPU (different streams without
// ordering between them) race on it; callers must order them.
#include <cuda_runtime.h>

#include "nvtx_range.h"
#include "quoka.h"

namespace {

__device__ __align__(256) unsigned char g_select_scratch[QUOKA_STATIC_SCRATCH_BYTES];

}  // namespace

namespace quoka {

// Device address of g_select_scratch in the current context. In host code
// the symbol name is only a host-side stand-in; the runtime resolves it for
// the context current at the call, so the address is looked up on every
// call rather than cached (a cached address would go stale after
// cudaDeviceReset or under another context on the same device).
quoka_status static_scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return QUOKA_ERR_CUDA;
  *out = p;
  return QUOKA_OK;
}

}  // namespace quoka

extern "C" quoka_status quoka_select_static(const quoka_tensor* Q, const quoka_tensor* K, int NQ,
                                            int BSA, int32_t* kv_idx, int32_t* kv_count,
                                            int32_t* q_idx, float* s_agg, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_select_static");
  if (Q == nullptr || K == nullptr) return QUOKA_ERR_INVALID_ARG;
  const size_t need = quoka_select_workspace_size((int)Q->shape[0], (int)Q->shape[1], (int)K->shape[1],
                                           (int)Q->shape[3], K->shape[2], (int)Q->shape[2], NQ, BSA,
                                           Q->dtype);
  if (need == 0) return QUOKA_ERR_INVALID_ARG;
  if (need > (size_t)QUOKA_STATIC_SCRATCH_BYTES) return QUOKA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const quoka_status st = quoka::static_scratch_address(&scratch);
  if (st != QUOKA_OK) return st;
  // quoka_select's first kernel clears the scratch's status words; every
  // other scratch region is fully written before it is read, so the previous
  // call's contents never leak into this one.
  return quoka_select(Q, K, NQ, BSA, kv_idx, kv_count, q_idx, s_agg, scratch,
                      (size_t)QUOKA_STATIC_SCRATCH_BYTES, stream);
}
