// Standalone gather of the selected K/V rows.
//
// [QUOKA §4.2, problem 3] the selected KV becomes the attention's input KV:
//   Ksel[b, j, n] = K[b, j, kv_idx[b, j, n]],  Vsel likewise, n < kv_count[b, j].
// The fused attention kernels read the selected rows in place; this kernel
// serves callers that want the selected KV materialised (for example to hand
// it to another attention implementation).
#include "common.cuh"
#include "kernels.h"

namespace quoka {

constexpr int GATHER_WARPS = 8;

// One warp per selected row: the row is copied in 16-byte vectors.
__global__ void __launch_bounds__(GATHER_WARPS * 32)
gather_kernel(const char* __restrict__ K, int64_t sKb, int64_t sKh, int64_t sKt,
              const char* __restrict__ V, int64_t sVb, int64_t sVh, int64_t sVt, int64_t T,
              const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_count, int bsa,
              int row_bytes, char* __restrict__ Ksel, char* __restrict__ Vsel, int* status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = blockIdx.x * GATHER_WARPS + warp;
  const int j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  const int64_t row = (int64_t)bi * nkv + j;
  const int cnt = min(kv_count[row], bsa);
  if (n >= cnt) return;
  const int32_t tau = kv_idx[row * bsa + n];
  if (tau < 0 || (int64_t)tau >= T) {
    if (lane == 0) latch_status(status, 6 /* QUOKA_ERR_BOUNDS */);
    return;
  }
  // strides are in bytes here
  const uint4* ks = reinterpret_cast<const uint4*>(K + bi * sKb + j * sKh + tau * sKt);
  const uint4* vs = reinterpret_cast<const uint4*>(V + bi * sVb + j * sVh + tau * sVt);
  uint4* kd = reinterpret_cast<uint4*>(Ksel + (row * bsa + n) * row_bytes);
  uint4* vd = reinterpret_cast<uint4*>(Vsel + (row * bsa + n) * row_bytes);
  const int nvec = row_bytes / 16;
  for (int v = lane; v < nvec; v += 32) {
    kd[v] = __ldg(ks + v);
    vd[v] = __ldg(vs + v);
  }
}

cudaError_t launch_gather(bool is_bf16, int d, Strided K, Strided V, int b, int nkv, int64_t T,
                          const int32_t* kv_idx, const int32_t* kv_count, int bsa, void* Ksel,
                          void* Vsel, int* status, cudaStream_t stream) {
  if (bsa == 0) return cudaSuccess;
  const int es = is_bf16 ? 2 : 4;
  dim3 grid((bsa + GATHER_WARPS - 1) / GATHER_WARPS, nkv, b);
  gather_kernel<<<grid, GATHER_WARPS * 32, 0, stream>>>(
      static_cast<const char*>(K.data), K.sb * es, K.sh * es, K.st * es,
      static_cast<const char*>(V.data), V.sb * es, V.sh * es, V.st * es, T, kv_idx, kv_count, bsa,
      d * es, static_cast<char*>(Ksel), static_cast<char*>(Vsel), status);
  return cudaGetLastError();
}

}  // namespace quoka
