// Gather of the selected K/V rows into contiguous buffers.
//
// [QUOKA §4.2, problem 3] the selected KV becomes the attention's input KV:
//   Ksel[b, j, n] = K[b, j, kv_idx[b, j, n]],  Vsel likewise, n < kv_count[b, j].
// Serves quoka_gather_kv, and the tensor-core attention, which then streams
// the selected keys as dense TMA tiles: the copy (b * nkv * BSA rows of K and
// V) is written just before the attention runs and stays in the 126 MB L2.
//
// The work is HBM-bound row traffic, so the kernel is plain vector copies
// with many 16-byte loads in flight per thread: each thread copies kItems
// (row, 16-byte chunk) items of K and of V, all loads issued before the
// stores. Consecutive threads cover consecutive chunks of one row, so each
// row is one coalesced 128/256/512-byte read.
#include "common.cuh"
#include "kernels.h"

namespace quoka {

namespace {

constexpr int kThreads = 256;
constexpr int kItems = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// grid (ceil(bsa * cpr / (kThreads * kItems)), nkv, b); strides in bytes.
// Rows n in [kv_count, bsa), and rows with an index outside [0, T), are
// written as zeros: the attention reads whole 128-row tiles and masks those
// rows in the softmax, so they must hold finite values.
__global__ void __launch_bounds__(kThreads)
gather_kernel(const char* __restrict__ K, int64_t sKb, int64_t sKh, int64_t sKt,
              const char* __restrict__ V, int64_t sVb, int64_t sVh, int64_t sVt, int64_t T,
              const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_count, int bsa,
              int cpr_log2, char* __restrict__ Ksel, char* __restrict__ Vsel, int* status) {
  const int j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  const int64_t row = (int64_t)bi * nkv + j;
  pdl_trigger();  // the attention may launch once every CTA has started
  pdl_wait();     // the indices may come from the previous kernel
  const int64_t nitems = (int64_t)bsa << cpr_log2;
  const int64_t i0 = (int64_t)blockIdx.x * (kThreads * kItems) + threadIdx.x;
  const int cmask = (1 << cpr_log2) - 1;
  const int row_bytes = 16 << cpr_log2;
  // The count and every item's index are loaded together (L2-coherent
  // loads: possibly written by the previous kernel); an index past the
  // count is read (the list has bsa entries per row) but not used.
  const int cnt_raw = __ldcg(kv_count + row);
  int32_t tau_u[kItems];
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    const int64_t i = i0 + u * kThreads;
    tau_u[u] = i < nitems ? __ldcg(kv_idx + row * bsa + (int)(i >> cpr_log2)) : -1;
  }
  const int cnt = max(0, min(cnt_raw, bsa));
  const char* Kb = K + bi * sKb + j * sKh;
  const char* Vb = V + bi * sVb + j * sVh;
  char* Kd = Ksel + row * bsa * row_bytes;
  char* Vd = Vsel + row * bsa * row_bytes;
  uint4 kv[kItems], vv[kItems];
  bool bad = false;
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    const int64_t i = i0 + u * kThreads;
    const int n = (int)(i >> cpr_log2);
    const int c = (int)(i & cmask);
    kv[u] = make_uint4(0, 0, 0, 0);
    vv[u] = kv[u];
    if (i >= nitems) continue;
    if (n < cnt) {
      const int32_t tau = tau_u[u];
      if (tau >= 0 && (int64_t)tau < T) {
        kv[u] = ld_stream(reinterpret_cast<const uint4*>(Kb + tau * sKt) + c);
        vv[u] = ld_stream(reinterpret_cast<const uint4*>(Vb + tau * sVt) + c);
      } else {
        bad = true;  // not read; written as zeros
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    const int64_t i = i0 + u * kThreads;
    if (i < nitems) {
      // plain stores: the copy is meant to stay in L2 for its reader
      reinterpret_cast<uint4*>(Kd)[i] = kv[u];
      reinterpret_cast<uint4*>(Vd)[i] = vv[u];
    }
  }
  if (bad && status != nullptr) latch_status(status, 6 /* QUOKA_ERR_BOUNDS */);
}

}  // namespace

cudaError_t launch_gather(bool is_bf16, int d, Strided K, Strided V, int b, int nkv, int64_t T,
                          const int32_t* kv_idx, const int32_t* kv_count, int bsa, void* Ksel,
                          void* Vsel, int* status, bool pdl, cudaStream_t stream) {
  if (bsa == 0) return cudaSuccess;
  const int es = is_bf16 ? 2 : 4;
  const int row_bytes = d * es;  // 128, 256 or 512
  int cpr_log2 = 0;
  while ((16 << cpr_log2) < row_bytes) ++cpr_log2;
  if ((16 << cpr_log2) != row_bytes) return cudaErrorNotSupported;
  const int64_t nitems = (int64_t)bsa << cpr_log2;
  const int64_t per_block = (int64_t)kThreads * kItems;
  dim3 grid((unsigned)((nitems + per_block - 1) / per_block), nkv, b);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  // the kernel reads nothing before its grid-dependency wait, so it may be
  // launched while its predecessor finishes
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gather_kernel, static_cast<const char*>(K.data), K.sb * es, K.sh * es,
                            K.st * es, static_cast<const char*>(V.data), V.sb * es, V.sh * es, V.st * es, T,
                            kv_idx, kv_count, bsa, cpr_log2, static_cast<char*>(Ksel), static_cast<char*>(Vsel),
                            status);
}

}  // namespace quoka
