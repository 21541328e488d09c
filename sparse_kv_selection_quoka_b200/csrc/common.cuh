// Device helpers shared by the QUOKA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace quoka {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Load 8 consecutive elements (one 16-byte vector for bf16, two for fp32)
// of a row into fp32 registers. `p` must be 16-byte aligned.
__device__ __forceinline__ void load8(const bf16* p, float (&v)[8]) {
  uint4 raw = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Order-preserving map from an fp32 score to an unsigned key: a < b as
// floats iff key(a) < key(b). -0 is folded onto +0 so equal scores give
// equal keys.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Programmatic dependent launch: a kernel launched with the programmatic
// stream serialisation attribute may start while its predecessor in the
// stream still runs; pdl_wait() blocks the calling thread until the
// predecessor grid has completed and its memory is visible (a no-op for a
// normal launch). pdl_trigger() lets the dependent grid launch once every
// CTA of this grid has called it or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Latch the first device-side fault of a call into the workspace status
// word (0 = no fault). Later faults keep the first code. The calls whose
// first kernel clears the status words (instead of a memset before the
// kernels) rely on this: the latch first waits for the predecessor grid
// (pdl_wait, a no-op without programmatic launch), and each kernel of such
// a call executes that wait before it completes, so every latch is ordered
// after the clearing. A latch happens only on a fault, so the wait costs
// nothing in a normal run.
__device__ __forceinline__ void latch_status(int* status, int code) {
  if (status == nullptr) return;
  pdl_wait();
  atomicCAS(status, 0, code);
}

// Record where the first device-side fault of a call happened (the word
// after the status word; diagnostic only). Ordered like latch_status.
__device__ __forceinline__ void latch_where(int* status, int where) {
  if (status == nullptr) return;
  pdl_wait();
  atomicCAS(status + 1, 0, where);
}

// Clear the two status words at the start of a call's first kernel (block
// 0, thread 0); see latch_status.
__device__ __forceinline__ void clear_status(int* status) {
  if (status != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
    status[0] = 0;
    status[1] = 0;
  }
}

// 12-bit bucket of a score, linear over [-1, 1] (cosine-type scores lie
// there): floor((s + 1) * 2048) clamped to [0, 4095]. Non-decreasing in the
// score's key order (every step rounds monotonically; a NaN goes to the end
// its key sorts to), so keys in a higher bucket are always larger.
__device__ __forceinline__ uint32_t score_bin(float s) {
  if (s != s) return (__float_as_uint(s) >> 31) ? 0u : 4095u;
  const float x = fminf(fmaxf((s + 1.f) * 2048.f, 0.f), 4095.f);
  return (uint32_t)x;
}

// The score an order-preserving key stands for (inverse of score_key).
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

}  // namespace quoka
