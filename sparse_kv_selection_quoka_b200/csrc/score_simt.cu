// Key scoring on the CUDA cores, in fp32.
//
// [QUOKA §2.2] cosine score, [QUOKA §2.3] S = Q_group . K_norm^T reduced by a
// max over the NQ chosen queries:
//   S_agg[b, j, tau] = max_i (Q_group[b, j, i] . K[b, j, tau]) / |K[b, j, tau]|
// (the max commutes with the positive 1/|k| factor, so the key is divided
// once, after the max). This variant serves fp32 inputs, where the fp32
// tolerance needs fp32 products; bf16 inputs use the tensor-core variant.
#include "common.cuh"
#include "kernels.h"

namespace quoka {

constexpr int SCORE_SIMT_THREADS = 128;

// One thread per key: the key row is held in registers (fp32), the NQ x D
// group queries in shared memory (read as broadcasts).
template <typename T, int D>
__global__ void __launch_bounds__(SCORE_SIMT_THREADS)
score_simt_kernel(const T* __restrict__ K, int64_t sKb, int64_t sKh, int64_t sKt, int64_t Tlen,
                  const float* __restrict__ Qg, int NQ, float* __restrict__ S_agg, int key_norm) {
  extern __shared__ float4 qs4[];
  const int j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  const int64_t row = (int64_t)bi * nkv + j;
  const float4* src = reinterpret_cast<const float4*>(Qg + row * NQ * D);
  for (int e = threadIdx.x; e < NQ * D / 4; e += SCORE_SIMT_THREADS) qs4[e] = src[e];
  __syncthreads();

  const int64_t tau = (int64_t)blockIdx.x * SCORE_SIMT_THREADS + threadIdx.x;
  if (tau >= Tlen) return;
  const T* kr = K + bi * sKb + j * sKh + tau * sKt;
  float k[D];
#pragma unroll
  for (int c = 0; c < D; c += 8) {
    float v[8];
    load8(kr + c, v);
#pragma unroll
    for (int u = 0; u < 8; ++u) k[c + u] = v[u];
  }
  float kk = 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) kk += k[c] * k[c];

  float best = -INFINITY;
  for (int i = 0; i < NQ; ++i) {
    const float4* q = qs4 + i * (D / 4);
    float dot = 0.f;
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
      const float4 w = q[c];
      dot += w.x * k[4 * c] + w.y * k[4 * c + 1] + w.z * k[4 * c + 2] + w.w * k[4 * c + 3];
    }
    best = fmaxf(best, dot);
  }
  S_agg[row * Tlen + tau] = key_norm ? best / fmaxf(sqrtf(kk), 1e-12f) : best;
}

template <typename T, int D>
static cudaError_t score_typed(Strided K, int b, int nkv, int64_t T_len, const float* Qg, int NQ,
                               float* S_agg, bool key_norm, cudaStream_t stream) {
  const size_t smem = (size_t)NQ * D * sizeof(float);
  auto kern = score_simt_kernel<T, D>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)((T_len + SCORE_SIMT_THREADS - 1) / SCORE_SIMT_THREADS), nkv, b);
  kern<<<grid, SCORE_SIMT_THREADS, smem, stream>>>(static_cast<const T*>(K.data), K.sb, K.sh, K.st,
                                                   T_len, Qg, NQ, S_agg, (int)key_norm);
  return cudaGetLastError();
}

cudaError_t launch_score_simt(bool is_bf16, int d, Strided K, int b, int nkv, int64_t T_len,
                              const float* Qg, int NQ, float* S_agg, bool key_norm, cudaStream_t stream) {
  if (T_len == 0) return cudaSuccess;
  if (is_bf16) {
    if (d == 128) return score_typed<bf16, 128>(K, b, nkv, T_len, Qg, NQ, S_agg, key_norm, stream);
    if (d == 64) return score_typed<bf16, 64>(K, b, nkv, T_len, Qg, NQ, S_agg, key_norm, stream);
  } else {
    if (d == 128) return score_typed<float, 128>(K, b, nkv, T_len, Qg, NQ, S_agg, key_norm, stream);
    if (d == 64) return score_typed<float, 64>(K, b, nkv, T_len, Qg, NQ, S_agg, key_norm, stream);
  }
  return cudaErrorNotSupported;
}

}  // namespace quoka
