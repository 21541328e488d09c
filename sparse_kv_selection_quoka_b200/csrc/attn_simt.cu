// Sparse GQA attention on the CUDA cores, in fp32.
//
// [QUOKA §4.2, problem 3] the selected KV is the attention's input, with no
// causal mask over it; the chunk's own keys follow causally:
//   O[b,h,t] = sum_k softmax_k(scale * q . k) v,
//   k over {K[b, j, kv_idx[b, j, n]] : n < kv_count[b, j]} U {Kc[b, j, s] : s <= t},
//   j = floor(h / G).
// Flash-style online softmax in fp32 (exp2 with log2(e) folded into the
// scale). This variant serves the fp32 inputs (whose tolerance needs fp32
// products) and cross-checks the tensor-core variant in the tests.
#include "common.cuh"
#include "kernels.h"

namespace quoka {

constexpr int AS_ROWS = 32;  // query rows per CTA
constexpr int AS_TPR = 4;    // threads per row (each owns d / 4 columns)
constexpr int AS_THREADS = AS_ROWS * AS_TPR;
constexpr int AS_KT = 32;    // keys per shared-memory tile

template <typename T, int D>
__global__ void __launch_bounds__(AS_THREADS)
attn_simt_kernel(AttnArgs a) {
  constexpr int DP = D / AS_TPR;  // columns per thread
  constexpr int LD = AS_TPR * (DP + 1);  // padded row: the 4 column groups hit distinct banks
  __shared__ float ks[AS_KT][LD];
  __shared__ float vs[AS_KT][LD];
  __shared__ int kvis[AS_KT];  // chunk position of the key (or -1 for a selected key), -2 = skip

  const int h = blockIdx.y, bi = blockIdx.z;
  const int G = a.nq / a.nkv, j = h / G;
  const int t0 = blockIdx.x * AS_ROWS;
  const int r = threadIdx.x / AS_TPR, part = threadIdx.x % AS_TPR;
  const int t = t0 + r;
  const bool row_ok = t < a.BCP;
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int nsel = a.bsa > 0 ? max(0, min(a.kv_count[kvrow], a.bsa)) : 0;
  const int nchunk = a.no_chunk ? 0 : min(a.BCP, t0 + AS_ROWS);
  const int total = nsel + nchunk;

  const float qscale = a.scale * 1.4426950408889634f;  // log2(e)
  float q[DP], o[DP];
  {
    const T* qp = static_cast<const T*>(a.Q.data) + bi * a.Q.sb + h * a.Q.sh +
                  (int64_t)(row_ok ? t : 0) * a.Q.st + part * DP;
#pragma unroll
    for (int k = 0; k < DP; ++k) {
      q[k] = to_f32(qp[k]) * qscale;
      o[k] = 0.f;
    }
  }
  float m = -INFINITY, l = 0.f;

  const T* Kb = static_cast<const T*>(a.K.data) + bi * a.K.sb + j * a.K.sh;
  const T* Vb = static_cast<const T*>(a.V.data) + bi * a.V.sb + j * a.V.sh;
  const T* Kcb = static_cast<const T*>(a.Kc.data) + bi * a.Kc.sb + j * a.Kc.sh;
  const T* Vcb = static_cast<const T*>(a.Vc.data) + bi * a.Vc.sb + j * a.Vc.sh;
  // no index list: the selected rows are already gathered (row n = key n)
  const int32_t* idx = a.kv_idx != nullptr ? a.kv_idx + kvrow * a.bsa : nullptr;

  for (int kb = 0; kb < total; kb += AS_KT) {
    __syncthreads();
    if (threadIdx.x < AS_KT) {
      const int n = kb + threadIdx.x;
      int vis = -2;
      if (n < nsel) {
        const int32_t tau = idx != nullptr ? idx[n] : n;
        if (tau >= 0 && (int64_t)tau < a.T) vis = -1;
        else latch_status(a.status, 6 /* QUOKA_ERR_BOUNDS */);
      } else if (n < total) {
        vis = n - nsel;
      }
      kvis[threadIdx.x] = vis;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < AS_KT * D; e += AS_THREADS) {
      const int kr = e / D, c = e % D;
      const int n = kb + kr;
      const int vis = kvis[kr];
      float kv = 0.f, vv = 0.f;
      if (vis == -1) {
        const int64_t tau = idx != nullptr ? idx[n] : n;
        kv = to_f32(Kb[tau * a.K.st + c]);
        vv = to_f32(Vb[tau * a.V.st + c]);
      } else if (vis >= 0) {
        kv = to_f32(Kcb[(int64_t)vis * a.Kc.st + c]);
        vv = to_f32(Vcb[(int64_t)vis * a.Vc.st + c]);
      }
      const int col = (c / DP) * (DP + 1) + (c % DP);
      ks[kr][col] = kv;
      vs[kr][col] = vv;
    }
    __syncthreads();
    const int kmax = min(AS_KT, total - kb);
    for (int kk = 0; kk < kmax; ++kk) {
      const float* kr = &ks[kk][part * (DP + 1)];
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < DP; ++k) s += q[k] * kr[k];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      const int vis = kvis[kk];
      const bool visible = (vis == -1) || (vis >= 0 && vis <= t);
      if (!visible) continue;
      const float m_new = fmaxf(m, s);
      const float corr = exp2f(m - m_new);
      const float p = exp2f(s - m_new);
      l = l * corr + p;
      const float* vr = &vs[kk][part * (DP + 1)];
#pragma unroll
      for (int k = 0; k < DP; ++k) o[k] = o[k] * corr + p * vr[k];
      m = m_new;
    }
  }
  if (!row_ok) return;
  const float inv = l > 0.f ? 1.f / l : 0.f;  // no visible key: O = 0, lse = -inf
  T* op = static_cast<T*>(a.O) + (((int64_t)bi * a.nq + h) * a.BCP + t) * D + part * DP;
#pragma unroll
  for (int k = 0; k < DP; ++k) op[k] = from_f32<T>(o[k] * inv);
  if (a.lse != nullptr && part == 0)
    a.lse[((int64_t)bi * a.nq + h) * a.BCP + t] = (m + log2f(l)) * 0.6931471805599453f;
}

cudaError_t launch_attn_simt(bool is_bf16, const AttnArgs& a, cudaStream_t stream) {
  dim3 grid((a.BCP + AS_ROWS - 1) / AS_ROWS, a.nq, a.b);
  if (is_bf16) {
    if (a.d == 128) attn_simt_kernel<bf16, 128><<<grid, AS_THREADS, 0, stream>>>(a);
    else if (a.d == 64) attn_simt_kernel<bf16, 64><<<grid, AS_THREADS, 0, stream>>>(a);
    else return cudaErrorNotSupported;
  } else {
    if (a.d == 128) attn_simt_kernel<float, 128><<<grid, AS_THREADS, 0, stream>>>(a);
    else if (a.d == 64) attn_simt_kernel<float, 64><<<grid, AS_THREADS, 0, stream>>>(a);
    else return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace quoka
