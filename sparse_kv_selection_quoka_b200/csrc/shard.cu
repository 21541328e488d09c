// Pieces of the context-parallel step: the prior keys (T) are split over
// ranks; each rank runs steps (a)-(e) on its shard and the exact global
// top-BSA is taken over the ranks' candidates; each rank then attends over
// its share of the selection and the partial results are merged by their
// log-sum-exp. (The QUOKA write-up, "QUOKA: how it reshapes LLM prefill
// efficiency", bqwf.cn news item 915859, describes one device; this is the
// split of its §2.3 top-k and §4.2 attention over devices.)
//
// Exactness of the merge: a key in the global top-BSA is in its own shard's
// top-BSA (fewer than BSA keys of the shard beat it), so the union of the
// shards' top-min(BSA, T_r) candidates holds the whole global selection.
// With the shards in rank order over the prior positions, ranking the
// concatenated candidates (rank-major, ascending positions within a rank)
// with ties to the lower list position breaks ties to the lower global key
// index, as the single-device select does.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "nvtx_range.h"
#include "quoka.h"

namespace quoka {

namespace {

constexpr int kShardThreads = 256;

// The candidate list of one rank, padded to the common length C: for
// n < kv_count[row] (<= Cl, the row length of kv_idx) cand = kv_idx[row, n]
// and scores = S_agg[row, cand]; beyond, cand = -1 and scores = -inf (such
// entries can never be picked over a real score).
__global__ void __launch_bounds__(kShardThreads)
candidate_scores_kernel(const float* __restrict__ s_agg, int64_t T, const int32_t* __restrict__ kv_idx,
                        const int32_t* __restrict__ kv_count, int Cl, int C, float* __restrict__ scores,
                        int32_t* __restrict__ cand, int* status) {
  const int64_t row = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
  const int n = blockIdx.x * kShardThreads + threadIdx.x;
  if (n >= C) return;
  const int cnt = max(0, min(kv_count[row], Cl));
  float v = -INFINITY;
  int32_t c = -1;
  if (n < cnt) {
    const int32_t tau = kv_idx[row * Cl + n];
    if (tau >= 0 && (int64_t)tau < T) {
      v = s_agg[row * T + tau];
      c = tau;
    } else if (status != nullptr) {
      latch_status(status, QUOKA_ERR_BOUNDS);
    }
  }
  scores[row * C + n] = v;
  cand[row * C + n] = c;
}

// out[row, r, :] = in[r, row, :]: the all-gathered (rank, row, C) lists
// into rank-major rows (row, N * C), 32-bit elements.
__global__ void __launch_bounds__(kShardThreads)
interleave_kernel(const uint32_t* __restrict__ in, int N, int64_t rows, int64_t C, uint32_t* __restrict__ out) {
  const int64_t g = (int64_t)blockIdx.x * kShardThreads + threadIdx.x;
  const int64_t total = (int64_t)N * rows * C;
  if (g >= total) return;
  const int64_t c = g % C, rr = g / C;
  const int64_t row = rr % rows, r = rr / rows;
  out[(row * N + r) * C + c] = in[g];
}

// One CTA per (batch, KV head): the global selection `pos` (ascending
// positions into the ranks' concatenated candidate lists, S of them) keeps
// the positions of rank `rank`'s list, [rank * C, (rank + 1) * C), mapped
// back to this rank's key indices through its candidate list `cand`.
__global__ void __launch_bounds__(kShardThreads)
take_shard_kernel(const int32_t* __restrict__ pos, const int32_t* __restrict__ pos_count, int S,
                  const int32_t* __restrict__ cand, int C, int rank, int32_t* __restrict__ out_idx,
                  int32_t* __restrict__ out_count, int* status) {
  __shared__ int lo_s, hi_s;
  const int64_t row = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
  const int n = max(0, min(pos_count[row], S));
  const int64_t first = (int64_t)rank * C, last = first + C;
  if (threadIdx.x == 0) {
    lo_s = 0;
    hi_s = 0;
  }
  __syncthreads();
  int lo = 0, hi = 0;  // entries below `first`, below `last`
  for (int e = threadIdx.x; e < n; e += kShardThreads) {
    const int32_t p = pos[row * S + e];
    lo += p < first;
    hi += p < last;
  }
  if (lo) atomicAdd(&lo_s, lo);
  if (hi) atomicAdd(&hi_s, hi);
  __syncthreads();
  lo = lo_s;
  hi = hi_s;
  for (int e = lo + threadIdx.x; e < hi; e += kShardThreads) {
    const int32_t p = pos[row * S + e];
    int32_t tau = -1;
    if (p >= first && p < last) tau = cand[row * C + (p - first)];
    if (tau < 0 && status != nullptr) latch_status(status, QUOKA_ERR_BOUNDS);
    out_idx[row * C + (e - lo)] = tau < 0 ? 0 : tau;
  }
  if (threadIdx.x == 0) out_count[row] = hi - lo;
}

// O = sum_r w_r O_r with w_r = exp(lse_r - LSE), LSE = log sum_r exp(lse_r):
// the softmax over the union of the ranks' key sets, from each rank's
// softmax over its own. Rows every rank saw empty (all lse = -inf) give
// O = 0 and LSE = -inf. One thread per (row, 8 consecutive elements).
template <typename T>
__global__ void __launch_bounds__(kShardThreads)
combine_kernel(const T* __restrict__ O_parts, const float* __restrict__ lse_parts, int N, int64_t rows, int d,
               T* __restrict__ O, float* __restrict__ lse) {
  const int per_row = d / 8;
  const int64_t g = (int64_t)blockIdx.x * kShardThreads + threadIdx.x;
  if (g >= rows * per_row) return;
  const int64_t row = g / per_row;
  const int c0 = (int)(g % per_row) * 8;
  float M = -INFINITY;
  for (int r = 0; r < N; ++r) M = fmaxf(M, lse_parts[(int64_t)r * rows + row]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float L = 0.f;
  if (M != -INFINITY) {
    for (int r = 0; r < N; ++r) {
      const float lr = lse_parts[(int64_t)r * rows + row];
      if (lr == -INFINITY) continue;
      const float w = expf(lr - M);
      L += w;
      const T* src = O_parts + ((int64_t)r * rows + row) * d + c0;
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] += w * to_f32(src[u]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* dst = O + row * d + c0;
#pragma unroll
  for (int u = 0; u < 8; ++u) dst[u] = from_f32<T>(acc[u] * inv);
  if (c0 == 0 && lse != nullptr) lse[row] = L > 0.f ? M + logf(L) : -INFINITY;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

quoka_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QUOKA_OK : QUOKA_ERR_CUDA; }

// The status word at the start of a caller's workspace (256-byte aligned,
// at least 8 bytes), cleared on the stream; null when no workspace is given.
quoka_status status_word(void* ws, size_t ws_bytes, cudaStream_t cs, int** status) {
  *status = nullptr;
  if (ws == nullptr) return QUOKA_OK;
  if (!aligned(ws, 256) || ws_bytes < 2 * sizeof(int)) return QUOKA_ERR_WORKSPACE;
  *status = static_cast<int*>(ws);
  return cudaMemsetAsync(*status, 0, 2 * sizeof(int), cs) == cudaSuccess ? QUOKA_OK : QUOKA_ERR_CUDA;
}

}  // namespace

}  // namespace quoka

extern "C" {

quoka_status quoka_shard_candidate_scores(const float* s_agg, int b, int nkv, int64_t T, const int32_t* kv_idx,
                                          const int32_t* kv_count, int Cl, int C, float* scores,
                                          int32_t* cand_idx, void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_shard_candidate_scores");
  if (b < 1 || nkv < 1 || b > 65535 || nkv > 65535 || T < 0 || Cl < 0 || C < Cl || kv_count == nullptr)
    return QUOKA_ERR_INVALID_ARG;
  if (C == 0) return QUOKA_OK;
  if (scores == nullptr || cand_idx == nullptr || (Cl > 0 && (s_agg == nullptr || kv_idx == nullptr)))
    return QUOKA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = nullptr;
  quoka_status st = quoka::status_word(ws, ws_bytes, cs, &status);
  if (st != QUOKA_OK) return st;
  dim3 grid((unsigned)((C + quoka::kShardThreads - 1) / quoka::kShardThreads), nkv, b);
  quoka::candidate_scores_kernel<<<grid, quoka::kShardThreads, 0, cs>>>(s_agg, T, kv_idx, kv_count, Cl, C, scores,
                                                                         cand_idx, status);
  return quoka::from_cuda(cudaGetLastError());
}

quoka_status quoka_shard_interleave(const void* in, int N, int64_t rows, int64_t C, void* out, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_shard_interleave");
  if (N < 1 || rows < 0 || C < 0) return QUOKA_ERR_INVALID_ARG;
  const int64_t total = (int64_t)N * rows * C;
  if (total == 0) return QUOKA_OK;
  if (in == nullptr || out == nullptr || !quoka::aligned(in, 4) || !quoka::aligned(out, 4))
    return QUOKA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)((total + quoka::kShardThreads - 1) / quoka::kShardThreads);
  quoka::interleave_kernel<<<grid, quoka::kShardThreads, 0, cs>>>(static_cast<const uint32_t*>(in), N, rows, C,
                                                                  static_cast<uint32_t*>(out));
  return quoka::from_cuda(cudaGetLastError());
}

quoka_status quoka_topk(const float* scores, int b, int nkv, int64_t T, int BSA, int32_t* kv_idx,
                        int32_t* kv_count, void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_topk");
  if (b < 1 || nkv < 1 || b > 65535 || nkv > 65535 || T < 0 || BSA < 0 || kv_count == nullptr)
    return QUOKA_ERR_INVALID_ARG;
  const int64_t bsa_eff = BSA < T ? BSA : T;
  if (bsa_eff > 0 && (scores == nullptr || kv_idx == nullptr)) return QUOKA_ERR_INVALID_ARG;
  if (T > quoka::topk_max_T()) return QUOKA_ERR_UNSUPPORTED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = nullptr;
  quoka_status st = quoka::status_word(ws, ws_bytes, cs, &status);
  if (st != QUOKA_OK) return st;
  if (bsa_eff == 0)
    return quoka::from_cuda(cudaMemsetAsync(kv_count, 0, sizeof(int32_t) * (size_t)b * nkv, cs));
  return quoka::from_cuda(
      quoka::launch_topk(scores, b, nkv, T, (int)bsa_eff, nullptr, kv_idx, kv_count, status, false, cs));
}

quoka_status quoka_shard_take(const int32_t* sel_pos, const int32_t* sel_count, int b, int nkv, int S,
                              const int32_t* cand_idx, int C, int rank, int32_t* kv_idx, int32_t* kv_count,
                              void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_shard_take");
  if (b < 1 || nkv < 1 || b > 65535 || nkv > 65535 || S < 0 || C < 0 || rank < 0 || sel_count == nullptr ||
      kv_count == nullptr)
    return QUOKA_ERR_INVALID_ARG;
  if ((S > 0 && sel_pos == nullptr) || (C > 0 && (cand_idx == nullptr || kv_idx == nullptr)))
    return QUOKA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = nullptr;
  quoka_status st = quoka::status_word(ws, ws_bytes, cs, &status);
  if (st != QUOKA_OK) return st;
  if (C == 0 || S == 0)
    return quoka::from_cuda(cudaMemsetAsync(kv_count, 0, sizeof(int32_t) * (size_t)b * nkv, cs));
  dim3 grid(1, nkv, b);
  quoka::take_shard_kernel<<<grid, quoka::kShardThreads, 0, cs>>>(sel_pos, sel_count, S, cand_idx, C, rank, kv_idx,
                                                                   kv_count, status);
  return quoka::from_cuda(cudaGetLastError());
}

quoka_status quoka_combine_partials(const void* O_parts, const float* lse_parts, int N, int b, int nq, int BCP,
                                    int d, quoka_dtype dtype, void* O, float* lse, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_combine_partials");
  if (N < 1 || b < 1 || nq < 1 || BCP < 1 || (d != 64 && d != 128)) return QUOKA_ERR_INVALID_ARG;
  if (dtype != QUOKA_F32 && dtype != QUOKA_BF16) return QUOKA_ERR_INVALID_ARG;
  if (O_parts == nullptr || lse_parts == nullptr || O == nullptr) return QUOKA_ERR_INVALID_ARG;
  if (!quoka::aligned(O_parts, 16) || !quoka::aligned(O, 16)) return QUOKA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int64_t rows = (int64_t)b * nq * BCP;
  const int64_t work = rows * (d / 8);
  const unsigned grid = (unsigned)((work + quoka::kShardThreads - 1) / quoka::kShardThreads);
  if (dtype == QUOKA_BF16)
    quoka::combine_kernel<__nv_bfloat16><<<grid, quoka::kShardThreads, 0, cs>>>(
        static_cast<const __nv_bfloat16*>(O_parts), lse_parts, N, rows, d, static_cast<__nv_bfloat16*>(O), lse);
  else
    quoka::combine_kernel<float><<<grid, quoka::kShardThreads, 0, cs>>>(static_cast<const float*>(O_parts),
                                                                        lse_parts, N, rows, d,
                                                                        static_cast<float*>(O), lse);
  return quoka::from_cuda(cudaGetLastError());
}

}  // extern "C"
