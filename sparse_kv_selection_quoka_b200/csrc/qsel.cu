// Query subselection and GQA group mean.
//
// Three variants of the selection kernel compute the same thing: the cluster
// one (the default) spreads a head's rows over up to 8 CTAs that exchange
// partial results through distributed shared memory; the staged one copies a
// head's query block into one CTA's shared memory; the direct one reads
// global memory and serves chunks whose rows fit neither.
//
// [QUOKA §2.1, Algorithm 1] MQ = mean of the chunk's queries over its tokens;
// SQ = -cos(Q, MQ); the NQ queries with the largest SQ are kept, in rank
// order. [QUOKA §2.3] the kept queries are L2-normalised and averaged over
// the G query heads of each KV head, rank by rank.
//
// (QUOKA = the technical write-up "QUOKA: how it reshapes LLM prefill
// efficiency", bqwf.cn news item 915859; § numbers are the write-up's.)
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace quoka {

constexpr int QSEL_THREADS = 256;
constexpr int QSEL_WARPS = QSEL_THREADS / 32;

// One CTA per (query head, batch). Dynamic shared memory: SQ[BCP] floats
// followed by the rank -> position table sel[NQ].
template <typename T, int D>
__global__ void __launch_bounds__(QSEL_THREADS)
qsel_kernel(const T* __restrict__ Q, int64_t sQb, int64_t sQh, int64_t sQt, int BCP, int NQ,
            float* __restrict__ Qhat, int32_t* __restrict__ q_idx, int normalize) {
  extern __shared__ float smem[];
  float* SQ = smem;
  int* sel = reinterpret_cast<int*>(smem + BCP);
  __shared__ float part[QSEL_THREADS];
  __shared__ float mq[D];
  __shared__ float mq_norm;

  const int h = blockIdx.x, bi = blockIdx.y, nq = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* Qh = Q + bi * sQb + h * sQh;

  // (a) mean over the chunk's tokens: column c = tid % D, token groups of
  // QSEL_THREADS / D rows; partial sums combined in a fixed order.
  constexpr int NGRP = QSEL_THREADS / D;
  {
    const int c = tid % D, grp = tid / D;
    float acc = 0.f;
    for (int t = grp; t < BCP; t += NGRP) acc += to_f32(Qh[(int64_t)t * sQt + c]);
    part[tid] = acc;
  }
  for (int i = tid; i < NQ; i += QSEL_THREADS) sel[i] = 0;
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < NGRP; ++g) s += part[g * D + tid];
    mq[tid] = s / (float)BCP;
  }
  __syncthreads();
  if (warp == 0) {
    float s = 0.f;
    for (int k = lane; k < D; k += 32) s += mq[k] * mq[k];
    s = warp_sum(s);
    if (lane == 0) mq_norm = sqrtf(s);
  }
  __syncthreads();

  // (a) SQ[t] = -(q_t . MQ) / max(|q_t| |MQ|, 1e-8), one warp per token.
  for (int t = warp; t < BCP; t += QSEL_WARPS) {
    const T* q = Qh + (int64_t)t * sQt;
    float dot = 0.f, qq = 0.f;
#pragma unroll
    for (int k = lane; k < D; k += 32) {
      float v = to_f32(q[k]);
      dot += v * mq[k];
      qq += v * v;
    }
    dot = warp_sum(dot);
    qq = warp_sum(qq);
    if (lane == 0) SQ[t] = -dot / fmaxf(sqrtf(qq) * mq_norm, 1e-8f);
  }
  __syncthreads();

  // (b) rank of token t = number of tokens that beat it (larger SQ, or equal
  // SQ at a lower position); ranks below NQ are kept.
  for (int t = tid; t < BCP; t += QSEL_THREADS) {
    const float v = SQ[t];
    int r = 0;
    for (int u = 0; u < BCP; ++u) {
      const float w = SQ[u];
      r += (w > v) | ((w == v) & (u < t));
    }
    if (r < NQ) sel[r] = t;
  }
  __syncthreads();

  // (c) L2-normalise the kept queries: one warp per rank.
  for (int i = warp; i < NQ; i += QSEL_WARPS) {
    const int t = sel[i];
    const T* q = Qh + (int64_t)t * sQt;
    float v[D / 32];
    float qq = 0.f;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      v[k] = to_f32(q[lane + 32 * k]);
      qq += v[k] * v[k];
    }
    qq = warp_sum(qq);
    const float nrm = normalize ? fmaxf(sqrtf(qq), 1e-12f) : 1.f;
    float* dst = Qhat + (((int64_t)bi * nq + h) * NQ + i) * D;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) dst[lane + 32 * k] = v[k] / nrm;
    if (lane == 0 && q_idx != nullptr) q_idx[((int64_t)bi * nq + h) * NQ + i] = t;
  }
}

constexpr int QSEL_STAGED_THREADS = 512;
constexpr int QSEL_STAGED_WARPS = QSEL_STAGED_THREADS / 32;
constexpr size_t QSEL_STAGED_MAX_BYTES = 192 * 1024;

// The same computation with the head's whole (BCP, D) query block staged in
// shared memory first (16-byte vector loads, all in flight at once), so that
// the mean, the scores and the normalisation read shared memory. Dynamic
// shared memory: the block (row-major, element type T), SQ[BCP], sel[NQ].
template <typename T, int D>
__global__ void __launch_bounds__(QSEL_STAGED_THREADS)
qsel_staged_kernel(const T* __restrict__ Q, int64_t sQb, int64_t sQh, int64_t sQt, int BCP, int NQ,
                   float* __restrict__ Qhat, int32_t* __restrict__ q_idx, int normalize) {
  extern __shared__ __align__(16) uint8_t qs_raw[];
  T* blk = reinterpret_cast<T*>(qs_raw);
  const size_t blk_bytes = ((size_t)BCP * D * sizeof(T) + 15) & ~size_t(15);
  float* SQ = reinterpret_cast<float*>(qs_raw + blk_bytes);
  int* sel = reinterpret_cast<int*>(SQ + BCP);
  __shared__ float part[QSEL_STAGED_THREADS];
  __shared__ float mq[D];
  __shared__ float mq_norm;

  const int h = blockIdx.x, bi = blockIdx.y, nq = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* Qh = Q + bi * sQb + h * sQh;

  // stage: row t, 16-byte vector v of the row
  constexpr int VPR = D * (int)sizeof(T) / 16;  // vectors per row
#pragma unroll 8
  for (int e = tid; e < BCP * VPR; e += QSEL_STAGED_THREADS) {
    const int t = e / VPR, v = e % VPR;
    reinterpret_cast<uint4*>(blk + (size_t)t * D)[v] =
        __ldg(reinterpret_cast<const uint4*>(Qh + (int64_t)t * sQt) + v);
  }
  for (int i = tid; i < NQ; i += QSEL_STAGED_THREADS) sel[i] = 0;
  __syncthreads();

  // (a) mean over tokens: column c = tid % D, token groups of 512 / D rows
  constexpr int NGRP = QSEL_STAGED_THREADS / D;
  {
    const int c = tid % D, grp = tid / D;
    float acc = 0.f;
    for (int t = grp; t < BCP; t += NGRP) acc += to_f32(blk[(size_t)t * D + c]);
    part[tid] = acc;
  }
  __syncthreads();
  if (tid < D) {
    float sum = 0.f;
#pragma unroll
    for (int g = 0; g < NGRP; ++g) sum += part[g * D + tid];
    mq[tid] = sum / (float)BCP;
  }
  __syncthreads();
  if (warp == 0) {
    float sum = 0.f;
    for (int k = lane; k < D; k += 32) sum += mq[k] * mq[k];
    sum = warp_sum(sum);
    if (lane == 0) mq_norm = sqrtf(sum);
  }
  __syncthreads();

  // (a) SQ[t] = -(q_t . MQ) / max(|q_t| |MQ|, 1e-8), one warp per token
  for (int t = warp; t < BCP; t += QSEL_STAGED_WARPS) {
    const T* q = blk + (size_t)t * D;
    float dot = 0.f, qq = 0.f;
#pragma unroll
    for (int k = lane; k < D; k += 32) {
      const float v = to_f32(q[k]);
      dot += v * mq[k];
      qq += v * v;
    }
    dot = warp_sum(dot);
    qq = warp_sum(qq);
    if (lane == 0) SQ[t] = -dot / fmaxf(sqrtf(qq) * mq_norm, 1e-8f);
  }
  __syncthreads();

  // (b) rank of token t = number of tokens that beat it (larger SQ, or equal
  // SQ at a lower position)
  for (int t = tid; t < BCP; t += QSEL_STAGED_THREADS) {
    const float v = SQ[t];
    int r = 0;
    for (int u = 0; u < BCP; ++u) {
      const float w = SQ[u];
      r += (w > v) | ((w == v) & (u < t));
    }
    if (r < NQ) sel[r] = t;
  }
  __syncthreads();

  // (c) L2-normalise the kept queries, one warp per rank
  for (int i = warp; i < NQ; i += QSEL_STAGED_WARPS) {
    const int t = sel[i];
    const T* q = blk + (size_t)t * D;
    float v[D / 32];
    float qq = 0.f;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      v[k] = to_f32(q[lane + 32 * k]);
      qq += v[k] * v[k];
    }
    qq = warp_sum(qq);
    const float nrm = normalize ? fmaxf(sqrtf(qq), 1e-12f) : 1.f;
    float* dst = Qhat + (((int64_t)bi * nq + h) * NQ + i) * D;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) dst[lane + 32 * k] = v[k] / nrm;
    if (lane == 0 && q_idx != nullptr) q_idx[((int64_t)bi * nq + h) * NQ + i] = t;
  }
}

constexpr int QSEL_CL_THREADS = 512;
constexpr int QSEL_CL_WARPS = QSEL_CL_THREADS / 32;
constexpr int QSEL_CL_MAX = 8;

// Cluster variant (the default): one cluster of C CTAs per (query head,
// batch); CTA c owns rows [c*slice, (c+1)*slice) of the chunk, stages them in
// shared memory, and contributes its column sums to the mean and its SQ
// values to the ranking through distributed shared memory. Each CTA ranks
// its own rows against all BCP scores (4 threads per row) and normalises the
// rows that rank below NQ. Dynamic shared memory: the row block (element type
// T), SQloc[slice], SQall[BCP].
template <typename T, int D>
__global__ void __launch_bounds__(QSEL_CL_THREADS)
qsel_cluster_kernel(const T* __restrict__ Q, int64_t sQb, int64_t sQh, int64_t sQt, int BCP, int NQ,
                    int slice, float* __restrict__ Qhat, int32_t* __restrict__ q_idx, int normalize) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int c = (int)cluster.block_rank();
  extern __shared__ __align__(16) uint8_t qc_raw[];
  T* blk = reinterpret_cast<T*>(qc_raw);
  const size_t blk_bytes = ((size_t)slice * D * sizeof(T) + 15) & ~size_t(15);
  float* SQloc = reinterpret_cast<float*>(qc_raw + blk_bytes);
  float* SQall = SQloc + slice;
  __shared__ float part[QSEL_CL_THREADS];
  __shared__ float colsum[D];
  __shared__ float mq[D];
  __shared__ float mq_norm;

  const int h = blockIdx.y, bi = blockIdx.z, nq = gridDim.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r0 = c * slice;
  const int nrows = max(0, min(slice, BCP - r0));
  const T* Qh = Q + bi * sQb + h * sQh;

  constexpr int VPR = D * (int)sizeof(T) / 16;  // 16-byte vectors per row
#pragma unroll 8
  for (int e = tid; e < nrows * VPR; e += QSEL_CL_THREADS) {
    const int t = e / VPR, v = e % VPR;
    reinterpret_cast<uint4*>(blk + (size_t)t * D)[v] =
        __ldg(reinterpret_cast<const uint4*>(Qh + (int64_t)(r0 + t) * sQt) + v);
  }
  __syncthreads();

  // (a) this CTA's column sums, combined over the cluster in rank order
  constexpr int NGRP = QSEL_CL_THREADS / D;
  {
    const int col = tid % D, grp = tid / D;
    float acc = 0.f;
    for (int t = grp; t < nrows; t += NGRP) acc += to_f32(blk[(size_t)t * D + col]);
    part[tid] = acc;
  }
  __syncthreads();
  if (tid < D) {
    float sum = 0.f;
#pragma unroll
    for (int g = 0; g < NGRP; ++g) sum += part[g * D + tid];
    colsum[tid] = sum;
  }
  cluster.sync();
  if (tid < D) {
    float sum = 0.f;
    for (int r = 0; r < C; ++r) sum += cluster.map_shared_rank(colsum, r)[tid];
    mq[tid] = sum / (float)BCP;
  }
  __syncthreads();
  if (warp == 0) {
    float sum = 0.f;
    for (int k = lane; k < D; k += 32) sum += mq[k] * mq[k];
    sum = warp_sum(sum);
    if (lane == 0) mq_norm = sqrtf(sum);
  }
  __syncthreads();

  // (a) SQ of this CTA's rows, one warp per row
  for (int t = warp; t < nrows; t += QSEL_CL_WARPS) {
    const T* q = blk + (size_t)t * D;
    float dot = 0.f, qq = 0.f;
#pragma unroll
    for (int k = lane; k < D; k += 32) {
      const float v = to_f32(q[k]);
      dot += v * mq[k];
      qq += v * v;
    }
    dot = warp_sum(dot);
    qq = warp_sum(qq);
    if (lane == 0) SQloc[t] = -dot / fmaxf(sqrtf(qq) * mq_norm, 1e-8f);
  }
  cluster.sync();
  for (int t = tid; t < BCP; t += QSEL_CL_THREADS) SQall[t] = cluster.map_shared_rank(SQloc, t / slice)[t % slice];
  __syncthreads();

  // (b) rank of each own row over all BCP scores (4 threads per row), and
  // (c) normalisation of the rows ranked below NQ
  const int sub = tid & 3;
  for (int tl0 = 0; tl0 < nrows; tl0 += QSEL_CL_THREADS / 4) {
    const int tl = tl0 + (tid >> 2);
    const bool ok = tl < nrows;
    const int t = r0 + (ok ? tl : 0);
    const float v = SQall[t];
    int rk = 0;
    if (ok) {
      for (int u = sub; u < BCP; u += 4) {
        const float w = SQall[u];
        rk += (w > v) | ((w == v) & (u < t));
      }
    }
    rk += __shfl_xor_sync(0xffffffffu, rk, 1);
    rk += __shfl_xor_sync(0xffffffffu, rk, 2);
    const bool keep = ok && rk < NQ;
    const T* q = blk + (size_t)(ok ? tl : 0) * D;
    float qq = 0.f;
#pragma unroll
    for (int k = sub; k < D; k += 4) {
      const float x = to_f32(q[k]);
      qq += x * x;
    }
    qq += __shfl_xor_sync(0xffffffffu, qq, 1);
    qq += __shfl_xor_sync(0xffffffffu, qq, 2);
    if (keep) {
      const float nrm = normalize ? fmaxf(sqrtf(qq), 1e-12f) : 1.f;
      float* dst = Qhat + (((int64_t)bi * nq + h) * NQ + rk) * D;
      for (int k = sub; k < D; k += 4) dst[k] = to_f32(q[k]) / nrm;
      if (sub == 0 && q_idx != nullptr) q_idx[((int64_t)bi * nq + h) * NQ + rk] = t;
    }
  }
  cluster.sync();  // keep this CTA's shared memory alive for remote readers
}

// Q_group[b, j, i, :] = (1/G) sum_{g<G} Qhat[b, jG+g, i, :], summed in head
// order; optionally split into bf16 hi = rn(x) and lo = rn(x - hi).
template <int D>
__global__ void __launch_bounds__(D)
qgroup_kernel(const float* __restrict__ Qhat, int nq, int NQ, float* __restrict__ Qg,
              bf16* __restrict__ Qg_hilo, uint32_t* __restrict__ hist, int* __restrict__ status) {
  const int i = blockIdx.x, j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  clear_status(status);  // (the query select before it latches nothing)
  const int G = nq / nkv;
  const int k = threadIdx.x;
  float acc = 0.f;
  for (int g = 0; g < G; ++g) acc += Qhat[(((int64_t)bi * nq + j * G + g) * NQ + i) * D + k];
  const float v = acc / (float)G;
  const int64_t row = (int64_t)bi * nkv + j;
  Qg[(row * NQ + i) * D + k] = v;
  if (Qg_hilo != nullptr) {
    const bf16 hi = __float2bfloat16_rn(v);
    const bf16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    Qg_hilo[(row * 2 * NQ + i) * D + k] = hi;
    Qg_hilo[(row * 2 * NQ + NQ + i) * D + k] = lo;
  }
  if (hist != nullptr) {
    // the NQ blocks of a row zero its histogram between them
    uint32_t* h = hist + row * TOPK_HIST_BINS;
    for (int e = i * D + k; e < TOPK_HIST_BINS; e += NQ * D) h[e] = 0u;
  }
}

template <typename T, int D>
static cudaError_t qsel_typed(Strided Q, int b, int nq, int BCP, int NQ, float* Qhat,
                              int32_t* q_idx, bool normalize, cudaStream_t stream) {
  {
    int C = (BCP + 127) / 128;
    if (C > QSEL_CL_MAX) C = QSEL_CL_MAX;
    const int slice = (BCP + C - 1) / C;
    const size_t cl_bytes = (((size_t)slice * D * sizeof(T) + 15) & ~size_t(15)) +
                            (size_t)(slice + BCP) * sizeof(float);
    if (cl_bytes <= QSEL_STAGED_MAX_BYTES) {
      auto kern = qsel_cluster_kernel<T, D>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cl_bytes);
      if (e != cudaSuccess) return e;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(C, nq, b);
      cfg.blockDim = dim3(QSEL_CL_THREADS);
      cfg.dynamicSmemBytes = cl_bytes;
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = C;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(Q.data), Q.sb, Q.sh, Q.st, BCP, NQ, slice,
                                Qhat, q_idx, (int)normalize);
    }
  }
  const size_t blk_bytes = ((size_t)BCP * D * sizeof(T) + 15) & ~size_t(15);
  const size_t staged = blk_bytes + (size_t)BCP * sizeof(float) + (size_t)NQ * sizeof(int);
  if (staged <= QSEL_STAGED_MAX_BYTES) {
    auto kern = qsel_staged_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)staged);
    if (e != cudaSuccess) return e;
    kern<<<dim3(nq, b), QSEL_STAGED_THREADS, staged, stream>>>(static_cast<const T*>(Q.data), Q.sb, Q.sh, Q.st,
                                                               BCP, NQ, Qhat, q_idx, (int)normalize);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)BCP * sizeof(float) + (size_t)NQ * sizeof(int);
  auto kern = qsel_kernel<T, D>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<dim3(nq, b), QSEL_THREADS, smem, stream>>>(static_cast<const T*>(Q.data), Q.sb, Q.sh, Q.st,
                                                    BCP, NQ, Qhat, q_idx, (int)normalize);
  return cudaGetLastError();
}

cudaError_t launch_qsel(bool is_bf16, int d, Strided Q, int b, int nq, int BCP, int NQ,
                        float* Qhat, int32_t* q_idx, bool normalize, cudaStream_t stream) {
  if (is_bf16) {
    if (d == 128) return qsel_typed<bf16, 128>(Q, b, nq, BCP, NQ, Qhat, q_idx, normalize, stream);
    if (d == 64) return qsel_typed<bf16, 64>(Q, b, nq, BCP, NQ, Qhat, q_idx, normalize, stream);
  } else {
    if (d == 128) return qsel_typed<float, 128>(Q, b, nq, BCP, NQ, Qhat, q_idx, normalize, stream);
    if (d == 64) return qsel_typed<float, 64>(Q, b, nq, BCP, NQ, Qhat, q_idx, normalize, stream);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_qgroup(int d, const float* Qhat, int b, int nq, int nkv, int NQ, float* Qg,
                          uint16_t* Qg_hilo, uint32_t* hist, int* status, cudaStream_t stream) {
  dim3 grid(NQ, nkv, b);
  bf16* hl = reinterpret_cast<bf16*>(Qg_hilo);
  if (d == 128) qgroup_kernel<128><<<grid, 128, 0, stream>>>(Qhat, nq, NQ, Qg, hl, hist, status);
  else if (d == 64) qgroup_kernel<64><<<grid, 64, 0, stream>>>(Qhat, nq, NQ, Qg, hl, hist, status);
  else return cudaErrorNotSupported;
  return cudaGetLastError();
}

}  // namespace quoka
