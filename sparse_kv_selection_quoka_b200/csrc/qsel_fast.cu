// Steps (a)-(c) fused for the common shapes (bf16, d = 128, BCP <= 512,
// NQ <= 32, G <= 8): query subselection and the GQA group mean in one
// kernel.
//
// [QUOKA §2.1 Algorithm 1] MQ = mean over the chunk's queries,
// SQ[t] = -cos(Q[t], MQ), keep the NQ queries with the largest SQ (ties to
// the lower position), in rank order; [QUOKA §2.3] L2-normalise them and
// average over each KV head's G query heads at the same rank:
//   Qhat[h, i] = Q[h, t_i] / |Q[h, t_i]|,
//   Q_group[j, i] = (1/G) sum_{g<G} Qhat[jG + g, i]   (summed in head order).
// (QUOKA = the technical write-up "QUOKA: how it reshapes LLM prefill
// efficiency", bqwf.cn news item 915859.)
//
// One CTA (512 threads) per query head; the G CTAs of a KV head form a
// thread-block cluster. Per CTA:
//   1. the head's BCP x 128 queries are staged in shared memory (coalesced
//      16-byte loads; each row's 16-byte chunks rotated by the row index so
//      that the per-row reads below are conflict-free), while every thread
//      sums its column chunk over its rows;
//   2. the column sums are reduced over the warps: MQ and |MQ|;
//   3. one thread per row: Q[t] . MQ and |Q[t]|, hence SQ[t];
//   4. each warp sorts its 32 rows by (SQ descending, position ascending)
//      with a register bitonic sort, and a tree of warp merges keeps the top
//      32 of the head;
//   5. the NQ winners are normalised into shared memory (rank order);
//   6. after one cluster barrier, CTA g averages ranks g, g + G, ... over the
//      G heads through distributed shared memory, writes Q_group (fp32) and
//      its bf16 hi / lo split, and zeroes its share of the score histogram.
#include <cooperative_groups.h>
#include <stddef.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace quoka {

namespace {

constexpr int QF_D = 128;
constexpr int QF_THREADS = 512;
constexpr int QF_WARPS = QF_THREADS / 32;
constexpr int QF_MAX_BCP = 512;
constexpr int QF_MAX_NQ = 32;
constexpr int QF_MAX_G = 8;
constexpr int QF_CHUNKS = QF_D / 8;  // 16-byte chunks per bf16 row
static_assert(QF_MAX_NQ * (QF_D / 4) % QF_THREADS == 0, "group-mean units per thread");

struct __align__(16) QfShared {
  alignas(16) float qhat[QF_MAX_NQ][QF_D];  // the normalised winners, rank order (read as float4)
  alignas(16) float colpart[QF_WARPS][QF_D];  // per-warp column sums
  alignas(16) float mq[QF_D];
  float nrm[QF_MAX_BCP];             // |Q[t]| (clamped)
  uint64_t lists[QF_WARPS][32];       // sorted (key, position) lists of the merge tree
  float mq_norm;
};
static_assert(offsetof(QfShared, qhat) % 16 == 0 && sizeof(float) * QF_D % 16 == 0, "float4 rows of qhat");

// Ordering key of a row: SQ's order-preserving key in the high word, the
// complemented position in the low word (larger key = earlier rank).
__device__ __forceinline__ uint64_t row_key(float sq, int t) {
  return ((uint64_t)score_key(sq) << 32) | (uint64_t)(~(uint32_t)t);
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort of one key per lane, descending (largest at lane 0).
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t key, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const uint64_t other = shfl_xor_u64(key, jj);
      const bool desc = (lane & k) == 0 || k == 32;
      const bool lower = (lane & jj) == 0;
      key = (lower == desc) ? (key > other ? key : other) : (key < other ? key : other);
    }
  }
  return key;
}

// The 32 largest of two descending lists a (this lane's a[lane]) and b,
// descending: max(a[i], b[31 - i]) is bitonic; a half-cleaner cascade sorts it.
__device__ __forceinline__ uint64_t warp_merge_top(uint64_t a, const uint64_t* b, int lane) {
  const uint64_t br = b[31 - lane];
  uint64_t key = a > br ? a : br;
#pragma unroll
  for (int jj = 16; jj > 0; jj >>= 1) {
    const uint64_t other = shfl_xor_u64(key, jj);
    const bool lower = (lane & jj) == 0;
    key = lower ? (key > other ? key : other) : (key < other ? key : other);
  }
  return key;
}

__device__ __forceinline__ void cl_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cl_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(QF_THREADS, 1)
qsel_fast_kernel(const bf16* __restrict__ Q, int64_t sQb, int64_t sQh, int64_t sQt, int nq, int BCP, int NQ,
                 int32_t* __restrict__ q_idx, float* __restrict__ Qg, bf16* __restrict__ Qg_hilo,
                 uint32_t* __restrict__ hist, int* __restrict__ status, int normalize) {
  extern __shared__ __align__(16) uint8_t qf_raw[];
  uint8_t* qs = qf_raw;  // [BCP][256 B], chunk c of row t at slot (c ^ (t & 15))
  __shared__ QfShared sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int G = (int)cluster.num_blocks();
  const int g = (int)cluster.block_rank();
  const int j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  const int h = j * G + g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bf16* Qh = Q + bi * sQb + h * sQh;
  clear_status(status);  // the call's first kernel
  pdl_trigger();  // the scoring kernel may launch and start streaming K

  // 1. stage the rows; thread (rg, cc) handles chunk cc of rows rg, rg + 32, ...
  {
    const int cc = tid & 15, rg = tid >> 4;
    float cs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint4 v[QF_MAX_BCP / 32];
#pragma unroll
    for (int m = 0; m < QF_MAX_BCP / 32; ++m) {
      const int t = rg + 32 * m;
      v[m] = t < BCP ? __ldg(reinterpret_cast<const uint4*>(Qh + (int64_t)t * sQt) + cc) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int m = 0; m < QF_MAX_BCP / 32; ++m) {
      const int t = rg + 32 * m;
      if (t < BCP) reinterpret_cast<uint4*>(qs + (size_t)t * 256)[cc ^ (t & 15)] = v[m];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[m]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(h2[u]);
        cs[2 * u] += f.x;
        cs[2 * u + 1] += f.y;
      }
    }
    // lanes cc and cc + 16 hold the same chunk
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 16);
    if (lane < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sh.colpart[warp][cc * 8 + e] = cs[e];
    }
  }
  __syncthreads();
  // 2. MQ and |MQ|
  if (tid < QF_D) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < QF_WARPS; ++w) s += sh.colpart[w][tid];
    sh.mq[tid] = s / (float)BCP;
  }
  __syncthreads();
  if (warp == 0) {
    float s = 0.f;
#pragma unroll
    for (int k = lane; k < QF_D; k += 32) s += sh.mq[k] * sh.mq[k];
    s = warp_sum(s);
    if (lane == 0) sh.mq_norm = sqrtf(s);
  }
  __syncthreads();
  // 3. one thread per row: SQ and |Q[t]|
  uint64_t key = 0u;  // rows past the chunk sort last
  {
    const int t = tid;
    if (t < BCP) {
      float dot4[4] = {0.f, 0.f, 0.f, 0.f}, qq4[4] = {0.f, 0.f, 0.f, 0.f};
      const uint4* row = reinterpret_cast<const uint4*>(qs + (size_t)t * 256);
#pragma unroll
      for (int c = 0; c < QF_CHUNKS; ++c) {
        const uint4 raw = row[c ^ (t & 15)];
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
        const float4 ma = reinterpret_cast<const float4*>(sh.mq)[2 * c];
        const float4 mb = reinterpret_cast<const float4*>(sh.mq)[2 * c + 1];
        const float mv[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __bfloat1622float2(h2[u]);
          dot4[u] = fmaf(f.x, mv[2 * u], dot4[u]);
          dot4[u] = fmaf(f.y, mv[2 * u + 1], dot4[u]);
          qq4[u] = fmaf(f.x, f.x, qq4[u]);
          qq4[u] = fmaf(f.y, f.y, qq4[u]);
        }
      }
      const float dot = (dot4[0] + dot4[1]) + (dot4[2] + dot4[3]);
      const float qq = (qq4[0] + qq4[1]) + (qq4[2] + qq4[3]);
      const float sq = -dot / fmaxf(sqrtf(qq) * sh.mq_norm, 1e-8f);
      sh.nrm[t] = fmaxf(sqrtf(qq), 1e-12f);
      key = row_key(sq, t);
    }
  }
  // 4. per-warp sort, then a merge tree over the warps' lists
  key = warp_sort_desc(key, lane);
  sh.lists[warp][lane] = key;
  __syncthreads();
  // warps 0-3 fold lists 4w+1 .. 4w+3 into list 4w; then warp 0 folds the
  // four results into list 0
  if (warp < 4) {
    uint64_t m = sh.lists[4 * warp][lane];
#pragma unroll 1
    for (int u = 1; u < 4; ++u) m = warp_merge_top(m, sh.lists[4 * warp + u], lane);
    __syncwarp();
    sh.lists[4 * warp][lane] = m;
  }
  __syncthreads();
  if (warp == 0) {
    uint64_t m = sh.lists[0][lane];
#pragma unroll 1
    for (int u = 1; u < 4; ++u) m = warp_merge_top(m, sh.lists[4 * u], lane);
    __syncwarp();
    sh.lists[0][lane] = m;
  }
  __syncthreads();
  // 5. normalise the winners (thread = rank i, chunk cc), rank order
  {
    const int i = tid >> 4, cc = tid & 15;
    if (i < NQ) {
      const int t = (int)(~(uint32_t)sh.lists[0][i]);
      const uint4 raw = reinterpret_cast<const uint4*>(qs + (size_t)t * 256)[cc ^ (t & 15)];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      const float nrm = normalize ? sh.nrm[t] : 1.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(h2[u]);
        sh.qhat[i][cc * 8 + 2 * u] = f.x / nrm;
        sh.qhat[i][cc * 8 + 2 * u + 1] = f.y / nrm;
      }
      if (cc == 0 && q_idx != nullptr) q_idx[((int64_t)bi * nq + h) * NQ + i] = t;
    }
  }
  // 6. the group mean over the cluster's G heads
  cl_arrive();
  cl_wait();
  const int64_t row = (int64_t)bi * nkv + j;
  const int units = ((NQ - g + G - 1) / G) * (QF_D / 4);  // float4 units of this CTA's ranks
  constexpr int UPT = QF_MAX_NQ * (QF_D / 4) / QF_THREADS;  // units per thread at most (2)
  float4 acc[UPT];
#pragma unroll
  for (int u = 0; u < UPT; ++u) {
    const int e = tid + u * QF_THREADS;
    acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < units) {
      const int i = g + G * (e / (QF_D / 4)), c4 = e % (QF_D / 4);
      for (int hh = 0; hh < G; ++hh) {
        const QfShared* rs = cluster.map_shared_rank(&sh, hh);
        const float4 v = reinterpret_cast<const float4*>(rs->qhat[i])[c4];
        acc[u].x += v.x;
        acc[u].y += v.y;
        acc[u].z += v.z;
        acc[u].w += v.w;
      }
    }
  }
  // done reading the other CTAs' winners; the wait at the end keeps every
  // CTA alive until all have read
  cl_arrive();
#pragma unroll
  for (int u = 0; u < UPT; ++u) {
    const int e = tid + u * QF_THREADS;
    if (e >= units) continue;
    const int i = g + G * (e / (QF_D / 4)), c4 = e % (QF_D / 4);
    const float inv = 1.f / (float)G;
    const float o[4] = {acc[u].x * inv, acc[u].y * inv, acc[u].z * inv, acc[u].w * inv};
    reinterpret_cast<float4*>(Qg + (row * NQ + i) * QF_D)[c4] = make_float4(o[0], o[1], o[2], o[3]);
    if (Qg_hilo != nullptr) {
      uint32_t hw[2], lw[2];
#pragma unroll
      for (int v2 = 0; v2 < 2; ++v2) {
        const bf16 h0 = __float2bfloat16_rn(o[2 * v2]), h1 = __float2bfloat16_rn(o[2 * v2 + 1]);
        const bf16 l0 = __float2bfloat16_rn(o[2 * v2] - __bfloat162float(h0));
        const bf16 l1 = __float2bfloat16_rn(o[2 * v2 + 1] - __bfloat162float(h1));
        hw[v2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        lw[v2] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
      }
      // 8-byte stores: element offsets are multiples of 4
      *reinterpret_cast<uint2*>(Qg_hilo + (row * 2 * NQ + i) * QF_D + 4 * c4) = make_uint2(hw[0], hw[1]);
      *reinterpret_cast<uint2*>(Qg_hilo + (row * 2 * NQ + NQ + i) * QF_D + 4 * c4) = make_uint2(lw[0], lw[1]);
    }
  }
  if (hist != nullptr) {
    uint32_t* hr = hist + row * TOPK_HIST_BINS;
    for (int z = g * QF_THREADS + tid; z < TOPK_HIST_BINS; z += G * QF_THREADS) hr[z] = 0u;
  }
  cl_wait();
}

// A chunk of one query (BCP = 1, a decode step): Algorithm 1 has a single
// candidate, so every head keeps position 0 (NQ = 1) and steps (a)-(b)
// leave nothing to compute. What remains of step (c): each of the G heads'
// query is L2-normalised and the G are averaged (in head order) as above.
// One CTA (4 warps) per (batch, KV head): a warp takes one head at a time,
// lane l holding columns 4l .. 4l + 3.
constexpr int Q1_THREADS = 128;
constexpr int Q1_MAX_G = 32;

__global__ void __launch_bounds__(Q1_THREADS)
qsel_one_kernel(const bf16* __restrict__ Q, int64_t sQb, int64_t sQh, int nq, int G, int32_t* __restrict__ q_idx,
                float* __restrict__ Qg, bf16* __restrict__ Qg_hilo, uint32_t* __restrict__ hist,
                int* __restrict__ status, int normalize) {
  __shared__ __align__(16) float qhat[Q1_MAX_G][QF_D];
  const int j = blockIdx.x, bi = blockIdx.y, nkv = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  clear_status(status);  // the call's first kernel
  pdl_trigger();  // the scoring kernel may launch and start streaming K
  for (int g = warp; g < G; g += Q1_THREADS / 32) {
    const int h = j * G + g;
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(Q + bi * sQb + h * sQh) + lane);
    const float f[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                        __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
    const float qq = warp_sum((f[0] * f[0] + f[1] * f[1]) + (f[2] * f[2] + f[3] * f[3]));
    const float nrm = normalize ? fmaxf(sqrtf(qq), 1e-12f) : 1.f;
    reinterpret_cast<float4*>(qhat[g])[lane] = make_float4(f[0] / nrm, f[1] / nrm, f[2] / nrm, f[3] / nrm);
    if (lane == 0 && q_idx != nullptr) q_idx[(int64_t)bi * nq + h] = 0;
  }
  __syncthreads();
  const int64_t row = (int64_t)bi * nkv + j;
  float acc = 0.f;
  for (int g = 0; g < G; ++g) acc += qhat[g][tid];
  const float o = acc * (1.f / (float)G);
  Qg[row * QF_D + tid] = o;
  if (Qg_hilo != nullptr) {
    const bf16 hi = __float2bfloat16_rn(o);
    Qg_hilo[row * 2 * QF_D + tid] = hi;
    Qg_hilo[(row * 2 + 1) * QF_D + tid] = __float2bfloat16_rn(o - __bfloat162float(hi));
  }
  if (hist != nullptr) {
    uint4* hr = reinterpret_cast<uint4*>(hist + row * TOPK_HIST_BINS);
    for (int z = tid; z < TOPK_HIST_BINS / 4; z += Q1_THREADS) hr[z] = make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

cudaError_t launch_qsel_group_fast(Strided Q, int b, int nq, int nkv, int BCP, int NQ, int32_t* q_idx, float* Qg,
                                   uint16_t* Qg_hilo, uint32_t* hist, int* status, bool normalize,
                                   cudaStream_t stream) {
  const int G = nq / nkv;
  if (BCP == 1 && NQ == 1 && G >= 1 && G <= Q1_MAX_G && b <= 65535) {
    qsel_one_kernel<<<dim3(nkv, b), Q1_THREADS, 0, stream>>>(static_cast<const bf16*>(Q.data), Q.sb, Q.sh, nq, G,
                                                             q_idx, Qg, reinterpret_cast<bf16*>(Qg_hilo), hist,
                                                             status, (int)normalize);
    return cudaGetLastError();
  }
  if (BCP < 1 || BCP > QF_MAX_BCP || NQ < 1 || NQ > QF_MAX_NQ || NQ > BCP || G < 1 || G > QF_MAX_G)
    return cudaErrorNotSupported;
  if (nkv > 65535 || b > 65535) return cudaErrorNotSupported;
  const size_t smem = (size_t)BCP * 256;
  cudaError_t e = cudaFuncSetAttribute(qsel_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(smem < 1024 ? 1024 : smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G, nkv, b);
  cfg.blockDim = dim3(QF_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qsel_fast_kernel, static_cast<const bf16*>(Q.data), Q.sb, Q.sh, Q.st, nq, BCP,
                            NQ, q_idx, Qg, reinterpret_cast<bf16*>(Qg_hilo), hist, status, (int)normalize);
}

}  // namespace quoka
