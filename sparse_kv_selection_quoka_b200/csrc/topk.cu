// Top-BSA key selection per (batch, KV head).
//
// [QUOKA §2.3] indices = topk(S_agg, BSA). Ties at the BSA-th score go to the
// lower key index, and the chosen indices are written in ascending key order
// (the sorted format the attention kernels read).
//
// One thread-block cluster per (batch, KV head). Each CTA of the cluster owns
// a contiguous slice of the T scores, converts them once into order-preserving
// 32-bit keys held in shared memory, and the cluster runs an exact MSB-first
// radix select with 12-, 12- and 8-bit digits: per pass every CTA builds a
// histogram (warp-aggregated shared-memory atomics) of the keys that still
// match the known prefix, every CTA sums the cluster's histograms through
// distributed shared memory and finds the bin that holds the BSA-th largest
// key. After three passes the exact threshold key u* is known, together with
// how many keys equal to u* must be taken. A final pass compacts, in index
// order (ballot + block scan), the keys > u* and the first such keys == u*.
// Nothing is written to global memory but the result.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace quoka {

constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_WARPS = TOPK_THREADS / 32;
constexpr int TOPK_MAX_CLUSTER = 8;
constexpr int TOPK_MAX_SLICE = 44 * 1024;  // keys per CTA (176 KiB of shared memory)
constexpr int TOPK_BINS = 4096;            // widest digit: 12 bits
constexpr int TOPK_PASSES = 3;
// Digits, most significant first: bits [31:20], [19:8], [7:0]. Scores lie in
// [-1, 1], so the top 12 bits (sign, exponent, 3 mantissa bits) already
// spread them over a few dozen bins.
__constant__ int kTopkShift[TOPK_PASSES] = {20, 8, 0};
__constant__ int kTopkBits[TOPK_PASSES] = {12, 12, 8};

int64_t topk_max_T() { return (int64_t)TOPK_MAX_CLUSTER * TOPK_MAX_SLICE; }

struct TopkShared {
  uint32_t hist[2][TOPK_BINS];
  uint32_t wsum[TOPK_WARPS];
  uint32_t woff[TOPK_WARPS];
  uint32_t counts[2];  // keys > u*, keys == u* in this CTA's slice
  uint32_t bin, above, round_total;
  uint32_t sel_base, take_eq;
};

// Inclusive block-wide scan of one value per thread, in thread order.
// *total receives the block sum. Contains three block barriers.
__device__ __forceinline__ uint32_t block_scan_incl(uint32_t v, TopkShared& sh, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) sh.wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = sh.wsum[lane];
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    sh.woff[lane] = wi - w;
    if (lane == 31) sh.round_total = wi;
  }
  __syncthreads();
  incl += sh.woff[warp];
  *total = sh.round_total;
  __syncthreads();  // woff / round_total are reused by the next call
  return incl;
}

// Exclusive rank of a 0/1 flag among the block's threads, in thread order.
__device__ __forceinline__ uint32_t block_rank(bool flag, TopkShared& sh, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) sh.wsum[warp] = __popc(ballot);
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = sh.wsum[lane];
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    sh.woff[lane] = wi - w;
    if (lane == 31) sh.round_total = wi;
  }
  __syncthreads();
  const uint32_t r = sh.woff[warp] + __popc(ballot & ((1u << lane) - 1u));
  *total = sh.round_total;
  __syncthreads();
  return r;
}

// Histogram increment aggregated over the lanes of a warp that hit the same
// bin (scores cluster in few bins, so plain atomics would serialise).
__device__ __forceinline__ void hist_add(uint32_t* H, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  const int lane = threadIdx.x & 31;
  if (lane == __ffs(peers) - 1) atomicAdd(&H[bin], (uint32_t)__popc(peers));
}

__global__ void __launch_bounds__(TOPK_THREADS)
topk_cluster_kernel(const float* __restrict__ S, int64_t T, int bsa, int slice,
                    int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_count) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int c = (int)cluster.block_rank();
  extern __shared__ uint32_t keys[];
  __shared__ TopkShared sh;

  const int tid = threadIdx.x;
  const int j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  const int64_t row = (int64_t)bi * nkv + j;
  const float* Sr = S + row * T;
  const int64_t lo = (int64_t)c * slice;
  const int n = (int)max((int64_t)0, min((int64_t)slice, T - lo));
  const int n_round = (n + TOPK_THREADS - 1) / TOPK_THREADS * TOPK_THREADS;

  // stage the slice as keys: 16-byte loads when the slice start is aligned
  if ((((uintptr_t)(Sr + lo)) & 15u) == 0u) {
    const int n4 = n >> 2;
    const float4* src4 = reinterpret_cast<const float4*>(Sr + lo);
#pragma unroll 4
    for (int e = tid; e < n4; e += TOPK_THREADS) {
      const float4 v = __ldg(src4 + e);
      keys[4 * e] = score_key(v.x);
      keys[4 * e + 1] = score_key(v.y);
      keys[4 * e + 2] = score_key(v.z);
      keys[4 * e + 3] = score_key(v.w);
    }
    for (int e = 4 * n4 + tid; e < n; e += TOPK_THREADS) keys[e] = score_key(Sr[lo + e]);
  } else {
    for (int e = tid; e < n; e += TOPK_THREADS) keys[e] = score_key(Sr[lo + e]);
  }

  uint32_t prefix = 0u, pmask = 0u;
  uint32_t need = (uint32_t)bsa;  // rank (1-based, from the top) still to place
#pragma unroll 1
  for (int p = 0; p < TOPK_PASSES; ++p) {
    const int shift = kTopkShift[p];
    const int nbins = 1 << kTopkBits[p];
    const uint32_t dmask = (uint32_t)nbins - 1u;
    uint32_t* H = sh.hist[p & 1];
    for (int i = tid; i < nbins; i += TOPK_THREADS) H[i] = 0u;
    __syncthreads();
    for (int e = tid; e < n_round; e += TOPK_THREADS) {
      const uint32_t k = e < n ? keys[e] : 0u;
      hist_add(H, (k >> shift) & dmask, e < n && (k & pmask) == prefix);
    }
    cluster.sync();  // every CTA's histogram of this pass is complete

    // Thread t owns the bins nbins-1-q*t .. nbins-q*(t+1) (largest keys first,
    // q = nbins / TOPK_THREADS bins each), summed over the cluster; the
    // inclusive scan gives the count of matching keys at or above each bin.
    const int q = nbins >= TOPK_THREADS ? nbins / TOPK_THREADS : 1;
    uint32_t mine[4] = {0u, 0u, 0u, 0u};
    uint32_t tot = 0u;
    if (tid * q < nbins) {
      // all remote loads are issued before any is used
      uint32_t got[TOPK_MAX_CLUSTER][4];
#pragma unroll
      for (int r = 0; r < TOPK_MAX_CLUSTER; ++r) {
        if (r < C) {
          const uint32_t* Hr = cluster.map_shared_rank(H, r);
#pragma unroll
          for (int u = 0; u < 4; ++u) got[r][u] = u < q ? Hr[nbins - 1 - (tid * q + u)] : 0u;
        }
      }
#pragma unroll
      for (int r = 0; r < TOPK_MAX_CLUSTER; ++r)
        if (r < C) {
#pragma unroll
          for (int u = 0; u < 4; ++u) mine[u] += got[r][u];
        }
      for (int u = 0; u < q; ++u) tot += mine[u];
    }
    uint32_t dummy;
    const uint32_t incl = block_scan_incl(tot, sh, &dummy);
    if (tid * q < nbins && incl >= need && incl - tot < need) {
      uint32_t acc = incl - tot;
      for (int u = 0; u < q; ++u) {
        if (acc + mine[u] >= need) {
          sh.bin = (uint32_t)(nbins - 1 - (tid * q + u));
          sh.above = acc;
          break;
        }
        acc += mine[u];
      }
    }
    __syncthreads();
    need -= sh.above;
    prefix |= sh.bin << shift;
    pmask |= dmask << shift;
    // This histogram buffer is next cleared two passes later, after another
    // cluster.sync, by which time every CTA has finished reading it.
  }
  const uint32_t ustar = prefix;

  // Count keys above and equal to u* in this slice, publish, and let every
  // CTA derive its output offset and its share of the tied keys.
  uint32_t gt = 0u, eq = 0u;
  for (int e = tid; e < n; e += TOPK_THREADS) {
    const uint32_t k = keys[e];
    gt += (k > ustar);
    eq += (k == ustar);
  }
  uint32_t tg, te;
  block_scan_incl(gt, sh, &tg);
  block_scan_incl(eq, sh, &te);
  if (tid == 0) {
    sh.counts[0] = tg;
    sh.counts[1] = te;
  }
  cluster.sync();
  if (tid == 0) {
    uint32_t sel_base = 0u, eq_seen = 0u, my_take = 0u;
    for (int r = 0; r < C; ++r) {
      const uint32_t* cr = cluster.map_shared_rank(sh.counts, r);
      const uint32_t g = cr[0], e = cr[1];
      const uint32_t take = need > eq_seen ? min(e, need - eq_seen) : 0u;
      if (r < c) sel_base += g + take;
      if (r == c) my_take = take;
      eq_seen += e;
    }
    sh.sel_base = sel_base;
    sh.take_eq = my_take;
  }
  __syncthreads();
  const uint32_t my_eq = sh.counts[1];
  const uint32_t take = sh.take_eq;
  const bool partial = take > 0u && take < my_eq;
  uint32_t out = sh.sel_base;
  uint32_t eq_seen = 0u;
  int32_t* dst = kv_idx + row * bsa;

  // Ordered compaction in rounds of TOPK_THREADS keys: thread order within a
  // round is key order, so block ranks give ascending output positions.
  for (int base = 0; base < n; base += TOPK_THREADS) {
    const int e = base + tid;
    const uint32_t k = e < n ? keys[e] : 0u;
    const bool is_gt = e < n && k > ustar;
    const bool is_eq = e < n && k == ustar;
    bool take_it;
    if (partial) {
      uint32_t eq_round;
      const uint32_t eq_rank = eq_seen + block_rank(is_eq, sh, &eq_round);
      take_it = is_gt || (is_eq && eq_rank < take);
      eq_seen += eq_round;
    } else {
      take_it = is_gt || (is_eq && take > 0u);
    }
    uint32_t sel_round;
    const uint32_t pos = block_rank(take_it, sh, &sel_round);
    if (take_it && out + pos < (uint32_t)bsa) dst[out + pos] = (int32_t)(lo + e);
    out += sel_round;
  }
  if (c == 0 && tid == 0) kv_count[row] = bsa;
  cluster.sync();  // keep this CTA's shared memory alive for remote readers
}

cudaError_t launch_topk(const float* S_agg, int b, int nkv, int64_t T, int bsa, int32_t* kv_idx,
                        int32_t* kv_count, cudaStream_t stream) {
  if (bsa <= 0 || T <= 0 || bsa > T || T > topk_max_T()) return cudaErrorInvalidValue;
  // Cluster size: about 8192 keys per CTA, at most 8 CTAs.
  int C = (int)((T + 8191) / 8192);
  if (C > TOPK_MAX_CLUSTER) C = TOPK_MAX_CLUSTER;
  if (C < 1) C = 1;
  // power of two keeps the cluster shape simple
  int Cp = 1;
  while (Cp < C) Cp <<= 1;
  C = Cp;
  const int slice = (int)((T + C - 1) / C);
  if (slice > TOPK_MAX_SLICE) return cudaErrorInvalidValue;
  const size_t smem = (size_t)slice * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(smem < 1024 ? 1024 : smem));
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, nkv, b);
  cfg.blockDim = dim3(TOPK_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, S_agg, T, bsa, slice, kv_idx, kv_count);
}

}  // namespace quoka
