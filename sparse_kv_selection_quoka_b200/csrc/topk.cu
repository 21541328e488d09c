// Top-BSA key selection per (batch, KV head).
//
// [QUOKA §2.3] indices = topk(S_agg, BSA). Ties at the BSA-th score go to the
// lower key index, and the chosen indices are written in ascending key order
// (the sorted format the attention kernels read). (QUOKA = the technical
// write-up "QUOKA: how it reshapes LLM prefill efficiency", bqwf.cn news item
// 915859.)
//
// One CTA per (batch, KV head) when the head's T scores fit in shared memory,
// else one thread-block cluster of C CTAs, each owning a contiguous slice.
// The scores are converted once into order-preserving 32-bit keys held in
// shared memory, and an exact MSB-first radix select with 12-, 12- and 8-bit
// digits finds the BSA-th largest key u*: the first digit's histogram comes
// from the scoring kernel when it made one (else it is built here); per
// later pass every CTA builds a histogram (warp-aggregated shared-memory
// atomics) of the keys that still match the known prefix; in a cluster the histograms are summed through
// distributed shared memory; a block scan finds the bin holding the BSA-th
// largest key. A final pass keeps the keys > u* and the first (in index
// order) keys == u* needed to reach BSA: each warp owns a contiguous segment
// of its CTA's slice, counts its picks, one block scan (plus a cluster
// exchange of CTA totals) gives every warp its output offset, and the warp
// writes its picks in order with ballots. Nothing is written to global memory
// but the result.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace quoka {

constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_WARPS = TOPK_THREADS / 32;
constexpr int TOPK_MAX_CLUSTER = 8;
constexpr int TOPK_MAX_SLICE = 44 * 1024;       // keys per CTA (176 KiB of shared memory)
constexpr int TOPK_SLICE_TARGET = 40 * 1024;    // one CTA per head up to this many keys
constexpr int TOPK_BINS = 4096;                 // widest digit: 12 bits
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
  uint32_t bin, above, total;
  uint32_t sel_base, take_eq;
};

// Inclusive block-wide scan of one value per thread, in thread order;
// *total receives the block sum. Three block barriers.
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
    if (lane == 31) sh.total = wi;
  }
  __syncthreads();
  incl += sh.woff[warp];
  *total = sh.total;
  __syncthreads();  // woff / total are reused by the next call
  return incl;
}

// Histogram increment aggregated over the lanes of a warp that hit the same
// bin (scores cluster in few bins, so plain atomics would serialise).
__device__ __forceinline__ void hist_add(uint32_t* H, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  if (act == (1u << (threadIdx.x & 31))) {  // alone in the warp: no aggregation needed
    atomicAdd(&H[bin], 1u);
    return;
  }
  const uint32_t peers = __match_any_sync(act, bin);
  const int lane = threadIdx.x & 31;
  if (lane == __ffs(peers) - 1) atomicAdd(&H[bin], (uint32_t)__popc(peers));
}

template <bool CLUSTER>
__global__ void __launch_bounds__(TOPK_THREADS)
topk_kernel(const float* __restrict__ S, int64_t T, int bsa, int slice, const uint32_t* __restrict__ ghist,
            int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_count) {
  extern __shared__ uint32_t keys[];
  __shared__ TopkShared sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = CLUSTER ? (int)cluster.num_blocks() : 1;
  const int c = CLUSTER ? (int)cluster.block_rank() : 0;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  const int64_t row = (int64_t)bi * nkv + j;
  const float* Sr = S + row * T;
  const int64_t lo = (int64_t)c * slice;
  const int n = (int)max((int64_t)0, min((int64_t)slice, T - lo));
  const int n_round = (n + TOPK_THREADS - 1) / TOPK_THREADS * TOPK_THREADS;

  // stage the slice as keys (16-byte loads when the slice start is aligned)
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
    // the first digit's histogram may come precomputed (whole head, global)
    const bool from_global = p == 0 && ghist != nullptr;
    if (!from_global) {
      for (int i = tid; i < nbins; i += TOPK_THREADS) H[i] = 0u;
      __syncthreads();
      for (int e = tid; e < n_round; e += TOPK_THREADS) {
        const uint32_t k = e < n ? keys[e] : 0u;
        hist_add(H, (k >> shift) & dmask, e < n && (k & pmask) == prefix);
      }
      if (CLUSTER) cluster.sync();  // every CTA's histogram of this pass is complete
      else __syncthreads();
    }

    // Thread t owns bins nbins-1-q*t .. nbins-q*(t+1) (largest keys first,
    // q = nbins / TOPK_THREADS bins each), summed over the cluster; the
    // inclusive scan gives the count of matching keys at or above each bin.
    const int q = nbins >= TOPK_THREADS ? nbins / TOPK_THREADS : 1;
    uint32_t mine[4] = {0u, 0u, 0u, 0u};
    uint32_t tot = 0u;
    if (tid * q < nbins && from_global) {
      const uint32_t* Hg = ghist + row * TOPK_BINS;
#pragma unroll
      for (int u = 0; u < 4; ++u) mine[u] = u < q ? __ldg(Hg + nbins - 1 - (tid * q + u)) : 0u;
      for (int u = 0; u < q; ++u) tot += mine[u];
    } else if (tid * q < nbins) {
      if (CLUSTER) {
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
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) mine[u] = u < q ? H[nbins - 1 - (tid * q + u)] : 0u;
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
    // cluster-wide barrier, by which time every CTA has finished reading it.
  }
  const uint32_t ustar = prefix;

  // Warp w owns the contiguous segment [w*seg, (w+1)*seg) of the slice and
  // counts its keys > u* and == u* (lane-strided reads: no bank conflicts).
  const int seg = (n + TOPK_WARPS - 1) / TOPK_WARPS;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  uint32_t g = 0u, q_eq = 0u;
  for (int e = s0 + lane; e < s1; e += 32) {
    const uint32_t k = keys[e];
    g += (k > ustar);
    q_eq += (k == ustar);
  }
  // both counts in one scan: (gt << 16) | eq (per-CTA counts < 65536)
  uint32_t packed = (g << 16) | q_eq;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) packed += __shfl_xor_sync(0xffffffffu, packed, o);
  uint32_t cta_total;
  const uint32_t wincl = block_scan_incl(lane == 0 ? packed : 0u, sh, &cta_total);
  const uint32_t wex = wincl - (lane == 0 ? packed : 0u);  // valid in lane 0
  const uint32_t w_gt_before = __shfl_sync(0xffffffffu, wex >> 16, 0);
  const uint32_t w_eq_before = __shfl_sync(0xffffffffu, wex & 0xFFFFu, 0);
  const uint32_t w_eq = packed & 0xFFFFu;  // warp sums are replicated in every lane
  if (tid == 0) {
    sh.counts[0] = cta_total >> 16;
    sh.counts[1] = cta_total & 0xFFFFu;
  }
  if (CLUSTER) cluster.sync();
  else __syncthreads();
  if (tid == 0) {
    uint32_t sel_base = 0u, eq_seen = 0u, my_take = 0u;
    for (int r = 0; r < C; ++r) {
      const uint32_t* cr = CLUSTER ? cluster.map_shared_rank(sh.counts, r) : sh.counts;
      const uint32_t gr = cr[0], er = cr[1];
      const uint32_t take = need > eq_seen ? min(er, need - eq_seen) : 0u;
      if (r < c) sel_base += gr + take;
      if (r == c) my_take = take;
      eq_seen += er;
    }
    sh.sel_base = sel_base;
    sh.take_eq = my_take;
  }
  __syncthreads();
  // this warp's share of the tied keys, and its first output position
  const uint32_t take_cta = sh.take_eq;
  const uint32_t w_take = take_cta > w_eq_before ? min(w_eq, take_cta - w_eq_before) : 0u;
  uint32_t out = sh.sel_base + w_gt_before + min(w_eq_before, take_cta);
  uint32_t eq_used = 0u;
  int32_t* dst = kv_idx + row * bsa;
  for (int base = s0; base < s1; base += 32) {
    const int e = base + lane;
    const uint32_t k = e < s1 ? keys[e] : 0u;
    const bool is_gt = e < s1 && k > ustar;
    const bool is_eq = e < s1 && k == ustar;
    const uint32_t below = (1u << lane) - 1u;
    const uint32_t eqb = __ballot_sync(0xffffffffu, is_eq);
    const bool take_it = is_gt || (is_eq && eq_used + (uint32_t)__popc(eqb & below) < w_take);
    const uint32_t selb = __ballot_sync(0xffffffffu, take_it);
    if (take_it) {
      const uint32_t pos = out + (uint32_t)__popc(selb & below);
      if (pos < (uint32_t)bsa) dst[pos] = (int32_t)(lo + e);
    }
    out += (uint32_t)__popc(selb);
    eq_used += (uint32_t)__popc(eqb);
  }
  if (c == 0 && tid == 0) kv_count[row] = bsa;
  if (CLUSTER) cluster.sync();  // keep this CTA's shared memory alive for remote readers
}

cudaError_t launch_topk(const float* S_agg, int b, int nkv, int64_t T, int bsa, const uint32_t* hist,
                        int32_t* kv_idx, int32_t* kv_count, cudaStream_t stream) {
  if (bsa <= 0 || T <= 0 || bsa > T || T > topk_max_T()) return cudaErrorInvalidValue;
  int C = (int)((T + TOPK_SLICE_TARGET - 1) / TOPK_SLICE_TARGET);
  if (C > TOPK_MAX_CLUSTER) C = TOPK_MAX_CLUSTER;
  if (C < 1) C = 1;
  const int slice = (int)((T + C - 1) / C);
  if (slice > TOPK_MAX_SLICE) return cudaErrorInvalidValue;
  const size_t smem = (size_t)slice * sizeof(uint32_t);
  if (C == 1) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(smem < 1024 ? 1024 : smem));
    if (e != cudaSuccess) return e;
    topk_kernel<false><<<dim3(1, nkv, b), TOPK_THREADS, smem, stream>>>(S_agg, T, bsa, slice, hist, kv_idx,
                                                                        kv_count);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  return cudaLaunchKernelEx(&cfg, topk_kernel<true>, S_agg, T, bsa, slice, hist, kv_idx, kv_count);
}

}  // namespace quoka
