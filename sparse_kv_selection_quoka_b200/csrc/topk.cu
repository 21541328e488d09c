// Top-BSA key selection per (batch, KV head).
//
// [QUOKA §2.3] the BSA keys of each KV head with the highest aggregated
// score S_agg are kept. Ties at the BSA-th score go to the
// lower key index, and the chosen indices are written in ascending key order
// (the sorted format the attention kernels read). (QUOKA = the technical
// write-up "QUOKA: how it reshapes LLM prefill efficiency", bqwf.cn news item
// 915859.)
//
// A thread-block cluster of C CTAs per (batch, KV head) (C = 1 for short
// rows), each owning a contiguous slice of the row, staged in shared memory
// as order-preserving 32-bit keys. The select finds the BSA-th largest key
// u* most significant part first:
//   1. The score's 12-bit value bucket (linear over [-1, 1], where the
//      scores lie; the bit pattern's top bits would put nearly all of them
//      in a few bins). Its histogram comes from the scoring kernel when it
//      made one (else it is built here, summed over the cluster); a block
//      scan finds the threshold bucket b0.
//   2. One pass over the slice counts the keys above b0 and lists the keys
//      in b0 (the candidates). After one cluster barrier every CTA reads all
//      ranks' counts and candidate lists (small: a bucket is 1/2048 of the
//      score range) and resolves u* among the candidates on its own (direct
//      ranking, or radix passes over the gathered list), and from the same
//      data its output offset: nothing else crosses between the CTAs.
//   3. The final pass keeps the keys > u* and the first (in index order)
//      keys == u* needed to reach BSA: each warp owns a contiguous segment of
//      the slice, counts its picks, one block scan gives every warp its
//      offset, and the warp writes its picks in order with ballots.
// When a bucket holds more candidates than the gathered list can take, the
// exact passes run over every slice instead, their histograms summed over
// the cluster through distributed shared memory.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace quoka {

namespace {

constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_WARPS = TOPK_THREADS / 32;
constexpr int TOPK_MAX_CLUSTER = 8;
constexpr int TOPK_MAX_SLICE = 36 * 1024;  // keys per CTA (144 KiB of shared memory; 208 KiB in all)
constexpr int TOPK_SLICE_TARGET = 4096;    // keys per CTA while the cluster can spread them
constexpr int TOPK_LIST_MAX = 4096;        // candidates gathered in every CTA
constexpr int TOPK_BINS = 4096;            // widest digit: 12 bits
static_assert(TOPK_BINS / TOPK_THREADS <= 4, "bins per thread in a pick");

struct TopkShared {
  uint32_t hist[2][TOPK_BINS];
  uint32_t wsum[TOPK_WARPS];
  uint32_t woff[TOPK_WARPS];
  uint32_t bin, above, total, bincount;
  uint32_t kmin, kmax;       // smallest / largest candidate key (this CTA)
  uint32_t gt0;              // keys of this slice above the threshold bucket
  uint32_t ncand;            // candidates of this slice (keys in the bucket)
  uint32_t rank_base[TOPK_MAX_CLUSTER + 1];  // gathered list: where each rank's part starts
  uint32_t rc_gt[TOPK_MAX_CLUSTER];   // per rank: keys above the threshold bucket
  uint32_t rc_n[TOPK_MAX_CLUSTER];    // per rank: candidates
  uint32_t rc_gtc[TOPK_MAX_CLUSTER];  // per rank: candidates > u*
  uint32_t rc_eqc[TOPK_MAX_CLUSTER];  // per rank: candidates == u*
  uint32_t cgt[TOPK_THREADS], ceq[TOPK_THREADS];  // direct ranking: per candidate, #greater / #equal
  uint8_t grank[TOPK_LIST_MAX];       // gathered list: the rank each candidate came from
  uint32_t ustar, need_eq;   // the BSA-th largest key; how many keys == u* the row keeps
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

// Split cluster barrier: every thread of every CTA arrives, then waits;
// work placed in between overlaps the barrier.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

template <bool CLUSTER>
__global__ void __launch_bounds__(TOPK_THREADS)
topk_kernel(const float* __restrict__ S, int64_t T, int bsa, int slice, const uint32_t* __restrict__ ghist,
            int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_count, const int* __restrict__ status) {
  extern __shared__ uint32_t smem_dyn[];
  uint32_t* keys = smem_dyn;          // [slice]: this CTA's keys
  uint32_t* glist = smem_dyn + slice;  // [TOPK_LIST_MAX]: all ranks' candidates, in rank order
  uint32_t* clist = glist + TOPK_LIST_MAX;  // [TOPK_LIST_MAX]: this slice's candidates
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

  pdl_trigger();
  if (tid == 0) {
    sh.kmin = 0xFFFFFFFFu;
    sh.kmax = 0u;
    sh.gt0 = 0u;
    sh.ncand = 0u;
  }
  if (tid < TOPK_MAX_CLUSTER) {
    sh.rc_gtc[tid] = 0u;
    sh.rc_eqc[tid] = 0u;
  }
  sh.cgt[tid] = 0u;
  sh.ceq[tid] = 0u;
  // the scoring kernel's histogram bins this thread owns in the first pick
  // (loaded first: the loads overlap the staging below)
  uint32_t g0[4] = {0u, 0u, 0u, 0u};
  // The scores and their histogram come from the previous kernel, which may
  // still run until this wait returns: they are read with L2-coherent loads
  // (never the read-only path, which assumes data fixed for the kernel's life).
  pdl_wait();
  // (the status word is loaded with the histogram and the scores, and
  // tested once they are staged)
  const int fault = status != nullptr ? __ldcg(status) : 0;
  if (ghist != nullptr) {
    const uint32_t* Hg = ghist + row * TOPK_BINS;
    constexpr int q0 = TOPK_BINS / TOPK_THREADS;
#pragma unroll
    for (int u = 0; u < q0; ++u) g0[u] = __ldcg(Hg + TOPK_BINS - 1 - (tid * q0 + u));
  }
  // stage the slice as keys (16-byte loads when the slice start is aligned)
  if ((((uintptr_t)(Sr + lo)) & 15u) == 0u) {
    const int n4 = n >> 2;
    const float4* src4 = reinterpret_cast<const float4*>(Sr + lo);
#pragma unroll 4
    for (int e = tid; e < n4; e += TOPK_THREADS) {
      const float4 v = __ldcg(src4 + e);
      reinterpret_cast<uint4*>(keys)[e] = make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
    }
    for (int e = 4 * n4 + tid; e < n; e += TOPK_THREADS) keys[e] = score_key(__ldcg(Sr + lo + e));
  } else {
    for (int e = tid; e < n; e += TOPK_THREADS) keys[e] = score_key(__ldcg(Sr + lo + e));
  }
  // A device fault latched earlier in the call (a scoring kernel that gave
  // up) leaves the scores and their histogram incomplete: select nothing.
  // Every CTA of the cluster read the same word (nothing writes it while
  // this kernel runs) before any cluster barrier, so they all leave here
  // together.
  if (fault != 0) {
    if (c == 0 && tid == 0) kv_count[row] = 0;
    return;
  }

  // From a histogram over `nbins` bins (this CTA's H, optionally summed over
  // the cluster, or the preloaded global one), the bin holding the need-th
  // largest of the counted keys, the count of counted keys in higher bins,
  // and the bin's own count. Thread t owns bins nbins-1-q*t .. nbins-q*(t+1)
  // (largest first, q = nbins / TOPK_THREADS bins each); an inclusive block
  // scan gives the count at or above each bin.
  auto pick_bin = [&](const uint32_t* H, int nbins, bool global, bool sum_cluster, uint32_t need_,
                      uint32_t* bin_out, uint32_t* above_out) {
    const int q = nbins >= TOPK_THREADS ? nbins / TOPK_THREADS : 1;
    uint32_t mine[4] = {0u, 0u, 0u, 0u};
    if (global) {
#pragma unroll
      for (int u = 0; u < 4; ++u) mine[u] = g0[u];
    } else if (tid * q < nbins) {
      if (CLUSTER && sum_cluster) {
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
    }
    const uint32_t tot = (mine[0] + mine[1]) + (mine[2] + mine[3]);
    uint32_t dummy;
    const uint32_t incl = block_scan_incl(tot, sh, &dummy);
    if (tid * q < nbins && incl >= need_ && incl - tot < need_) {
      uint32_t acc = incl - tot;
      for (int u = 0; u < q; ++u) {
        if (acc + mine[u] >= need_) {
          sh.bin = (uint32_t)(nbins - 1 - (tid * q + u));
          sh.above = acc;
          sh.bincount = mine[u];
          break;
        }
        acc += mine[u];
      }
    }
    __syncthreads();
    *bin_out = sh.bin;
    *above_out = sh.above;
  };

  // Exact passes over candidate keys: 12-bit digits of the key from the
  // highest bit where the smallest and largest candidate differ (the bits
  // above it are common to all candidates). `full_scan`: walk the slice,
  // testing the bucket (histograms summed over the cluster); else walk
  // list[0 .. nlist) (this CTA alone). Returns u*; `need` becomes the
  // number of keys == u* to keep.
  uint32_t need = (uint32_t)bsa;  // rank (1-based, from the top) still to place
  uint32_t b0 = 0u, above = 0u;
  auto exact_passes = [&](uint32_t kmin, uint32_t kmax, bool full_scan, const uint32_t* list, int nlist) {
    uint32_t prefix = kmin;  // all candidates equal: u* is their key
    if (kmin == kmax) return prefix;
    int hb = 31 - __clz(kmin ^ kmax);
    uint32_t pmask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    prefix = kmax & pmask;
    const int nlist_round = (nlist + TOPK_THREADS - 1) / TOPK_THREADS * TOPK_THREADS;
#pragma unroll 1
    for (int p = 1;; ++p) {
      const int width = min(12, hb + 1), shift = hb + 1 - width;
      const int nbins = 1 << width;
      const uint32_t dmask = (uint32_t)nbins - 1u;
      // this buffer was last read (remotely too) two passes ago, before a
      // cluster-wide barrier every CTA has since passed
      uint32_t* H = sh.hist[p & 1];
      for (int i = tid; i < nbins; i += TOPK_THREADS) H[i] = 0u;
      __syncthreads();
      if (full_scan) {
        for (int e = tid; e < n_round; e += TOPK_THREADS) {
          const uint32_t k = e < n ? keys[e] : 0u;
          const bool cand = e < n && (k & pmask) == prefix && score_bin(key_score(k)) == b0;
          hist_add(H, (k >> shift) & dmask, cand);
        }
        if (CLUSTER) cluster.sync();
        else __syncthreads();
      } else {
        for (int i = tid; i < nlist_round; i += TOPK_THREADS) {
          const uint32_t k = i < nlist ? list[i] : 0u;
          hist_add(H, (k >> shift) & dmask, i < nlist && (k & pmask) == prefix);
        }
        __syncthreads();
      }
      uint32_t bin;
      pick_bin(H, nbins, false, full_scan, need, &bin, &above);
      need -= above;
      prefix |= bin << shift;
      pmask |= dmask << shift;
      if (shift == 0) break;
      hb = shift - 1;
    }
    return prefix;
  };

  // 1. the value bucket b0 holding the BSA-th largest score
  {
    uint32_t* H = sh.hist[0];
    if (ghist == nullptr) {
      for (int i = tid; i < TOPK_BINS; i += TOPK_THREADS) H[i] = 0u;
      __syncthreads();
      for (int e = tid; e < n_round; e += TOPK_THREADS) {
        const uint32_t k = e < n ? keys[e] : 0u;
        hist_add(H, score_bin(key_score(k)), e < n);
      }
      if (CLUSTER) cluster.sync();  // every CTA's histogram is complete
      else __syncthreads();
    }
    pick_bin(H, TOPK_BINS, ghist != nullptr, true, need, &b0, &above);
    need -= above;
  }
  const uint32_t cnt0 = sh.bincount;  // keys of the whole row in bucket b0
  const bool gathered = cnt0 <= (uint32_t)TOPK_LIST_MAX;  // the same in every CTA

  uint32_t ustar;
  if (gathered) {
    // 2a. count this slice's keys above b0 and list its keys in b0
    uint32_t gt = 0u;
    for (int e0 = 0; e0 < n_round; e0 += TOPK_THREADS) {
      const int e = e0 + tid;
      const uint32_t k = e < n ? keys[e] : 0u;
      const uint32_t bk = score_bin(key_score(k));
      gt += (e < n && bk > b0) ? 1u : 0u;
      const bool cand = e < n && bk == b0;
      const uint32_t cb = __ballot_sync(0xffffffffu, cand);
      if (cb != 0u) {
        uint32_t base = 0u;
        if (lane == 0) base = atomicAdd(&sh.ncand, (uint32_t)__popc(cb));
        base = __shfl_sync(0xffffffffu, base, 0);
        const uint32_t pos = base + (uint32_t)__popc(cb & ((1u << lane) - 1u));
        if (cand && pos < (uint32_t)TOPK_LIST_MAX) clist[pos] = k;  // pos < cnt0 <= TOPK_LIST_MAX
      }
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    if (lane == 0 && gt != 0u) atomicAdd(&sh.gt0, gt);
    // 2b. every rank's counts and candidates, gathered in rank order
    if (CLUSTER) {
      cluster_arrive();
      cluster_wait();
    } else {
      __syncthreads();
    }
    // warp 0: every rank's counts, and where its part of the gathered list
    // starts (exclusive scan over the ranks)
    if (warp == 0) {
      uint32_t gtr = 0u, nr = 0u;
      if (lane < C) {
        const TopkShared* shr = CLUSTER ? cluster.map_shared_rank(&sh, lane) : &sh;
        gtr = shr->gt0;
        nr = shr->ncand;
      }
      uint32_t incl = nr;
#pragma unroll
      for (int o = 1; o < TOPK_MAX_CLUSTER; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane < C) {
        sh.rc_gt[lane] = gtr;
        sh.rank_base[lane] = incl - nr;
      }
      if (lane == C - 1) sh.rank_base[C] = incl;
    }
    __syncthreads();
    // == cnt0 (the bounds below only guard the shared-memory lists should
    // a histogram ever disagree with the scores)
    const int nl = min((int)sh.rank_base[C], TOPK_LIST_MAX);
    for (int g = tid; g < nl; g += TOPK_THREADS) {
      int r = 0;
      while (r + 1 < C && (uint32_t)g >= sh.rank_base[r + 1]) ++r;
      const uint32_t* cl = CLUSTER ? cluster.map_shared_rank(clist, r) : clist;
      const uint32_t at = (uint32_t)g - sh.rank_base[r];
      glist[g] = at < (uint32_t)TOPK_LIST_MAX ? cl[at] : 0u;
      sh.grank[g] = (uint8_t)r;
    }
    // done reading the other CTAs' shared memory (their wait at the end
    // keeps every CTA alive until all have read)
    if (CLUSTER) cluster_arrive();
    __syncthreads();
    // 2c. u* among the gathered candidates, and how many candidates of each
    // rank lie above it / equal it
    if (nl <= TOPK_THREADS) {
      // Direct ranking: candidate i counts the candidates greater than /
      // equal to it (the comparisons split over the idle warps, partial
      // counts summed in shared memory). u* is the key whose rank range
      // [#greater, #greater + #equal) holds `need`; a candidate is above u*
      // exactly when its whole range lies before `need`.
      const int ncw = (nl + 31) / 32;      // warps of candidates
      const int nsplit = TOPK_WARPS / ncw;  // comparison groups
      const int grp = warp / ncw;
      if (grp < nsplit) {
        const int i = (warp % ncw) * 32 + lane;
        const uint32_t k = i < nl ? glist[i] : 0u;
        const int jlen = (nl + nsplit - 1) / nsplit;
        const int j0 = grp * jlen, j1 = min(nl, j0 + jlen);
        uint32_t ngt = 0u, neq = 0u;
#pragma unroll 4
        for (int jj = j0; jj < j1; ++jj) {
          const uint32_t o = glist[jj];
          ngt += o > k;
          neq += o == k;
        }
        if (i < nl && (ngt | neq) != 0u) {
          atomicAdd(&sh.cgt[i], ngt);
          atomicAdd(&sh.ceq[i], neq);
        }
      }
      __syncthreads();
      if (tid < nl) {
        const uint32_t ngt = sh.cgt[tid], neq = sh.ceq[tid];
        const int r = sh.grank[tid];
        if (ngt + neq < need) {
          atomicAdd(&sh.rc_gtc[r], 1u);
        } else if (ngt < need) {  // equal keys agree
          sh.ustar = glist[tid];
          sh.need_eq = need - ngt;
          atomicAdd(&sh.rc_eqc[r], 1u);
        }
      }
      __syncthreads();
      ustar = sh.ustar;
      need = sh.need_eq;
    } else {
      uint32_t lo_k = 0xFFFFFFFFu, hi_k = 0u;
      for (int i = tid; i < nl; i += TOPK_THREADS) {
        lo_k = min(lo_k, glist[i]);
        hi_k = max(hi_k, glist[i]);
      }
      lo_k = __reduce_min_sync(0xffffffffu, lo_k);
      hi_k = __reduce_max_sync(0xffffffffu, hi_k);
      if (lane == 0) {
        atomicMin(&sh.kmin, lo_k);
        atomicMax(&sh.kmax, hi_k);
      }
      __syncthreads();
      ustar = exact_passes(sh.kmin, sh.kmax, false, glist, nl);
      for (int g = tid; g < nl; g += TOPK_THREADS) {
        const uint32_t k = glist[g];
        const int r = sh.grank[g];
        if (k > ustar) atomicAdd(&sh.rc_gtc[r], 1u);
        if (k == ustar) atomicAdd(&sh.rc_eqc[r], 1u);
      }
      __syncthreads();
    }
    // 2d. this CTA's output offset: per lower rank, its keys > u* and its
    // share (in rank order) of the keys == u*
    uint32_t* rc_gt = sh.rc_gt;
    uint32_t* rc_gtc = sh.rc_gtc;
    uint32_t* rc_eqc = sh.rc_eqc;
    if (tid == 0) {
      uint32_t sel_base = 0u, eq_seen = 0u, my_take = 0u;
      for (int r = 0; r <= c; ++r) {
        const uint32_t er = rc_eqc[r];
        const uint32_t take = need > eq_seen ? min(er, need - eq_seen) : 0u;
        if (r < c) sel_base += rc_gt[r] + rc_gtc[r] + take;
        if (r == c) my_take = take;
        eq_seen += er;
      }
      sh.sel_base = sel_base;
      sh.take_eq = my_take;
    }
    __syncthreads();
  }
  else {
    // Many candidates: their smallest / largest key over the cluster, then
    // exact passes over every slice with cluster-summed histograms.
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int e = tid; e < n; e += TOPK_THREADS) {
      const uint32_t k = keys[e];
      if (score_bin(key_score(k)) == b0) {
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      atomicMin(&sh.kmin, kmin);
      atomicMax(&sh.kmax, kmax);
    }
    if (CLUSTER) cluster.sync();
    else __syncthreads();
    kmin = 0xFFFFFFFFu;
    kmax = 0u;
    for (int r = 0; r < C; ++r) {
      const TopkShared* shr = CLUSTER ? cluster.map_shared_rank(&sh, r) : &sh;
      kmin = min(kmin, shr->kmin);
      kmax = max(kmax, shr->kmax);
    }
    ustar = exact_passes(kmin, kmax, true, nullptr, 0);
    // this slice's keys > u* and == u*, exchanged for the output offsets
    uint32_t g = 0u, q_eq = 0u;
    for (int e = tid; e < n; e += TOPK_THREADS) {
      const uint32_t k = keys[e];
      g += k > ustar;
      q_eq += k == ustar;
    }
    g = __reduce_add_sync(0xffffffffu, g);
    q_eq = __reduce_add_sync(0xffffffffu, q_eq);
    if (lane == 0) {
      atomicAdd(&sh.rc_gtc[c], g);
      atomicAdd(&sh.rc_eqc[c], q_eq);
    }
    if (CLUSTER) cluster.sync();
    else __syncthreads();
    if (tid == 0) {
      uint32_t sel_base = 0u, eq_seen = 0u, my_take = 0u;
      for (int r = 0; r <= c; ++r) {
        const TopkShared* shr = CLUSTER ? cluster.map_shared_rank(&sh, r) : &sh;
        const uint32_t gr = shr->rc_gtc[r], er = shr->rc_eqc[r];
        const uint32_t take = need > eq_seen ? min(er, need - eq_seen) : 0u;
        if (r < c) sel_base += gr + take;
        if (r == c) my_take = take;
        eq_seen += er;
      }
      sh.sel_base = sel_base;
      sh.take_eq = my_take;
    }
    __syncthreads();
  }

  // 3. The picks in index order, in rounds of 4 * TOPK_THREADS keys: in a
  // round thread t owns the 4 consecutive keys from 4 * TOPK_THREADS * r +
  // 4 t (one 16-byte shared-memory read), counts its keys > u* and == u*,
  // and one block scan of both counts places every thread: it writes its
  // keys > u* and the ties that still fall within this CTA's share, in
  // order.
  const uint32_t take_cta = sh.take_eq;
  uint32_t out_base = sh.sel_base;  // output position of this round's first pick
  uint32_t eq_base = 0u;            // ties of this slice in earlier rounds
  int32_t* dst = kv_idx + row * bsa;
  for (int r0 = 0; r0 < n; r0 += 4 * TOPK_THREADS) {
    const int e0 = r0 + 4 * tid;
    uint32_t k[4];
    if (e0 + 3 < n) {
      const uint4 v = *reinterpret_cast<const uint4*>(keys + e0);
      k[0] = v.x;
      k[1] = v.y;
      k[2] = v.z;
      k[3] = v.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) k[u] = e0 + u < n ? keys[e0 + u] : 0u;
    }
    uint32_t g = 0u, q_eq = 0u;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool valid = e0 + u < n;
      g += valid && k[u] > ustar;
      q_eq += valid && k[u] == ustar;
    }
    // both counts in one scan: (gt << 16) | eq (per-round counts <= 4096)
    const uint32_t packed = (g << 16) | q_eq;
    uint32_t tot;
    const uint32_t ex = block_scan_incl(packed, sh, &tot) - packed;
    uint32_t eq_seen = eq_base + (ex & 0xFFFFu);  // ties of this slice before this thread's keys
    uint32_t pos = out_base + (ex >> 16) + min(eq_seen, take_cta) - min(eq_base, take_cta);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (e0 + u >= n) continue;
      bool take = k[u] > ustar;
      if (k[u] == ustar) take = eq_seen++ < take_cta;
      if (take) {
        if (pos < (uint32_t)bsa) dst[pos] = (int32_t)(lo + e0 + u);
        ++pos;
      }
    }
    out_base += (tot >> 16) + min(eq_base + (tot & 0xFFFFu), take_cta) - min(eq_base, take_cta);
    eq_base += tot & 0xFFFFu;
  }
  if (c == 0 && tid == 0) kv_count[row] = bsa;
  // every CTA stays until the others are done reading its shared memory
  if (CLUSTER) {
    if (gathered) cluster_wait();
    else cluster.sync();
  }
}

}  // namespace

int64_t topk_max_T() { return (int64_t)TOPK_MAX_CLUSTER * TOPK_MAX_SLICE; }

cudaError_t launch_topk(const float* S_agg, int b, int nkv, int64_t T, int bsa, const uint32_t* hist,
                        int32_t* kv_idx, int32_t* kv_count, int* status, bool pdl, cudaStream_t stream) {
  // (every wait in the kernel is a hardware barrier phase that all threads
  // reach; `status` is only read, to skip the select after an earlier fault)
  if (bsa <= 0 || T <= 0 || bsa > T || T > topk_max_T()) return cudaErrorInvalidValue;
  int C = (int)((T + TOPK_SLICE_TARGET - 1) / TOPK_SLICE_TARGET);
  if (C > TOPK_MAX_CLUSTER) C = TOPK_MAX_CLUSTER;
  if (C < 1) C = 1;
  const int slice = (int)((T + C - 1) / C);
  if (slice > TOPK_MAX_SLICE) return cudaErrorInvalidValue;
  const size_t smem = ((size_t)slice + 2 * TOPK_LIST_MAX) * sizeof(uint32_t);
  auto kern = C == 1 ? topk_kernel<false> : topk_kernel<true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, nkv, b);
  cfg.blockDim = dim3(TOPK_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (C > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = C;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, S_agg, T, bsa, slice, hist, kv_idx, kv_count,
                            static_cast<const int*>(status));
}

}  // namespace quoka
