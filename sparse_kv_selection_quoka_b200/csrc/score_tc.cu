// Key scoring on the tcgen05 tensor cores, K streamed from HBM once by TMA.
//
// [QUOKA §2.2] cosine score, [QUOKA §2.3] S = Q_group . K_norm^T reduced by a
// max over the NQ chosen queries:
//   S_agg[b, j, tau] = max_i (Q_group[b, j, i] . K[b, j, tau]) / |K[b, j, tau]|
// The max commutes with the positive factor 1/|k|, so each key is divided
// once, after the max. (QUOKA = the technical write-up "QUOKA: how it
// reshapes LLM prefill efficiency", bqwf.cn news item 915859.)
//
// Precision: K is bf16 (exact on the tensor core); the fp32 group means are
// split into bf16 hi + lo and both halves are multiplied, so the score
// carries ~16 significant bits of the query instead of 8:
//   D[key, i] = K . hi_i,  D[key, NQp + i] = K . lo_i  (NQp = NQ rounded up to 16),  s_i = D[key,i] + D[key,NQp+i]
// with fp32 accumulation; |k| is summed in fp32 from the same shared-memory
// tile the tensor core reads.
//
// Work split: each CTA owns a contiguous range of 128-key tiles of one
// (batch, KV head); the grid has about one CTA per SM.
// Warp roles (448 threads):
//   warp 0      TMA producer: 4-D tensor map over the (possibly strided) K
//               view, two 64-column boxes per tile in the 128-byte swizzle,
//               into a ring of up to 6 stages (no multicast); it starts
//               before the query groups are staged;
//   warp 1      TMEM allocation and single-thread MMA issue,
//               M=128 keys x N=2*NQp x K=128, into accumulator tile % 3;
//   warps 2-13  epilogue, three warpgroups taking the tiles round-robin,
//               each with its own TMEM accumulator (one warpgroup alone is
//               latency-bound well below the HBM rate): thread = key (TMEM
//               lane): max over the NQ columns, |k| from shared memory,
//               S_agg store, histogram of the value buckets. A stage is
//               released once its warpgroup has read |k| from it.
// Measured on B200 (Qwen-shaped layer): computing |k|^2 on the tensor core
// instead (the diagonal of a K K^T product) costs more MMA time per tile
// than it saves.
// Every wait is bounded (by the launch's wait limit, 2 s unless a test sets
// another); a wait that gives up records QUOKA_ERR_TIMEOUT and a fault-site
// code, and the CTA unwinds: the producer waits for the tile loads it issued
// to land, the MMA warp for its products, TMEM is freed, and the CTA exits.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.cuh"

namespace quoka {

using namespace sm100;

namespace {

constexpr int SC_D = 128;
constexpr int SC_KEYS = 128;
constexpr int SC_EPI = 3;                        // epilogue warpgroups (tiles round-robin)
constexpr int SC_THREADS = 64 + 128 * SC_EPI;
constexpr int SC_MAX_STAGES = 6;
constexpr int SC_TILE_BYTES = SC_KEYS * SC_D * 2;  // 32 KiB
constexpr int SC_ATOM = SC_KEYS * 128;             // one 64-column atom of a K tile

struct ScoreBars {
  uint64_t full[SC_MAX_STAGES];
  uint64_t empty[SC_MAX_STAGES];
  uint64_t tfull[SC_EPI];   // accumulator g holds a finished tile (g = tile % SC_EPI)
  uint64_t tempty[SC_EPI];  // epilogue warpgroup g has read accumulator g
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

struct ScoreArgs {
  const uint16_t* qg_hilo;  // (b, nkv, 2*NQ, d) bf16: rows [0,NQ) hi, [NQ,2NQ) lo
  float* s_agg;             // (b, nkv, T)
  uint32_t* hist;           // (b, nkv, TOPK_HIST_BINS): histogram of score_bin(S_agg)
  int* status;
  int64_t T;
  int NQ, NQp, nstages, tiles_per_cta, ntiles;
  int nepi;                 // epilogue warpgroups in use (TMEM holds one accumulator each)
  uint32_t tmem_cols;
  int key_norm;             // 1: divide by |k| (cosine score); 0: plain dot product
  uint64_t wait_ns;         // bound of every wait
  int inject;               // test hook: accumulator 0's release expects one arrival more than it gets
};

__device__ __forceinline__ void sc_abort(ScoreBars& sb, int* status, int where) {
  sb.abort = 1;
  latch_status(status, 5 /* QUOKA_ERR_TIMEOUT */);
  latch_where(status, where);
}

__device__ __forceinline__ bool sc_warp_wait(uint64_t* bar, uint32_t parity, ScoreBars& sb, int* status,
                                             int where, uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, &sb.abort, limit_ns);
  const bool all_ok = __all_sync(0xffffffffu, ok);
  if (!all_ok && (threadIdx.x & 31) == 0) sc_abort(sb, status, where);
  return all_ok;
}

__global__ void __launch_bounds__(SC_THREADS, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmap, const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  const int N = 2 * a.NQp;                         // MMA N: hi rows then lo rows
  const int ACC = N;                               // columns of one accumulator
  uint8_t* qg_s = base;                            // [2 atoms][N rows][128 B]
  const int qg_bytes = ((N * 256) + 1023) & ~1023;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(base + qg_bytes);  // [TOPK_HIST_BINS]
  uint8_t* ring = base + qg_bytes + TOPK_HIST_BINS * 4;             // [nstages][32 KiB]
  ScoreBars& sb = *reinterpret_cast<ScoreBars*>(ring + (size_t)a.nstages * SC_TILE_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.y, bi = blockIdx.z, nkv = gridDim.y;
  const int64_t row = (int64_t)bi * nkv + j;
  pdl_trigger();
  const int t_begin = blockIdx.x * a.tiles_per_cta;
  const int n = max(0, min(a.ntiles, t_begin + a.tiles_per_cta) - t_begin);
  const int NS = a.nstages;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sb.full[s], 1);
      // released once the tile's MMAs are done (one commit) and the epilogue
      // warpgroup has read |k| from it (128 arrivals)
      mbar_init(&sb.empty[s], 129);
    }
    for (int q = 0; q < SC_EPI; ++q) {
      mbar_init(&sb.tfull[q], 1);
      // (the test hook makes accumulator 0 wait for an arrival that never comes)
      mbar_init(&sb.tempty[q], (q == 0 && a.inject) ? 129 : 128);
    }
    mbar_init(&sb.done, 1);
    sb.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmap);
  }
  if (warp == 1) {
    tmem_alloc(&sb.tmem_base, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();  // barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = sb.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // (starts at once: the K stream does not depend on the query groups)
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n; ++it) {
        const int s = it % NS;
        if (it >= NS && !mbar_wait(&sb.empty[s], ((it / NS) - 1) & 1, &sb.abort, a.wait_ns)) {
          sc_abort(sb, a.status, 51);
          break;
        }
        const uint32_t dst = smem_u32(ring + (size_t)s * SC_TILE_BYTES);
        mbar_arrive_expect_tx(&sb.full[s], SC_TILE_BYTES);
        const int y = (t_begin + it) * SC_KEYS;
        tma_load_4d(dst, &tmap, &sb.full[s], 0, y, j, bi);
        tma_load_4d(dst + SC_ATOM, &tmap, &sb.full[s], 64, y, j, bi);
        issued = it + 1;
      }
      // Wait (bounded) until the last load into each stage has landed, so that
      // no copy is still writing this CTA's shared memory when it exits, even
      // if a consumer gave up before reading it. In a normal run every load
      // has been consumed already and these return at once.
      for (int s = 0; s < NS; ++s) {
        const int nf = issued > s ? (issued - s + NS - 1) / NS : 0;  // loads into stage s
        if (nf > 0 && !mbar_drain(&sb.full[s], (nf - 1) & 1, a.wait_ns)) sc_abort(sb, a.status, 57);
      }
    }
    __syncwarp();
  }
  const int nstage_threads = SC_THREADS - 32;  // everyone but the producer
  const int st = tid - 32;
  if (warp != 0) {
  // the query groups (and the zeroed histogram) come from the previous kernel
  pdl_wait();
  for (int e = st; e < TOPK_HIST_BINS; e += nstage_threads) hist_s[e] = 0u;
  // B operand: the group means (hi rows then lo rows, each padded to NQp
  // with zero rows) in the K-major 128-byte-swizzled layout.
  {
    const uint16_t* src = a.qg_hilo + row * 2 * a.NQ * SC_D;
    for (int e = st; e < N * 16; e += nstage_threads) {
      const int r = e >> 4, c = e & 15;
      const int half = r >= a.NQp;  // 0 = hi, 1 = lo
      const int i = r - half * a.NQp;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      // (written by the previous kernel: L2-coherent load)
      if (i < a.NQ) v = __ldcg(reinterpret_cast<const uint4*>(src + ((int64_t)(half * a.NQ + i)) * SC_D + c * 8));
      *reinterpret_cast<uint4*>(qg_s + sw128_offset(r, c, N)) = v;
    }
    fence_proxy_async_smem();
  }
  // the query groups and the zeroed histogram are in place (the producer
  // does not take part)
  named_barrier_sync(1, nstage_threads);
  }

  if (warp == 0) {
    // (the producer ran above)
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // The whole warp runs this loop in step (waits on every lane, warp-uniform
    // results); one elected lane issues each MMA and commit.
    const uint32_t idesc = idesc_bf16_f32(SC_KEYS, N, 0, 0);
    const uint32_t qg = smem_u32(qg_s);
    bool alive = true;
    int where = 0;
    const int NE = a.nepi;
    for (int it = 0; it < n && alive; ++it) {
      const int s = it % NS, acc = it % NE;
      where = 52;
      alive = mbar_wait_warp(&sb.full[s], (it / NS) & 1, &sb.abort, a.wait_ns);
      if (alive && it >= NE) {
        where = 53;
        alive = mbar_wait_warp(&sb.tempty[acc], ((it / NE) - 1) & 1, &sb.abort, a.wait_ns);
      }
      if (!alive) break;
      tc_fence_after();
      const uint32_t ks = smem_u32(ring + (size_t)s * SC_TILE_BYTES);
      const uint32_t d = tmem + (uint32_t)(acc * ACC);
#pragma unroll
      for (int kk = 0; kk < SC_D / 16; ++kk) {
        const uint64_t ad = sw128_desc(ks + (kk >> 2) * SC_ATOM + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = sw128_desc(qg + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss_warp(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      umma_commit_warp(&sb.tfull[acc]);
      umma_commit_warp(&sb.empty[s]);  // the stage's share of its release
    }
    if (!alive && lane == 0) sc_abort(sb, a.status, where);
    umma_commit_warp(&sb.done);
    const bool drained = __all_sync(0xffffffffu, mbar_drain(&sb.done, 0, a.wait_ns));
    if (!drained && lane == 0) sc_abort(sb, a.status, 54);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int g = (warp - 2) >> 2;           // epilogue warpgroup: tiles g, g + SC_EPI, ...
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    const int r = q * 32 + lane;             // key within the tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float* out = a.s_agg + row * a.T;
    const int NE = a.nepi;  // warpgroups g >= NE stay idle
    for (int it = g; it < n && g < NE; it += NE) {
      const int s = it % NS, acc = g;
      // |k| first, straight from the landed tile (the TMA writes are visible
      // to threads that observe the stage's barrier), so that the stage is
      // released without waiting for this tile's MMA result
      if (!sc_warp_wait(&sb.full[s], (it / NS) & 1, sb, a.status, 56, a.wait_ns)) break;
      const uint8_t* tile = ring + (size_t)s * SC_TILE_BYTES;
      // eight independent partial sums keep the FMA chain short
      float ss8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 raw = *reinterpret_cast<const uint4*>(tile + sw128_offset(r, c, SC_KEYS));
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __bfloat1622float2(h2[u]);
          ss8[2 * u] = fmaf(f.x, f.x, ss8[2 * u]);
          ss8[2 * u + 1] = fmaf(f.y, f.y, ss8[2 * u + 1]);
        }
      }
      const float ss = ((ss8[0] + ss8[1]) + (ss8[2] + ss8[3])) + ((ss8[4] + ss8[5]) + (ss8[6] + ss8[7]));
      mbar_arrive(&sb.empty[s]);
      // then the tile's scores against the group means, from TMEM
      if (!sc_warp_wait(&sb.tfull[acc], (it / NE) & 1, sb, a.status, 55, a.wait_ns)) break;
      tc_fence_after();
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      const uint32_t tbase = tmem + lane_off + (uint32_t)(acc * ACC);
      for (int c0 = 0; c0 < a.NQp; c0 += 16) {
        float hi[16], lo[16];
        tmem_ld16(tbase + c0, hi);
        tmem_ld16(tbase + a.NQp + c0, lo);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (c0 + u < a.NQ) mx4[u & 3] = fmaxf(mx4[u & 3], hi[u] + lo[u]);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      tc_fence_before();
      mbar_arrive(&sb.tempty[acc]);
      const int64_t key = (int64_t)(t_begin + it) * SC_KEYS + r;
      const float score = a.key_norm ? mx / fmaxf(sqrtf(ss), 1e-12f) : mx;
      if (key < a.T) out[key] = score;
      // first digit of the top-k select: the score's 12-bit value bucket,
      // counted once per distinct bucket within the warp
      const bool counted = key < a.T;
      const uint32_t bin = score_bin(score);
      const uint32_t act = __ballot_sync(0xffffffffu, counted);
      if (counted) {
        const uint32_t peers = __match_any_sync(act, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist_s[bin], (uint32_t)__popc(peers));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
  // fold this CTA's histogram into the head's (zeroed by the previous kernel)
  pdl_wait();
  uint32_t* gh = a.hist + row * TOPK_HIST_BINS;
  for (int e = tid; e < TOPK_HIST_BINS; e += SC_THREADS) {
    const uint32_t v = hist_s[e];
    if (v != 0u) atomicAdd(gh + e, v);
  }
}

}  // namespace

cudaError_t launch_score_tc(int d, Strided K, int b, int nkv, int64_t T, const uint16_t* Qg_hilo, int NQ,
                            float* S_agg, uint32_t* hist, int* status, bool pdl, bool key_norm,
                            cudaStream_t stream) {
  if (d != SC_D || NQ < 1 || NQ > 128 || T <= 0 || T > (int64_t)INT32_MAX - SC_KEYS) return cudaErrorNotSupported;
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;

  CUtensorMap tmap;
  const cuuint64_t dims[4] = {(cuuint64_t)SC_D, (cuuint64_t)T, (cuuint64_t)nkv, (cuuint64_t)b};
  const cuuint64_t strides[3] = {(cuuint64_t)K.st * 2, (cuuint64_t)K.sh * 2, (cuuint64_t)K.sb * 2};
  const cuuint32_t box[4] = {64, SC_KEYS, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(K.data), dims, strides, box,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorNotSupported;

  ScoreArgs a;
  a.qg_hilo = Qg_hilo;
  a.s_agg = S_agg;
  a.hist = hist;
  a.status = status;
  a.key_norm = key_norm ? 1 : 0;
  const WaitHooks hooks = wait_hooks();
  a.wait_ns = hooks.wait_ns;
  a.inject = hooks.inject == INJECT_SCORE_TC ? 1 : 0;
  a.T = T;
  a.NQ = NQ;
  a.NQp = (NQ + 15) / 16 * 16;  // the epilogue reads 16-column groups
  const int N = 2 * a.NQp;
  const int acc_cols = N;
  a.nepi = 512 / acc_cols < SC_EPI ? 512 / acc_cols : SC_EPI;  // N <= 256: at least 1
  uint32_t cols = 32;
  while (cols < (uint32_t)(a.nepi * acc_cols)) cols <<= 1;
  a.tmem_cols = cols;
  const int qg_bytes = ((N * 256) + 1023) & ~1023;
  const int smem_cap = 227 * 1024;
  const int bars = (int)sizeof(ScoreBars) + 1024;
  a.nstages = (smem_cap - qg_bytes - TOPK_HIST_BINS * 4 - bars) / SC_TILE_BYTES;
  if (a.nstages > SC_MAX_STAGES) a.nstages = SC_MAX_STAGES;
  if (a.nstages < 2) return cudaErrorNotSupported;
  a.ntiles = (int)((T + SC_KEYS - 1) / SC_KEYS);

  int num_sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  // at most one CTA per SM in total (one CTA fills an SM's shared memory)
  int per_head = num_sms / (nkv * b);
  if (per_head > a.ntiles) per_head = a.ntiles;
  if (per_head < 1) per_head = 1;
  a.tiles_per_cta = (a.ntiles + per_head - 1) / per_head;
  per_head = (a.ntiles + a.tiles_per_cta - 1) / a.tiles_per_cta;

  const size_t smem =
      (size_t)qg_bytes + TOPK_HIST_BINS * 4 + (size_t)a.nstages * SC_TILE_BYTES + sizeof(ScoreBars) + 1024;
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(per_head, nkv, b);
  cfg.blockDim = dim3(SC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, score_tc_kernel, tmap, a);
}

}  // namespace quoka
