// Sparse GQA attention on the tcgen05 tensor cores, gathering the selected
// K/V rows while loading them (bf16 in, fp32 accumulate).
//
// [QUOKA §4.2, problem 3] the selected KV is the attention's input, with no
// causal mask over it; the chunk's own keys follow causally:
//   O[b,h,t] = sum_k softmax_k(scale * q . k) v,
//   k over {K[b, j, kv_idx[b, j, n]] : n < kv_count[b, j]} U {Kc[b, j, s] : s <= t},
//   j = floor(h / G).
// (QUOKA = the technical write-up "QUOKA: how it reshapes LLM prefill
// efficiency", bqwf.cn news item 915859.)
//
// This variant serves callers whose workspace has no room for a gathered
// copy of the selected rows; with one, the gather kernel runs first and the
// TMA-streaming kernel (attn_tma.cu) does the attention, faster.
//
// Work split: a CTA takes two 128-row query tiles (Q0, Q1) of one KV head
// (attn_tma.cu instead gives a CTA one query tile and splits its key tiles
// between the two softmax warpgroups); its key tiles are ceil(nsel/128) tiles of selected prior
// rows (read in place through the sorted index list; rows past nsel are
// zero-filled and masked) followed by ceil(nchunk/128) tiles of the chunk's
// own keys. When the grid would fill less than half of the GPU, the key
// tiles are split between the two CTAs of a cluster, and the partial results
// are combined through distributed shared memory.
//
// Warp roles (544 threads):
//   warps 0-7   softmax of Q0 (warps 0-3) and Q1 (warps 4-7), one query row
//               per thread (attn_common.cuh); final normalisation, combine,
//               store.
//   warp 8      TMEM allocation and the single-thread MMA issue, ordered
//               QK0(i), PV1(i-1), QK1(i), PV0(i).
//   warps 9-16  loaders (256 threads): cp.async 16-byte row chunks, gathered
//               by index, into a 2-stage K/V ring in the 128-byte-swizzled
//               UMMA layout (zero-fill past the end of a list); each thread
//               owns one 16-byte column chunk of 8 rows per tile, prefetches
//               the next tile's gather indices, and its arrival on the stage
//               barrier fires when its copies land. The Q tiles are 4-D TMA
//               boxes (no multicast). Row gathers need many issuing threads:
//               measured on B200, 16-byte cp.async gathers reach ~47 GB/s per
//               SM from 256 threads but ~24 GB/s from 96, and TMA
//               tile::gather4 ~16 GB/s.
// Every wait is bounded: a wait that gives up records QUOKA_ERR_TIMEOUT and
// the CTA unwinds (waits for in-flight copies and MMAs, frees TMEM).
#include "attn_common.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace quoka {

using namespace sm100;
using namespace attn;

namespace {

constexpr int AT_STAGES = 2;     // K/V ring depth
constexpr int AT_THREADS = 544;
constexpr int AT_MMA_WARP = 8;
constexpr int AT_LD_WARP0 = 9;
constexpr int AT_LD_THREADS = 256;
constexpr int LD_ROWS = N * 16 / AT_LD_THREADS;  // rows per loader thread per tile (8)

// TMA tensor map of the queries (4-D boxes of 64 columns x 128 rows).
struct AttnMaps {
  CUtensorMap q;
};

struct __align__(1024) AttnSmem {
  uint8_t q[2][TILE_BYTES];
  uint8_t kv[AT_STAGES][2][TILE_BYTES];  // [stage][0 = K, 1 = V]
  uint64_t q_full;
  uint64_t kv_full[AT_STAGES];
  uint64_t kv_empty[AT_STAGES];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_final;
  uint64_t mma_done;
  uint64_t xfer_free;   // (rank 1) rank 0's landing zone is free
  uint64_t xfer_full;   // (rank 0) rank 1's partial results have landed
  uint32_t tmem_base;
  int abort;
  uint64_t wait_ns;     // bound of every wait
};
// The split-KV landing zone in rank 0 reuses the K/V ring (partial O, fp32,
// [tile][row][128] with a per-row chunk rotation) and the Q area (m, l).
static_assert(sizeof(float) * 2 * 128 * D <= AT_STAGES * 2 * TILE_BYTES, "landing zone");

__global__ void __launch_bounds__(AT_THREADS, 1)
attn_gather_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a, int nsplit) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(align_smem_1024(smem_raw));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.y, bi = blockIdx.z;
  const int G = a.nq / a.nkv;
  const int split = nsplit > 1 ? (int)cluster_ctarank() : 0;
  const int pair = blockIdx.x / nsplit;
  const int ntt = (a.BCP + 127) / 128;  // row tiles per query head
  TileInfo ti[2];
  pair_tiles(pair, j, G, ntt, ti);
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int nsel = a.bsa > 0 ? max(0, min(a.kv_count[kvrow], a.bsa)) : 0;
  const int max_t0 = ti[1].valid ? max(ti[0].t0, ti[1].t0) : ti[0].t0;
  const int nchunk = min(a.BCP, max_t0 + 128);
  const int ntile_sel = (nsel + N - 1) / N;
  const int ntile_chk = (nchunk + N - 1) / N;
  const int nT = ntile_sel + ntile_chk;
  const int per = (nT + nsplit - 1) / nsplit;
  const int first = min(nT, split * per);
  const int ntiles = min(nT, first + per) - first;  // key tiles of this CTA (may be 0)

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < AT_STAGES; ++s) {
      mbar_init(&sm.kv_full[s], AT_LD_THREADS);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&sm.s_full[w], 1);
      mbar_init(&sm.p_full[w], 128);
    }
    mbar_init(&sm.o_final, 1);
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.xfer_free, 1);
    mbar_init(&sm.xfer_full, SOFTMAX_THREADS);
    sm.abort = 0;
    sm.wait_ns = kWaitLimitNs;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == AT_MMA_WARP) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  if (nsplit > 1) {
    // both CTAs' barriers must be initialised before any remote arrive
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp >= AT_LD_WARP0) {
    // ------------------------------------------------------------ loaders
    const int lt = tid - AT_LD_WARP0 * 32;  // 0..255
    const int c = lt & 15;                   // 16-byte chunk of a row
    const int rg = lt >> 4;                  // rows rg, rg + 16, ... of a tile
    if (lt == 0) {
      tma_prefetch_desc(&maps.q);
      mbar_arrive_expect_tx(&sm.q_full, (ti[1].valid ? 2 : 1) * TILE_BYTES);
      for (int w = 0; w < 2; ++w) {
        if (!ti[w].valid) continue;
        const uint32_t q_s = smem_u32(sm.q[w]);
        tma_load_4d(q_s, &maps.q, &sm.q_full, 0, ti[w].t0, ti[w].h, bi);
        tma_load_4d(q_s + ATOM_BYTES, &maps.q, &sm.q_full, 64, ti[w].t0, ti[w].h, bi);
      }
    }
    const bf16* Kb = static_cast<const bf16*>(a.K.data) + bi * a.K.sb + j * a.K.sh + c * 8;
    const bf16* Vb = static_cast<const bf16*>(a.V.data) + bi * a.V.sb + j * a.V.sh + c * 8;
    const bf16* Kcb = static_cast<const bf16*>(a.Kc.data) + bi * a.Kc.sb + j * a.Kc.sh + c * 8;
    const bf16* Vcb = static_cast<const bf16*>(a.Vc.data) + bi * a.Vc.sb + j * a.Vc.sh + c * 8;
    const int32_t* idx = a.kv_idx + kvrow * a.bsa;
    bool bad_index = false;
    // gather indices of this thread's rows of selected tile `gi` (-1: past nsel)
    int32_t tau[LD_ROWS];
    auto fetch_idx = [&](int gi) {
#pragma unroll
      for (int k = 0; k < LD_ROWS; ++k) {
        const int n = gi * N + rg + 16 * k;
        tau[k] = n < nsel ? __ldg(idx + n) : -1;
      }
    };
    if (ntiles > 0 && first < ntile_sel) fetch_idx(first);
    bool alive = true;
    for (int it = 0; it < ntiles && alive; ++it) {
      const int s = it % AT_STAGES;
      const int gi = first + it;
      if (it >= AT_STAGES) alive = warp_wait(&sm.kv_empty[s], ((it / AT_STAGES) - 1) & 1, sm, a.status, 11);
      if (!alive) break;
      const uint32_t k_s = smem_u32(sm.kv[s][0]), v_s = smem_u32(sm.kv[s][1]);
      if (gi < ntile_sel) {
#pragma unroll
        for (int k = 0; k < LD_ROWS; ++k) {
          const int r = rg + 16 * k;
          const int32_t tv = tau[k];
          const bool ok = tv >= 0 && (int64_t)tv < a.T;
          bad_index |= (tv != -1) && !ok;
          const uint32_t off = sw128_offset(r, c, 128);
          cp_async_16(k_s + off, ok ? Kb + (int64_t)tv * a.K.st : Kcb, ok ? 16u : 0u);
          cp_async_16(v_s + off, ok ? Vb + (int64_t)tv * a.V.st : Vcb, ok ? 16u : 0u);
        }
        if (gi + 1 < ntile_sel && it + 1 < ntiles) fetch_idx(gi + 1);
      } else {
        const int p0 = (gi - ntile_sel) * N;
#pragma unroll
        for (int k = 0; k < LD_ROWS; ++k) {
          const int r = rg + 16 * k;
          const int p = p0 + r;
          const bool ok = p < nchunk;
          const uint32_t off = sw128_offset(r, c, 128);
          cp_async_16(k_s + off, Kcb + (int64_t)(ok ? p : 0) * a.Kc.st, ok ? 16u : 0u);
          cp_async_16(v_s + off, Vcb + (int64_t)(ok ? p : 0) * a.Vc.st, ok ? 16u : 0u);
        }
      }
      cp_async_arrive_noinc(&sm.kv_full[s]);
    }
    cp_async_wait<0>();
    if (bad_index) latch_status(a.status, 6 /* QUOKA_ERR_BOUNDS */);
  } else if (warp == AT_MMA_WARP) {
    // ------------------------------------------------------------ MMA issue
    // The whole warp runs this loop in step (waits on every lane, warp-uniform
    // results); one elected lane issues each MMA and commit.
    const uint32_t q0 = smem_u32(sm.q[0]), q1 = smem_u32(sm.q[1]);
    const bool v0 = ti[0].valid, v1 = ti[1].valid;
    auto qk = [&](int w, int s) {
      issue_qk(tmem + 128u * w, w ? q1 : q0, smem_u32(sm.kv[s][0]));
      umma_commit_warp(&sm.s_full[w]);
    };
    auto pv = [&](int w, int s, bool acc) {
      issue_pv(tmem + 256u + 128u * w, tmem + 128u * w, smem_u32(sm.kv[s][1]), acc);
    };
    int where = 21;
    bool alive = mbar_wait_warp(&sm.q_full, 0, &sm.abort);
    for (int it = 0; it < ntiles && alive; ++it) {
      const int s = it % AT_STAGES;
      const int sp = (it + AT_STAGES - 1) % AT_STAGES;
      where = 22;
      alive = mbar_wait_warp(&sm.kv_full[s], (it / AT_STAGES) & 1, &sm.abort);
      if (!alive) break;
      fence_proxy_async_smem();  // the cp.async writes become visible to the tensor core
      tc_fence_after();
      if (v0) qk(0, s);
      if (it > 0) {
        if (v1) {
          where = 23;
          alive = mbar_wait_warp(&sm.p_full[1], (it - 1) & 1, &sm.abort);
          if (!alive) break;
          tc_fence_after();
          pv(1, sp, it - 1 > 0);
        }
        umma_commit_warp(&sm.kv_empty[sp]);
      }
      if (v1) qk(1, s);
      if (v0) {
        where = 24;
        alive = mbar_wait_warp(&sm.p_full[0], it & 1, &sm.abort);
        if (!alive) break;
        tc_fence_after();
        pv(0, s, it > 0);
      }
    }
    if (alive && ntiles > 0 && v1) {
      where = 25;
      alive = mbar_wait_warp(&sm.p_full[1], (ntiles - 1) & 1, &sm.abort);
      if (alive) {
        tc_fence_after();
        pv(1, (ntiles - 1) % AT_STAGES, ntiles - 1 > 0);
      }
    }
    if (!alive && lane == 0) record_abort(sm, a.status, where);
    umma_commit_warp(&sm.o_final);
    umma_commit_warp(&sm.mma_done);
    const bool drained = __all_sync(0xffffffffu, mbar_drain(&sm.mma_done, 0));
    if (lane == 0) {
      if (!drained) record_abort(sm, a.status, 26);
      // rank 0: every MMA is done, so its K/V ring and Q area may now take
      // rank 1's partial results
      if (nsplit > 1 && split == 0) mbar_arrive_remote(mapa_shared(smem_u32(&sm.xfer_free), 1));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int w = warp >> 2;           // query tile of this warpgroup
    const int r = tid & 127;           // row == TMEM lane
    const int t = ti[w].t0 + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t S = tmem + lane_off + 128u * w;
    const uint32_t O = tmem + lane_off + 256u + 128u * w;
    const float qscale = a.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    bool alive = true;
    const bool active = ti[w].valid != 0;
    for (int it = 0; it < ntiles && alive && active; ++it) {
      alive = warp_wait(&sm.s_full[w], it & 1, sm, a.status, 31 + w);
      if (!alive) break;
      tc_fence_after();
      const int gi = first + it;
      const bool sel_tile = gi < ntile_sel;
      // first key of the tile: selected-list index or chunk position; key c
      // of the tile is visible to row t when it is a selected key below
      // nsel, or a chunk key at a position p < nchunk with p <= t
      const int base_n = sel_tile ? gi * N : (gi - ntile_sel) * N;
      const int lim = sel_tile ? nsel : min(nchunk, t + 1);
      softmax_tile(S, O, it > 0, base_n, lim, qscale, m, l);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[w]);
    }

    // ------------------------------------------------ epilogue / combine
    const bool have = active && ntiles > 0;
    if (alive) alive = warp_wait(&sm.o_final, 0, sm, a.status, 33);
    tc_fence_after();
    const float ln2 = 0.6931471805599453f;
    float* land_o = reinterpret_cast<float*>(&sm.kv[0][0][0]) + (size_t)(w * 128 + r) * D;
    float* land_ml = reinterpret_cast<float*>(&sm.q[0][0]) + (size_t)(w * 128 + r) * 2;
    if (nsplit > 1 && split == 1) {
      // send (O, m, l) of this row to rank 0 once its landing zone is free
      if (alive) alive = warp_wait_cluster(&sm.xfer_free, 0, sm, a.status, 41);
      if (alive) {
        const uint32_t ro = mapa_shared(smem_u32(land_o), 0);
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          float o[32];
          if (have) {
            tmem_ld32(O + 32 * c4, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = 0.f;
          }
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            const int chunk = (32 * c4 + u) >> 2;  // 16-byte chunk 0..31, rotated by row
            st_cluster_v4(ro + (uint32_t)(((chunk + r) & 31) << 4), make_float4(o[u], o[u + 1], o[u + 2], o[u + 3]));
          }
        }
        const uint32_t rml = mapa_shared(smem_u32(land_ml), 0);
        st_cluster_f32(rml, have ? m : -INFINITY);
        st_cluster_f32(rml + 4, have ? l : 0.f);
      }
      mbar_arrive_remote(mapa_shared(smem_u32(&sm.xfer_full), 0));
    } else if (active) {
      float m_o = -INFINITY, l_o = 0.f;
      if (nsplit > 1) {
        if (alive) alive = warp_wait_cluster(&sm.xfer_full, 0, sm, a.status, 42);
        if (alive) {
          m_o = land_ml[0];
          l_o = land_ml[1];
        }
      }
      // warp-uniform from here on (tcgen05.ld is a warp-collective); only
      // the stores are predicated on the row being inside the chunk
      if (alive) {
        const bool row_ok = t < a.BCP;
        const float mm = have ? m : -INFINITY;
        const float ll = have ? l : 0.f;
        const float M = fmaxf(mm, m_o);
        const float f_me = mm == -INFINITY ? 0.f : ex2(mm - M);
        const float f_ot = m_o == -INFINITY ? 0.f : ex2(m_o - M);
        const float L = f_me * ll + f_ot * l_o;
        const float inv = 1.f / L;
        bf16* orow = static_cast<bf16*>(a.O) + (((int64_t)bi * a.nq + ti[w].h) * a.BCP + t) * D;
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          float o[32];
          if (have) {
            tmem_ld32(O + 32 * c4, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = 0.f;
          }
          if (nsplit > 1) {
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
              const int chunk = (32 * c4 + u) >> 2;
              const float4 p = *reinterpret_cast<const float4*>(land_o + 4 * ((chunk + r) & 31));
              o[u] = o[u] * f_me + p.x * f_ot;
              o[u + 1] = o[u + 1] * f_me + p.y * f_ot;
              o[u + 2] = o[u + 2] * f_me + p.z * f_ot;
              o[u + 3] = o[u + 3] * f_me + p.w * f_ot;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] *= f_me;
          }
#pragma unroll
          for (int u = 0; u < 32; u += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(o[u] * inv, o[u + 1] * inv);
            pk.y = pack_bf16x2(o[u + 2] * inv, o[u + 3] * inv);
            pk.z = pack_bf16x2(o[u + 4] * inv, o[u + 5] * inv);
            pk.w = pack_bf16x2(o[u + 6] * inv, o[u + 7] * inv);
            if (row_ok) *reinterpret_cast<uint4*>(orow + 32 * c4 + u) = pk;
          }
        }
        if (row_ok && a.lse != nullptr)
          a.lse[((int64_t)bi * a.nq + ti[w].h) * a.BCP + t] = (M + __log2f(L)) * ln2;
      }
    } else if (nsplit > 1) {
      // an empty second tile on rank 0 still consumes its landing signal
      warp_wait_cluster(&sm.xfer_full, 0, sm, a.status, 43);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == AT_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attn_tc_gather(const AttnArgs& a, cudaStream_t stream) {
  if (a.d != D || a.no_chunk) return cudaErrorNotSupported;
  AttnMaps maps;
  if (!encode_bf16_4d(&maps.q, a.Q.data, D, a.BCP, a.nq, a.b, a.Q.st, a.Q.sh, a.Q.sb, 128))
    return cudaErrorNotSupported;
  const size_t smem = sizeof(AttnSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int G = a.nq / a.nkv;
  const int R = G * ((a.BCP + 127) / 128);
  const int npairs = (R + 1) / 2;
  const long ctas = (long)npairs * a.nkv * a.b;
  int num_sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int nsplit = (2 * ctas <= num_sms) ? 2 : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(npairs * nsplit, a.nkv, a.b);
  cfg.blockDim = dim3(AT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_gather_kernel, maps, a, nsplit);
}

}  // namespace quoka
