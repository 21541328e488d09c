// Sparse GQA attention on the tcgen05 tensor cores (bf16 in, fp32 accumulate).
//
// [QUOKA §4.2, problem 3] the selected KV is the attention's input, with no
// causal mask over it; the chunk's own keys follow causally:
//   O[b,h,t] = sum_k softmax_k(scale * q . k) v,
//   k over {K[b, j, kv_idx[b, j, n]] : n < kv_count[b, j]} U {Kc[b, j, s] : s <= t},
//   j = floor(h / G).
// (QUOKA = the technical write-up "QUOKA: how it reshapes LLM prefill
// efficiency", bqwf.cn news item 915859.)
//
// Work split. The query rows of one KV head j are cut into 128-row tiles
// (one query head, 128 consecutive chunk positions each); a CTA takes two
// such tiles (Q0, Q1) of the same KV head, so every K/V tile it brings in
// feeds two 128x128x128 QK^T and two PV products. The key tiles of a CTA
// are ceil(nsel/128) tiles of selected prior rows (rows past nsel are
// masked) followed by ceil(nchunk/128) tiles of the chunk's own keys. When
// the grid would fill less than half of the GPU, the key tiles are split
// between the two CTAs of a cluster, and the partial results are combined
// through distributed shared memory.
//
// Warp roles (320 or 544 threads):
//   warps 0-3   softmax of Q0, warps 4-7 softmax of Q1: thread r owns query
//               row r = TMEM lane r. Two passes over its S row in TMEM (row
//               max, then exp2 on the MUFU); P is written back as bf16 over
//               the S columns it has consumed, and is the A operand of PV
//               straight from TMEM. The running max is only moved (and the O
//               accumulator rescaled in TMEM) when it grows by more than 2^8,
//               so rescales are rare. Final normalisation, combine and store.
//   warp 8      TMEM allocation and the single-thread MMA issue, ordered
//               QK0(i), PV1(i-1), QK1(i), PV0(i): while one softmax group
//               works, the tensor core runs the other group's products.
//   Two loader variants (a template parameter):
//   (TMA)       warp 9 issues TMA boxes: the selected keys come from a
//               contiguous copy made by the gather kernel just before (so
//               they are L2-resident), the chunk keys and Q from the inputs.
//               320 threads. Used whenever the workspace holds the copy.
//   (gather)    warps 9-16  loaders (256 threads): cp.async 16-byte row chunks, gathered
//               by index, into a 2-stage K/V ring in the 128-byte-swizzled
//               UMMA layout (zero-fill past the end of a list); each thread
//               owns one 16-byte column chunk of 8 rows per tile, prefetches
//               the next tile's gather indices, and its arrival on the stage
//               barrier fires when its copies land. The Q tiles are 4-D TMA
//               boxes (no multicast). Row gathers need many issuing threads:
//               measured on B200, 16-byte cp.async gathers reach ~47 GB/s per
//               SM from 256 threads but ~24 GB/s from 96, and TMA
//               tile::gather4 ~16 GB/s.
// TMEM: S0 | S1 | O0 | O1, 128 columns each (512).
// Every wait is bounded: a wait that gives up records QUOKA_ERR_TIMEOUT and
// the CTA unwinds (waits for in-flight copies and MMAs, frees TMEM).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.cuh"

namespace quoka {

using namespace sm100;

namespace {

constexpr int AT_D = 128;        // head dim
constexpr int AT_N = 128;        // keys per tile
constexpr int AT_STAGES = 2;     // K/V ring depth
template <bool TMA_KV>
struct AttnCfg {
  static constexpr int threads = TMA_KV ? 320 : 544;
  static constexpr int kv_arrivals = TMA_KV ? 1 : 256;  // arrivals per stage fill
};
constexpr int AT_MMA_WARP = 8;
constexpr int AT_LD_WARP0 = 9;
constexpr int AT_LD_THREADS = 256;
constexpr int AT_SM_THREADS = 256;
constexpr int LD_ROWS = AT_N * 16 / AT_LD_THREADS;  // rows per loader thread per tile (8)
constexpr int TILE_BYTES = 128 * AT_D * 2;  // 128 rows x 256 B
constexpr int ATOM_BYTES = 128 * 128;       // one 64-column swizzle atom of a 128-row tile
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.f;    // log2 units

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, AT_N, 0, 0);  // A=Q K-major, B=K K-major
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, AT_D, 0, 1);  // A=P (TMEM), B=V MN-major

// TMA tensor maps (4-D boxes of 64 columns x 128 rows): the queries, and for
// the TMA loader the gathered selected K/V (b, nkv, BSA, d) and the chunk's
// K/V (b, nkv, BCP, d).
struct AttnMaps {
  CUtensorMap q, ks, vs, kc, vc;
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
};
// The split-KV landing zone in rank 0 reuses the K/V ring (partial O, fp32,
// [tile][row][128] with a per-row chunk rotation) and the Q area (m, l).
static_assert(sizeof(float) * 2 * 128 * AT_D <= AT_STAGES * 2 * TILE_BYTES, "landing zone");

struct TileInfo {
  int valid, h, t0;
};

// A wait gave up: stop the CTA's other roles and record the fault and the
// waiting site (a small code naming the barrier).
__device__ __forceinline__ void record_abort(AttnSmem& sm, int* status, int where) {
  sm.abort = 1;
  latch_status(status, 5 /* QUOKA_ERR_TIMEOUT */);
  latch_where(status, where);
}

// Warp-uniform bounded wait (every lane polls; all lanes agree on the result).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, AttnSmem& sm, int* status, int where) {
  const bool ok = mbar_wait(bar, parity, &sm.abort);
  const bool all_ok = __all_sync(0xffffffffu, ok);
  if (!all_ok && (threadIdx.x & 31) == 0) record_abort(sm, status, where);
  return all_ok;
}

// The same for a barrier that another CTA of the cluster arrives on.
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity, AttnSmem& sm, int* status,
                                                  int where) {
  bool ok = mbar_try_wait_cluster(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    while (!ok && globaltimer_ns() - t0 < kWaitLimitNs) ok = mbar_try_wait_cluster(bar, parity);
  }
  const bool all_ok = __all_sync(0xffffffffu, ok);
  if (!all_ok && (threadIdx.x & 31) == 0) record_abort(sm, status, where);
  return all_ok;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <bool TMA_KV>
__global__ void __launch_bounds__(AttnCfg<TMA_KV>::threads, 1)
attn_tc_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a, int nsplit) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.y, bi = blockIdx.z;
  const int G = a.nq / a.nkv;
  const int split = nsplit > 1 ? (int)cluster_ctarank() : 0;
  const int pair = blockIdx.x / nsplit;
  const int ntt = (a.BCP + 127) / 128;  // row tiles per query head
  const int R = G * ntt;                // row tiles per KV head

  TileInfo ti[2];
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int r = 2 * pair + w;
    ti[w].valid = r < R;
    ti[w].h = j * G + (r < R ? r / ntt : 0);
    ti[w].t0 = (r < R ? r % ntt : 0) * 128;
  }
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int nsel = a.bsa > 0 ? max(0, min(a.kv_count[kvrow], a.bsa)) : 0;
  const int max_t0 = ti[1].valid ? max(ti[0].t0, ti[1].t0) : ti[0].t0;
  const int nchunk = min(a.BCP, max_t0 + 128);
  const int ntile_sel = (nsel + AT_N - 1) / AT_N;
  const int ntile_chk = (nchunk + AT_N - 1) / AT_N;
  const int nT = ntile_sel + ntile_chk;
  const int per = (nT + nsplit - 1) / nsplit;
  const int first = min(nT, split * per);
  const int ntiles = min(nT, first + per) - first;  // key tiles of this CTA (may be 0)

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < AT_STAGES; ++s) {
      mbar_init(&sm.kv_full[s], AttnCfg<TMA_KV>::kv_arrivals);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&sm.s_full[w], 1);
      mbar_init(&sm.p_full[w], 128);
    }
    mbar_init(&sm.o_final, 1);
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.xfer_free, 1);
    mbar_init(&sm.xfer_full, AT_SM_THREADS);
    sm.abort = 0;
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

  if (TMA_KV && warp == AT_LD_WARP0) {
    // ------------------------------------------------------------ TMA loads
    bool alive = true;
    int issued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.ks);
      tma_prefetch_desc(&maps.vs);
      tma_prefetch_desc(&maps.kc);
      tma_prefetch_desc(&maps.vc);
      mbar_arrive_expect_tx(&sm.q_full, (ti[1].valid ? 2 : 1) * TILE_BYTES);
      for (int w = 0; w < 2; ++w) {
        if (!ti[w].valid) continue;
        const uint32_t q_s = smem_u32(sm.q[w]);
        tma_load_4d(q_s, &maps.q, &sm.q_full, 0, ti[w].t0, ti[w].h, bi);
        tma_load_4d(q_s + ATOM_BYTES, &maps.q, &sm.q_full, 64, ti[w].t0, ti[w].h, bi);
      }
      for (int it = 0; it < ntiles && alive; ++it) {
        const int s = it % AT_STAGES;
        const int gi = first + it;
        if (it >= AT_STAGES && !mbar_wait(&sm.kv_empty[s], ((it / AT_STAGES) - 1) & 1, &sm.abort)) {
          record_abort(sm, a.status, 11);
          alive = false;
          break;
        }
        const uint32_t k_s = smem_u32(sm.kv[s][0]), v_s = smem_u32(sm.kv[s][1]);
        mbar_arrive_expect_tx(&sm.kv_full[s], 2 * TILE_BYTES);
        // selected tiles read the gathered copy (rows past nsel are zero
        // fill or stale copies, masked by the softmax); chunk tiles the chunk
        const bool sel_tile = gi < ntile_sel;
        const CUtensorMap* mk = sel_tile ? &maps.ks : &maps.kc;
        const CUtensorMap* mv = sel_tile ? &maps.vs : &maps.vc;
        const int y = sel_tile ? gi * AT_N : (gi - ntile_sel) * AT_N;
        tma_load_4d(k_s, mk, &sm.kv_full[s], 0, y, j, bi);
        tma_load_4d(k_s + ATOM_BYTES, mk, &sm.kv_full[s], 64, y, j, bi);
        tma_load_4d(v_s, mv, &sm.kv_full[s], 0, y, j, bi);
        tma_load_4d(v_s + ATOM_BYTES, mv, &sm.kv_full[s], 64, y, j, bi);
        issued = it + 1;
      }
      // no copy may still be landing when the CTA exits (matters only when
      // a consumer gave up early): wait, bounded, for the last fill of each
      // stage and for Q
      for (int s = 0; s < AT_STAGES; ++s) {
        const int nf = issued > s ? (issued - s + AT_STAGES - 1) / AT_STAGES : 0;
        if (nf > 0 && !mbar_drain(&sm.kv_full[s], (nf - 1) & 1)) record_abort(sm, a.status, 12);
      }
      if (!mbar_drain(&sm.q_full, 0)) record_abort(sm, a.status, 13);
    }
    __syncwarp();
  } else if (!TMA_KV && warp >= AT_LD_WARP0) {
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
        const int n = gi * AT_N + rg + 16 * k;
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
        const int p0 = (gi - ntile_sel) * AT_N;
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
    if (lane == 0) {
      const uint32_t q0 = smem_u32(sm.q[0]), q1 = smem_u32(sm.q[1]);
      const bool v0 = ti[0].valid, v1 = ti[1].valid;
      auto qk = [&](int w, int s) {
        const uint32_t qs = w ? q1 : q0, ks = smem_u32(sm.kv[s][0]);
#pragma unroll
        for (int kk = 0; kk < AT_D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * ATOM_BYTES + (kk & 3) * 32;
          umma_bf16_ss(tmem + 128u * w, sw128_desc(qs + koff, 16, 1024), sw128_desc(ks + koff, 16, 1024),
                       IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.s_full[w]);
      };
      auto pv = [&](int w, int s, bool acc) {
        const uint32_t vs = smem_u32(sm.kv[s][1]);
#pragma unroll
        for (int kk = 0; kk < AT_N / 16; ++kk)
          umma_bf16_ts(tmem + 256u + 128u * w, tmem + 128u * w + kk * 8,
                       sw128_desc(vs + kk * 2048, ATOM_BYTES, 1024), IDESC_PV, (acc || kk > 0) ? 1u : 0u);
      };
      int where = 21;
      bool alive = mbar_wait(&sm.q_full, 0, &sm.abort);
      for (int it = 0; it < ntiles && alive; ++it) {
        const int s = it % AT_STAGES;
        const int sp = (it + AT_STAGES - 1) % AT_STAGES;
        where = 22;
        alive = mbar_wait(&sm.kv_full[s], (it / AT_STAGES) & 1, &sm.abort);
        if (!alive) break;
        fence_proxy_async_smem();  // the cp.async writes become visible to the tensor core
        tc_fence_after();
        if (v0) qk(0, s);
        if (it > 0) {
          if (v1) {
            where = 23;
            alive = mbar_wait(&sm.p_full[1], (it - 1) & 1, &sm.abort);
            if (!alive) break;
            tc_fence_after();
            pv(1, sp, it - 1 > 0);
          }
          umma_commit(&sm.kv_empty[sp]);
        }
        if (v1) qk(1, s);
        if (v0) {
          where = 24;
          alive = mbar_wait(&sm.p_full[0], it & 1, &sm.abort);
          if (!alive) break;
          tc_fence_after();
          pv(0, s, it > 0);
        }
      }
      if (alive && ntiles > 0 && v1) {
        where = 25;
        alive = mbar_wait(&sm.p_full[1], (ntiles - 1) & 1, &sm.abort);
        if (alive) {
          tc_fence_after();
          pv(1, (ntiles - 1) % AT_STAGES, ntiles - 1 > 0);
        }
      }
      if (!alive) record_abort(sm, a.status, where);
      umma_commit(&sm.o_final);
      umma_commit(&sm.mma_done);
      if (!mbar_drain(&sm.mma_done, 0)) record_abort(sm, a.status, 26);
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
      // first key of the tile: selected-list index or chunk position
      const int base_n = sel_tile ? gi * AT_N : (gi - ntile_sel) * AT_N;
      // key c of the tile is visible to row t: a selected key below nsel, or
      // a chunk key at a position p < nchunk with p <= t
      const int lim = sel_tile ? nsel : min(nchunk, t + 1);
      // rows whose every key of this tile is visible skip the per-key test
      const bool all_vis = base_n + AT_N <= lim;
      // pass 1: row max. TMEM loads are warp-collective, so they stay
      // outside per-row branches; 64 columns per round trip.
      float mx = -INFINITY;
#pragma unroll 1
      for (int h2 = 0; h2 < 2; ++h2) {
        float v[64];
        __syncwarp();
        tmem_ld32(S + 64 * h2, *reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_ld32(S + 64 * h2 + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
        tmem_wait_ld();
        if (all_vis) {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int u = 0; u < 64; ++u) m4[u & 3] = fmaxf(m4[u & 3], v[u]);
          mx = fmaxf(mx, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * qscale);
        } else {
#pragma unroll
          for (int u = 0; u < 64; ++u) {
            const bool vis = base_n + 64 * h2 + u < lim;
            mx = vis ? fmaxf(mx, v[u] * qscale) : mx;
          }
        }
      }
      const float m_cand = fmaxf(m, mx);
      const float m_new = (m_cand > m + RESCALE_THRESHOLD || m == -INFINITY) ? m_cand : m;
      const float corr = (m_new == m) ? 1.f : ex2(m - m_new);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      // pass 2: P = 2^(s - m) in bf16, written over the S columns already read
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int h2 = 0; h2 < 2; ++h2) {
        float v[64];
        __syncwarp();
        tmem_ld32(S + 64 * h2, *reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_ld32(S + 64 * h2 + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
        tmem_wait_ld();
        if (!all_vis) {
#pragma unroll
          for (int u = 0; u < 64; ++u) {
            const bool vis = base_n + 64 * h2 + u < lim;
            v[u] = vis ? v[u] : -INFINITY;
          }
        }
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            const float p0 = ex2(fmaf(v[32 * c2 + u], qscale, -m_use));
            const float p1 = ex2(fmaf(v[32 * c2 + u + 1], qscale, -m_use));
            rs4[(u >> 1) & 3] += p0 + p1;
            pk[u >> 1] = pack_bf16x2(p0, p1);
          }
          __syncwarp();
          tmem_st16(S + 32 * h2 + 16 * c2, pk);
        }
      }
      const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      l = l * corr + rs;
      m = m_new;
      // O holds the products of the previous tiles (complete: they were
      // issued before this tile's QK^T, whose completion we waited for)
      // (warp-uniform condition: the rescale's TMEM traffic is collective)
      if (it > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          float o[32];
          tmem_ld32(O + 32 * c4, o);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] *= corr;
          tmem_st32(O + 32 * c4, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[w]);
    }

    // ------------------------------------------------ epilogue / combine
    const bool have = active && ntiles > 0;
    if (alive) alive = warp_wait(&sm.o_final, 0, sm, a.status, 33);
    tc_fence_after();
    const float ln2 = 0.6931471805599453f;
    float* land_o = reinterpret_cast<float*>(&sm.kv[0][0][0]) + (size_t)(w * 128 + r) * AT_D;
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
        bf16* orow = static_cast<bf16*>(a.O) + (((int64_t)bi * a.nq + ti[w].h) * a.BCP + t) * AT_D;
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

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t stream) {
  if (a.d != AT_D) return cudaErrorNotSupported;
  // with no selected keys every tile is a chunk tile: TMA boxes as well
  const bool tma_kv = a.kv_idx == nullptr || a.bsa == 0;
  AttnMaps maps;
  if (!encode_bf16_4d(&maps.q, a.Q.data, AT_D, a.BCP, a.nq, a.b, a.Q.st, a.Q.sh, a.Q.sb, 128))
    return cudaErrorNotSupported;
  if (tma_kv) {
    if (!encode_bf16_4d(&maps.kc, a.Kc.data, AT_D, a.BCP, a.nkv, a.b, a.Kc.st, a.Kc.sh, a.Kc.sb, 128) ||
        !encode_bf16_4d(&maps.vc, a.Vc.data, AT_D, a.BCP, a.nkv, a.b, a.Vc.st, a.Vc.sh, a.Vc.sb, 128))
      return cudaErrorNotSupported;
    if (a.bsa > 0) {
      // the gathered selected rows (b, nkv, bsa, d); rows past a list's
      // count are masked in the softmax
      if (!encode_bf16_4d(&maps.ks, a.K.data, AT_D, a.bsa, a.nkv, a.b, a.K.st, a.K.sh, a.K.sb, 128) ||
          !encode_bf16_4d(&maps.vs, a.V.data, AT_D, a.bsa, a.nkv, a.b, a.V.st, a.V.sh, a.V.sb, 128))
        return cudaErrorNotSupported;
    } else {
      maps.ks = maps.kc;  // never read: there are no selected tiles
      maps.vs = maps.vc;
    }
  } else {
    maps.ks = maps.vs = maps.kc = maps.vc = maps.q;  // unused by the gather loader
  }
  const size_t smem = sizeof(AttnSmem) + 1024;
  auto kern = tma_kv ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
  cfg.blockDim = dim3(tma_kv ? AttnCfg<true>::threads : AttnCfg<false>::threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, maps, a, nsplit);
}

}  // namespace quoka
