// Sparse GQA attention on the tcgen05 tensor cores over dense K/V tiles
// streamed by TMA (bf16 in, fp32 accumulate).
//
// [QUOKA §4.2, problem 3] the selected KV is the attention's input, with no
// causal mask over it; the chunk's own keys follow causally:
//   O[b,h,t] = sum_k softmax_k(scale * q . k) v,
//   k over {Ksel[b, j, n] : n < kv_count[b, j]} U {Kc[b, j, s] : s <= t},
//   j = floor(h / G),
// where Ksel / Vsel hold the selected rows already gathered (by the gather
// kernel, just before, so that they are L2-resident).
// (QUOKA = the technical write-up "QUOKA: how it reshapes LLM prefill
// efficiency", bqwf.cn news item 915859.)
//
// Work split. The query rows of one KV head j are cut into 128-row tiles
// (one query head, 128 consecutive chunk positions each); a CTA takes two
// such tiles (Q0, Q1) of the same KV head, so every K/V tile it brings in
// feeds two 128x128x128 QK^T and two PV products. Its key tiles are
// ceil(nsel/128) tiles of selected rows (rows past nsel are masked)
// followed by ceil(nchunk/128) tiles of the chunk's own keys. When the grid
// would fill less than half of the GPU, the key tiles are split between the
// two CTAs of a cluster: rank r finalises query tile r, and each rank sends
// its partial (O, m, l) of the other tile to the peer with bulk
// shared-to-shared copies over the cluster (both directions at once).
//
// Warp roles (352 threads):
//   warps 0-7   softmax of Q0 (warps 0-3) and Q1 (warps 4-7), one query row
//               per thread (attn_common.cuh); then normalisation, combine,
//               and the bf16 output tile written to shared memory and
//               stored with TMA.
//   warp 8      TMEM allocation and the single-thread MMA issue, ordered
//               QK0(i), PV1(i-1), QK1(i), PV0(i): while one softmax group
//               works, the tensor core runs the other group's products.
//   warp 9      TMA loads of Q and of the K tiles (2-stage ring; a stage is
//               released as soon as both QK^T products of its tile are done).
//   warp 10     TMA loads of the V tiles (3-stage ring; released after the
//               second PV product). Separate rings keep the next tiles'
//               loads in flight while the current tile is still in use.
// TMEM: S0 | S1 | O0 | O1, 128 columns each (512).
// Every wait is bounded: a wait that gives up records QUOKA_ERR_TIMEOUT and
// the CTA unwinds (waits for in-flight copies and MMAs, frees TMEM).
#include <stddef.h>

#include "attn_common.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace quoka {

using namespace sm100;
using namespace attn;

namespace {

constexpr int KST = 2;  // K ring depth
constexpr int VST = 3;  // V ring depth
constexpr int THREADS = 352;
constexpr int MMA_WARP = 8;
constexpr int KLOAD_WARP = 9;
constexpr int VLOAD_WARP = 10;
// Of every 8 key pairs, how many take the FMA-pipe exp2 in the softmax.
// Measured on B200 (Qwen-shaped layer): 0 and 2 run equally fast, more is
// slower; 0 keeps the kernel free of register spills.
constexpr int SOFTMAX_FMA_PAIRS = 0;
// P of a tile is released to the P V product in this many key ranges.
constexpr int PV_PARTS = 2;
// split-KV payload of one query tile: partial O (fp32, 128 rows x 128, each
// row's 16-byte chunks rotated by the row index) followed by (m, l) per row;
// staged at OUT_OFF of the K/V span, received at IN_OFF
constexpr uint32_t XFER_O_BYTES = 128 * D * 4;
constexpr uint32_t XFER_BYTES = XFER_O_BYTES + 128 * 2 * 4;
constexpr uint32_t XFER_OUT_OFF = 0;
constexpr uint32_t XFER_IN_OFF = 80 * 1024;
constexpr uint32_t XFER_PIECE = 32768;  // bytes per bulk copy

struct Maps {
  CUtensorMap q, ks, vs, kc, vc, o;
};

struct __align__(1024) Smem {
  uint8_t q[2][TILE_BYTES];    // Q tiles; after the last MMA, the bf16 output tiles
  uint8_t k[KST][TILE_BYTES];  // K ring  } one span: after the last MMA, the split-KV
  uint8_t v[VST][TILE_BYTES];  // V ring  }   payload (rank 1 sends, rank 0 receives)
  uint64_t q_full;
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[2], p_part[2][PV_PARTS];
  uint64_t o_final, mma_done;
  uint64_t xfer_free;  // the peer's landing zone is free (its MMAs are done)
  uint64_t xfer_full;  // the peer's partial of this rank's tile has landed
  uint64_t xfer_done;  // the peer holds this rank's payload: the source may go
  uint32_t tmem_base;
  int abort;
};
static_assert(XFER_OUT_OFF + XFER_BYTES <= XFER_IN_OFF && XFER_IN_OFF + XFER_BYTES <= (KST + VST) * TILE_BYTES,
              "split-KV payloads");
static_assert(offsetof(Smem, v) == offsetof(Smem, k) + KST * TILE_BYTES, "K and V rings adjacent");

// Loader of one ring: TMA boxes of the key tiles [first, first + ntiles)
// (selected tiles from the gathered map, then chunk tiles), one stage per
// tile, waiting for a stage to be released before refilling it. Then waits,
// bounded, until its last copies have landed (so none is in flight when the
// CTA exits, even if a consumer gave up).
template <int STAGES>
__device__ __forceinline__ void load_ring(Smem& sm, uint8_t (*ring)[TILE_BYTES], uint64_t* full, uint64_t* empty,
                                          const CUtensorMap* sel_map, const CUtensorMap* chunk_map, int first,
                                          int ntiles, int ntile_sel, int j, int bi, int* status, int where) {
  int issued = 0;
  for (int it = 0; it < ntiles; ++it) {
    const int s = it % STAGES;
    if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1, &sm.abort)) {
      record_abort(sm, status, where);
      break;
    }
    const int gi = first + it;
    const bool sel_tile = gi < ntile_sel;
    const CUtensorMap* m = sel_tile ? sel_map : chunk_map;
    const int y = (sel_tile ? gi : gi - ntile_sel) * N;
    const uint32_t dst = smem_u32(ring[s]);
    mbar_arrive_expect_tx(&full[s], TILE_BYTES);
    tma_load_4d(dst, m, &full[s], 0, y, j, bi);
    tma_load_4d(dst + ATOM_BYTES, m, &full[s], 64, y, j, bi);
    issued = it + 1;
  }
  for (int s = 0; s < STAGES; ++s) {
    const int nf = issued > s ? (issued - s + STAGES - 1) / STAGES : 0;
    if (nf > 0 && !mbar_drain(&full[s], (nf - 1) & 1)) record_abort(sm, status, where + 1);
  }
}

__global__ void __launch_bounds__(THREADS, 1)
attn_tma_kernel(const __grid_constant__ Maps maps, const AttnArgs a, int nsplit) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.y, bi = blockIdx.z;
  const int G = a.nq / a.nkv;
  const int split = nsplit > 1 ? (int)cluster_ctarank() : 0;
  const int pair = blockIdx.x / nsplit;
  const int ntt = (a.BCP + 127) / 128;  // row tiles per query head
  TileInfo ti[2];
  pair_tiles(pair, j, G, ntt, ti);      // ti[0] is always valid

  // Setup and the Q loads touch nothing the previous kernel writes: they run
  // before the grid-dependency wait, overlapping that kernel's tail.
  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&sm.s_full[w], 1);
      for (int c = 0; c < PV_PARTS; ++c) mbar_init(&sm.p_part[w][c], 4);  // one arrival per warp
    }
    mbar_init(&sm.o_final, 1);
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.xfer_free, 1);
    mbar_init(&sm.xfer_full, 1);
    mbar_init(&sm.xfer_done, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // rank r finalises query tile r: it expects the peer's partial of that
    // tile before the peer can send anything
    if (nsplit > 1 && ti[split].valid) mbar_arrive_expect_tx(&sm.xfer_full, XFER_BYTES);
  }
  if (warp == MMA_WARP) {
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
  if (warp == KLOAD_WARP && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.ks);
    tma_prefetch_desc(&maps.kc);
    tma_prefetch_desc(&maps.o);
    mbar_arrive_expect_tx(&sm.q_full, (ti[1].valid ? 2 : 1) * TILE_BYTES);
    for (int w = 0; w < 2; ++w) {
      if (!ti[w].valid) continue;
      const uint32_t q_s = smem_u32(sm.q[w]);
      tma_load_4d(q_s, &maps.q, &sm.q_full, 0, ti[w].t0, ti[w].h, bi);
      tma_load_4d(q_s + ATOM_BYTES, &maps.q, &sm.q_full, 64, ti[w].t0, ti[w].h, bi);
    }
  }

  pdl_wait();  // the gathered rows and their counts come from the previous kernel
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int nsel = a.bsa > 0 ? max(0, min(__ldcg(a.kv_count + kvrow), a.bsa)) : 0;
  const int max_t0 = ti[1].valid ? max(ti[0].t0, ti[1].t0) : ti[0].t0;
  const int nchunk = min(a.BCP, max_t0 + 128);
  const int ntile_sel = (nsel + N - 1) / N;
  const int ntile_chk = (nchunk + N - 1) / N;
  const int nT = ntile_sel + ntile_chk;
  // split: the ranks take halves of the key tiles (each finalises one query
  // tile and waits for the other's partial of it, so an uneven split would
  // only make the longer rank longer)
  const int n0 = nsplit > 1 ? (nT + 1) / 2 : nT;
  const int first = split == 0 ? 0 : n0;
  const int ntiles = split == 0 ? n0 : nT - n0;  // key tiles of this CTA (may be 0)

  if (warp == KLOAD_WARP) {
    // ------------------------------------------------------------ K loads
    if (lane == 0) {
      load_ring<KST>(sm, sm.k, sm.k_full, sm.k_empty, &maps.ks, &maps.kc, first, ntiles, ntile_sel, j, bi,
                     a.status, 11);
      if (!mbar_drain(&sm.q_full, 0)) record_abort(sm, a.status, 13);
    }
    __syncwarp();
  } else if (warp == VLOAD_WARP) {
    // ------------------------------------------------------------ V loads
    if (lane == 0) {
      tma_prefetch_desc(&maps.vs);
      tma_prefetch_desc(&maps.vc);
      load_ring<VST>(sm, sm.v, sm.v_full, sm.v_empty, &maps.vs, &maps.vc, first, ntiles, ntile_sel, j, bi,
                     a.status, 14);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issue
    // The whole warp runs this loop in step (waits on every lane, warp-uniform
    // results); one elected lane issues each MMA and commit.
    const uint32_t q0 = smem_u32(sm.q[0]), q1 = smem_u32(sm.q[1]);
    const bool v1 = ti[1].valid;
    int where = 21;
    // O_w (+)= P_w V for the tile whose P parts complete phase `ph`, each
    // part issued as soon as the softmax releases it
    auto pv = [&](int w, uint32_t v_smem, int ph, bool accumulate) -> bool {
      for (int c = 0; c < PV_PARTS; ++c) {
        if (!mbar_wait_warp(&sm.p_part[w][c], ph, &sm.abort)) return false;
        tc_fence_after();
        issue_pv_part<PV_PARTS>(tmem + 256u + 128u * w, tmem + 128u * w, v_smem, c, accumulate);
      }
      return true;
    };
    bool alive = mbar_wait_warp(&sm.q_full, 0, &sm.abort);
    for (int it = 0; it < ntiles && alive; ++it) {
      const int ks = it % KST, vs = it % VST, vp = (it + VST - 1) % VST;
      where = 22;
      alive = mbar_wait_warp(&sm.k_full[ks], (it / KST) & 1, &sm.abort);
      if (!alive) break;
      tc_fence_after();
      issue_qk(tmem, q0, smem_u32(sm.k[ks]));
      umma_commit_warp(&sm.s_full[0]);
      if (it > 0) {
        if (v1) {
          where = 23;
          alive = pv(1, smem_u32(sm.v[vp]), (it - 1) & 1, it - 1 > 0);
          if (!alive) break;
        }
        umma_commit_warp(&sm.v_empty[vp]);
      }
      if (v1) {
        issue_qk(tmem + 128u, q1, smem_u32(sm.k[ks]));
        umma_commit_warp(&sm.s_full[1]);
      }
      umma_commit_warp(&sm.k_empty[ks]);
      where = 24;
      alive = mbar_wait_warp(&sm.v_full[vs], (it / VST) & 1, &sm.abort);
      if (!alive) break;
      where = 25;
      alive = pv(0, smem_u32(sm.v[vs]), it & 1, it > 0);
      if (!alive) break;
    }
    if (alive && ntiles > 0 && v1) {
      where = 26;
      alive = pv(1, smem_u32(sm.v[(ntiles - 1) % VST]), (ntiles - 1) & 1, ntiles - 1 > 0);
    }
    if (!alive && lane == 0) record_abort(sm, a.status, where);
    umma_commit_warp(&sm.o_final);
    umma_commit_warp(&sm.mma_done);
    const bool drained = __all_sync(0xffffffffu, mbar_drain(&sm.mma_done, 0));
    if (lane == 0) {
      if (!drained) record_abort(sm, a.status, 27);
      // every MMA is done (and every load they waited for has landed), so
      // this rank's K/V span may now take the peer's payload
      if (nsplit > 1) mbar_arrive_remote(mapa_shared(smem_u32(&sm.xfer_free), (uint32_t)(split ^ 1)));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int w = warp >> 2;  // query tile of this warpgroup
    const int r = tid & 127;  // row == TMEM lane
    const int t = ti[w].t0 + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t S = tmem + lane_off + 128u * w;
    const uint32_t O = tmem + lane_off + 256u + 128u * w;
    const float qscale = a.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    bool alive = true;
    const bool active = ti[w].valid != 0;  // warpgroup-uniform
    for (int it = 0; it < ntiles && alive && active; ++it) {
      alive = warp_wait(&sm.s_full[w], it & 1, sm, a.status, 31 + w);
      if (!alive) break;
      tc_fence_after();
      const int gi = first + it;
      const bool sel_tile = gi < ntile_sel;
      // key c of the tile is key number base_n + c of its list; it is
      // visible to row t when it is a selected key below nsel, or a chunk
      // key at a position p < nchunk with p <= t
      const int base_n = (sel_tile ? gi : gi - ntile_sel) * N;
      const int lim = sel_tile ? nsel : min(nchunk, t + 1);
      softmax_tile_split<SOFTMAX_FMA_PAIRS, PV_PARTS>(S, O, it > 0, base_n, lim, qscale, m, l, sm.p_part[w]);
    }

    // ------------------------------------------------ epilogue / combine
    const bool have = active && ntiles > 0;  // warp-uniform: TMEM loads below are collective
    if (alive) alive = warp_wait(&sm.o_final, 0, sm, a.status, 33);
    tc_fence_after();
    uint8_t* span = reinterpret_cast<uint8_t*>(&sm) + offsetof(Smem, k);  // K ring, then V ring
    const uint32_t peer = (uint32_t)(split ^ 1);
    // Split-KV: rank `split` finalises query tile `split`; the warpgroup of
    // the other tile stages its partial and sends it to the peer, so both
    // directions move at once and both warpgroups work.
    const bool send = nsplit > 1 && w != split;
    if (send) {
      if (active) {
        float* out_o = reinterpret_cast<float*>(span + XFER_OUT_OFF) + (size_t)r * D;
        float* out_ml = reinterpret_cast<float*>(span + XFER_OUT_OFF + XFER_O_BYTES) + (size_t)r * 2;
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
            *reinterpret_cast<float4*>(out_o + 4 * ((chunk + r) & 31)) =
                make_float4(o[u], o[u + 1], o[u + 2], o[u + 3]);
          }
        }
        out_ml[0] = have ? m : -INFINITY;
        out_ml[1] = have ? l : 0.f;
        fence_proxy_async_smem();  // the staged payload becomes visible to the bulk copy
        named_barrier_sync(2 + w, 128);
        if (r == 0) {
          bool ok = wait_cluster(&sm.xfer_free, 0);
          if (ok) {
            const uint32_t src = smem_u32(span + XFER_OUT_OFF);
            const uint32_t dst = mapa_shared(smem_u32(span + XFER_IN_OFF), peer);
            const uint32_t bar = mapa_shared(smem_u32(&sm.xfer_full), peer);
            for (uint32_t off = 0; off < XFER_BYTES; off += XFER_PIECE)
              bulk_copy_to_cluster(dst + off, src + off, min(XFER_PIECE, XFER_BYTES - off), bar);
            // the source must stay in place until the peer holds the payload
            ok = wait_cluster(&sm.xfer_done, 0);
          }
          if (!ok) record_abort(sm, a.status, 41);
        }
      }
    } else if (active) {
      float m_o = -INFINITY, l_o = 0.f;  // the peer's part
      const float* in_o = reinterpret_cast<const float*>(span + XFER_IN_OFF) + (size_t)r * D;
      const float* in_ml = reinterpret_cast<const float*>(span + XFER_IN_OFF + XFER_O_BYTES) + (size_t)r * 2;
      if (nsplit > 1) {
        if (alive) alive = warp_wait_cluster(&sm.xfer_full, 0, sm, a.status, 42);
        if (alive) {
          m_o = in_ml[0];
          l_o = in_ml[1];
        }
        if (r == 0) mbar_arrive_remote(mapa_shared(smem_u32(&sm.xfer_done), peer));
      }
      const float mm = have ? m : -INFINITY;
      const float ll = have ? l : 0.f;
      const float M = fmaxf(mm, m_o);
      const float f_me = mm == -INFINITY ? 0.f : ex2(mm - M);
      const float f_ot = m_o == -INFINITY ? 0.f : ex2(m_o - M);
      const float L = f_me * ll + f_ot * l_o;
      const float inv = 1.f / L;
      // the normalised row, bf16, into the tile's 128-byte-swizzled output
      // staging (the Q area: every MMA is done)
      uint8_t* ot = sm.q[w];
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
            const float4 p = *reinterpret_cast<const float4*>(in_o + 4 * ((chunk + r) & 31));
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
          *reinterpret_cast<uint4*>(ot + sw128_offset(r, (32 * c4 + u) >> 3, 128)) = pk;
        }
      }
      if (t < a.BCP && a.lse != nullptr)
        a.lse[((int64_t)bi * a.nq + ti[w].h) * a.BCP + t] = (M + __log2f(L)) * 0.6931471805599453f;
      // rows past the chunk are clipped by the store
      fence_proxy_async_smem();
      named_barrier_sync(2 + w, 128);
      if (r == 0) {
        tma_store_4d(&maps.o, smem_u32(ot), 0, ti[w].t0, ti[w].h, bi);
        tma_store_4d(&maps.o, smem_u32(ot) + ATOM_BYTES, 64, ti[w].t0, ti[w].h, bi);
        bulk_commit_group();
        bulk_wait_group_read_0();  // the staging may go once the copy has read it
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attn_tc(const AttnArgs& a, bool pdl, cudaStream_t stream) {
  if (a.d != D) return cudaErrorNotSupported;
  // rows gathered by index while loading: the other kernel
  if (a.kv_idx != nullptr && a.bsa > 0) return launch_attn_tc_gather(a, stream);
  Maps maps;
  const int64_t oh = (int64_t)a.BCP * D, ob = (int64_t)a.nq * oh;  // O is contiguous
  if (!encode_bf16_4d(&maps.q, a.Q.data, D, a.BCP, a.nq, a.b, a.Q.st, a.Q.sh, a.Q.sb, 128) ||
      !encode_bf16_4d(&maps.kc, a.Kc.data, D, a.BCP, a.nkv, a.b, a.Kc.st, a.Kc.sh, a.Kc.sb, 128) ||
      !encode_bf16_4d(&maps.vc, a.Vc.data, D, a.BCP, a.nkv, a.b, a.Vc.st, a.Vc.sh, a.Vc.sb, 128) ||
      !encode_bf16_4d(&maps.o, a.O, D, a.BCP, a.nq, a.b, D, oh, ob, 128))
    return cudaErrorNotSupported;
  if (a.bsa > 0) {
    // the gathered selected rows (b, nkv, bsa, d)
    if (!encode_bf16_4d(&maps.ks, a.K.data, D, a.bsa, a.nkv, a.b, a.K.st, a.K.sh, a.K.sb, 128) ||
        !encode_bf16_4d(&maps.vs, a.V.data, D, a.bsa, a.nkv, a.b, a.V.st, a.V.sh, a.V.sb, 128))
      return cudaErrorNotSupported;
  } else {
    maps.ks = maps.kc;  // never read: there are no selected tiles
    maps.vs = maps.vc;
  }
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, attn_tma_kernel, maps, a, nsplit);
}

}  // namespace quoka
