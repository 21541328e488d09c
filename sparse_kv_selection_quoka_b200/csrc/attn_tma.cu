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
// (one query head, 128 consecutive chunk positions each); a CTA takes one
// such tile. Its key tiles are ceil(nsel/128) tiles of selected rows (rows
// past nsel are masked) followed by the chunk's own keys up to the tile's
// last row, ceil(nchunk/128) tiles. The two softmax warpgroups take the key
// tiles alternately (warpgroup w: tiles w, w + 2, ...), each with its own
// online-softmax state and its own O accumulator in TMEM, so the tensor core
// always has the other warpgroup's products to run while one computes its
// softmax. After the last tile the two partial results of every row are in
// the same SM's TMEM and are combined there.
//
// Split key ranges: when the query tiles alone leave most SMs idle (short
// chunks, few heads), each query tile's key tiles are cut into nsplit
// contiguous ranges and the grid runs one CTA per (tile, range). Such a CTA
// stores its range's output, normalised by the range's own softmax sum, as
// a bf16 tile (the same TMA store, into a partial buffer) with the range's
// log-sum-exp in fp32; a merge kernel then combines the
// ranges of every row: O = sum_s exp(lse_s - LSE) O_s, LSE = log sum_s
// exp(lse_s).
//
// Warp roles (352 threads):
//   warps 0-7   softmax: warpgroup w = warp / 4, one query row per thread
//               (row = TMEM lane); then the combine of the two partials,
//               normalisation, and the bf16 output tile stored with TMA.
//   warp 8      TMEM allocation and the MMA issue (the whole warp in step,
//               one elected lane issuing), per pair of key tiles (2i, 2i+1):
//               QK0(2i), PV1(2i-1), QK1(2i+1), PV0(2i). Each PV starts on
//               the first half of its keys as soon as that half of P is in
//               TMEM.
//   warp 9      TMA loads of Q, then of each key tile's K (3-stage ring, a
//               stage released by its QK^T).
//   warp 10     TMA loads of each key tile's V (3-stage ring, a stage
//               released by its PV).
// TMEM: S0 | S1 | O0 | O1, 128 columns each (512).
// Every wait is bounded (by the launch's wait limit, 2 s unless a test sets
// another): a wait that gives up records QUOKA_ERR_TIMEOUT and a fault-site
// code, and the CTA unwinds (waits for in-flight copies and MMAs, frees
// TMEM, stores no output tile).
#include <stddef.h>

#include <algorithm>

#include "attn_common.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace quoka {

using namespace sm100;
using namespace attn;

namespace {

constexpr int KST = 3;  // K ring depth
constexpr int VST = 3;  // V ring depth
constexpr int THREADS = 352;
constexpr int MMA_WARP = 8;
constexpr int LOAD_WARP = 9;    // Q and K
constexpr int VLOAD_WARP = 10;  // V
// P of a tile is released to the P V product in this many key ranges.
constexpr int PV_PARTS = 2;

struct Maps {
  CUtensorMap q, ks, vs, kc, vc, o;
  CUtensorMap op;  // split key ranges: the partial outputs, (nsplit * b, nq, BCP, d)
};

struct __align__(1024) Smem {
  uint8_t q[TILE_BYTES];       // the Q tile; after the last MMA, the bf16 output tile
  uint8_t k[KST][TILE_BYTES];  // K ring; after the last MMA, the (m, l) exchange
  uint8_t v[VST][TILE_BYTES];  // V ring
  uint64_t q_full;
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[2], p_part[2][PV_PARTS];
  uint64_t o_final, mma_done;
  uint32_t tmem_base;
  int abort;
  uint64_t wait_ns;  // bound of every wait
};

// TMA boxes of one 128-row tile (two 64-column atoms).
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* m, uint64_t* bar, int y, int j, int bi) {
  mbar_arrive_expect_tx(bar, TILE_BYTES);
  tma_load_4d(dst, m, bar, 0, y, j, bi);
  tma_load_4d(dst + ATOM_BYTES, m, bar, 64, y, j, bi);
}

// Waits, bounded, until the last copy into each stage of a ring has landed
// (nload copies were issued in ring order), so that none is in flight when
// the CTA exits, even if a consumer gave up.
template <int STAGES>
__device__ __forceinline__ void drain_ring(Smem& sm, uint64_t* full, int nload, int* status, int where) {
  for (int s = 0; s < STAGES; ++s) {
    const int nf = nload > s ? (nload - s + STAGES - 1) / STAGES : 0;
    if (nf > 0 && !mbar_drain(&full[s], (nf - 1) & 1, sm.wait_ns)) record_abort(sm, status, where);
  }
}

// One thread per ring (K or V): the tiles 0 .. nT - 1 (selected tiles from
// the gathered maps, then chunk tiles), each into the next stage of its ring
// once that stage is released. The stages tile kt needs are released by the
// QK^T (K) and the PV (V) of tile kt - 3; the MMA order (QK0(2i), PV1(2i-1),
// QK1(2i+1), PV0(2i)) issues the PV of a tile right after the QK^T of the
// next one, so both come before the QK^T of tile kt - 1: the loads never
// wait on a product that waits on a later load. With a thread per ring, a K
// load never queues behind a V stage that is released later.
template <bool IS_V>
__device__ __forceinline__ void load_kv(Smem& sm, const Maps& maps, int nT, int kt_base, int ntile_sel, int j,
                                        int bi, int* status) {
  constexpr int ST = IS_V ? VST : KST;
  uint64_t* const full = IS_V ? sm.v_full : sm.k_full;
  uint64_t* const empty = IS_V ? sm.v_empty : sm.k_empty;
  int nl = 0;
  for (int kt = 0; kt < nT; ++kt) {
    const bool sel_tile = kt_base + kt < ntile_sel;
    const int s = kt % ST;
    if (kt >= ST && !mbar_wait(&empty[s], ((kt / ST) - 1) & 1, &sm.abort, sm.wait_ns)) {
      record_abort(sm, status, IS_V ? 14 : 11);
      break;
    }
    const CUtensorMap* m = IS_V ? (sel_tile ? &maps.vs : &maps.vc) : (sel_tile ? &maps.ks : &maps.kc);
    load_tile(smem_u32(IS_V ? sm.v[s] : sm.k[s]), m, &full[s],
              (sel_tile ? kt_base + kt : kt_base + kt - ntile_sel) * N, j, bi);
    nl = kt + 1;
  }
  drain_ring<ST>(sm, full, nl, status, IS_V ? 15 : 12);
  if (!IS_V && !mbar_drain(&sm.q_full, 0, sm.wait_ns)) record_abort(sm, status, 13);
}

__global__ void __launch_bounds__(THREADS, 1)
attn_tma_kernel(const __grid_constant__ Maps maps, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(align_smem_1024(smem_raw));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.y, bi = blockIdx.z;
  const int G = a.nq / a.nkv;
  const int ntt = (a.BCP + 127) / 128;  // row tiles per query head
  const int qt = (int)blockIdx.x % (G * ntt), split = (int)blockIdx.x / (G * ntt);
  const int h = j * G + qt / ntt;
  const int t0 = (qt % ntt) * 128;

  // Setup and the Q load touch nothing the previous kernel writes: they run
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
      // one arrival per warp (the test hook makes the first part of
      // warpgroup 0 wait for an arrival that never comes)
      for (int c = 0; c < PV_PARTS; ++c) mbar_init(&sm.p_part[w][c], (a.inject && w == 0 && c == 0) ? 5 : 4);
    }
    mbar_init(&sm.o_final, 1);
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    sm.wait_ns = a.wait_ns;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp == LOAD_WARP && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.ks);
    tma_prefetch_desc(&maps.vs);
    tma_prefetch_desc(&maps.kc);
    tma_prefetch_desc(&maps.vc);
    tma_prefetch_desc(&maps.o);
    mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES);
    tma_load_4d(smem_u32(sm.q), &maps.q, &sm.q_full, 0, t0, h, bi);
    tma_load_4d(smem_u32(sm.q) + ATOM_BYTES, &maps.q, &sm.q_full, 64, t0, h, bi);
  }

  pdl_wait();  // the gathered rows and their counts come from the previous kernel
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int nsel = a.bsa > 0 ? max(0, min(__ldcg(a.kv_count + kvrow), a.bsa)) : 0;
  const int nchunk = a.no_chunk ? 0 : min(a.BCP, t0 + 128);
  const int ntile_sel = (nsel + N - 1) / N;
  const int nT_all = ntile_sel + (nchunk + N - 1) / N;  // key tiles (0 only without the chunk's keys)
  // this CTA's key tiles: range `split` of nsplit (all of them when 1)
  const int kt_base = (int)((int64_t)nT_all * split / a.nsplit);
  const int nT = (int)((int64_t)nT_all * (split + 1) / a.nsplit) - kt_base;
  const int npair = (nT + 1) / 2;

  if (warp == LOAD_WARP) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) load_kv<false>(sm, maps, nT, kt_base, ntile_sel, j, bi, a.status);
    __syncwarp();
  } else if (warp == VLOAD_WARP) {
    if (lane == 0) load_kv<true>(sm, maps, nT, kt_base, ntile_sel, j, bi, a.status);
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issue
    // The whole warp runs this loop in step (waits on every lane, warp-uniform
    // results); one elected lane issues each MMA and commit.
    const uint32_t q0 = smem_u32(sm.q);
    int where = 21;
    // S_w = Q K(kt)^T, the K stage released once the product is done
    auto qk = [&](int w, int kt) -> bool {
      const int ks = kt % KST;
      if (!mbar_wait_warp(&sm.k_full[ks], (kt / KST) & 1, &sm.abort, sm.wait_ns)) return false;
      tc_fence_after();
      issue_qk(tmem + 128u * w, q0, smem_u32(sm.k[ks]));
      umma_commit_warp(&sm.s_full[w]);
      umma_commit_warp(&sm.k_empty[ks]);
      return true;
    };
    // O_w (+)= P_w V(kt), the i-th tile of warpgroup w: each part of P is
    // issued as soon as the softmax releases it; the V stage is released
    // once the product is done
    auto pv = [&](int w, int kt, int i) -> bool {
      const int vs = kt % VST;
      if (!mbar_wait_warp(&sm.v_full[vs], (kt / VST) & 1, &sm.abort, sm.wait_ns)) return false;
      for (int c = 0; c < PV_PARTS; ++c) {
        if (!mbar_wait_warp(&sm.p_part[w][c], i & 1, &sm.abort, sm.wait_ns)) return false;
        tc_fence_after();
        issue_pv_part<PV_PARTS>(tmem + 256u + 128u * w, tmem + 128u * w, smem_u32(sm.v[vs]), c, i > 0);
      }
      umma_commit_warp(&sm.v_empty[vs]);
      return true;
    };
    bool alive = mbar_wait_warp(&sm.q_full, 0, &sm.abort, sm.wait_ns);
    for (int i = 0; i < npair && alive; ++i) {
      const int kt0 = 2 * i, kt1 = 2 * i + 1;
      where = 22;
      alive = qk(0, kt0);
      if (!alive) break;
      if (i > 0) {
        where = 23;
        alive = pv(1, kt1 - 2, i - 1);
        if (!alive) break;
      }
      if (kt1 < nT) {
        where = 24;
        alive = qk(1, kt1);
        if (!alive) break;
      }
      where = 25;
      alive = pv(0, kt0, i);
    }
    // the last odd tile's product
    if (alive && nT > 0 && (nT & 1) == 0) {
      where = 26;
      alive = pv(1, nT - 1, npair - 1);
    }
    if (!alive && lane == 0) record_abort(sm, a.status, where);
    umma_commit_warp(&sm.o_final);
    umma_commit_warp(&sm.mma_done);
    const bool drained = __all_sync(0xffffffffu, mbar_drain(&sm.mma_done, 0, sm.wait_ns));
    if (!drained && lane == 0) record_abort(sm, a.status, 27);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int w = warp >> 2;  // key tiles w, w + 2, ... of this warpgroup
    const int r = tid & 127;  // row == TMEM lane
    const int t = t0 + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t S = tmem + lane_off + 128u * w;
    const float qscale = a.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    bool alive = true;
    const int nmine = (nT - w + 1) / 2;  // key tiles of this warpgroup (warpgroup-uniform)
    // the range's selected tiles come first (none when it starts past them);
    // selected key numbers relative to the range's first key
    const int sel_rel = ntile_sel - kt_base;
    const int nsel_rel = nsel - kt_base * N;
    for (int i = 0; i < nmine && alive; ++i) {
      alive = warp_wait(&sm.s_full[w], i & 1, sm, a.status, 31 + w);
      if (!alive) break;
      tc_fence_after();
      const int kt = 2 * i + w;  // (within this CTA's key range)
      const bool sel_tile = kt < sel_rel;
      // key c of the tile is key number base_n + c of its list (selected
      // keys counted from the range's first one); it is visible to row t
      // when it is a selected key below nsel, or a chunk key at a position
      // p < nchunk with p <= t
      const int base_n = (sel_tile ? kt : kt - sel_rel) * N;
      const int lim = sel_tile ? nsel_rel : min(nchunk, t + 1);
      softmax_tile_split<PV_PARTS>(S, tmem + lane_off + 256u + 128u * w, i > 0, base_n, lim,
                                                     qscale, m, l, sm.p_part[w]);
    }

    // ------------------------------------------------ combine and store
    // (both warpgroups reach the named barriers below, whatever happened
    // in the loop)
    if (alive) alive = warp_wait(&sm.o_final, 0, sm, a.status, 33);
    tc_fence_after();
    // (m, l) of both partials of every row (the K ring is free: every MMA
    // is done)
    float* ml = reinterpret_cast<float*>(sm.k[0]);  // [2][128][2]
    ml[(w * 128 + r) * 2] = nmine > 0 ? m : -INFINITY;
    ml[(w * 128 + r) * 2 + 1] = nmine > 0 ? l : 0.f;
    named_barrier_sync(1, 256);
    const float m0 = ml[r * 2], l0 = ml[r * 2 + 1];
    const float m1 = ml[(128 + r) * 2], l1 = ml[(128 + r) * 2 + 1];
    const bool have0 = nT > 0, have1 = nT > 1;  // uniform: warpgroup w accumulated into O_w
    const float M = fmaxf(m0, m1);
    const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - M);
    const float f1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
    const float L = f0 * l0 + f1 * l1;
    const float inv = L > 0.f ? 1.f / L : 0.f;  // no visible key: O = 0, lse = -inf
    // warpgroup w combines, normalises and stages output columns
    // [64w, 64w + 64) of its rows, bf16, in the 128-byte-swizzled layout the
    // TMA store reads (the Q area: every MMA is done); a key range of a split
    // tile stores them to its partial output instead
    const uint32_t O0 = tmem + lane_off + 256u + 64u * w;
    const uint32_t O1 = tmem + lane_off + 384u + 64u * w;
    const bool part = a.nsplit > 1;
#pragma unroll 1
    for (int c2 = 0; c2 < 2; ++c2) {
      float o[32], p[32];
      if (have0) tmem_ld32(O0 + 32 * c2, o);
      if (have1) tmem_ld32(O1 + 32 * c2, p);
      tmem_wait_ld();
      if (!have0) {
#pragma unroll
        for (int u = 0; u < 32; ++u) o[u] = 0.f;
      }
      if (!have1) {
#pragma unroll
        for (int u = 0; u < 32; ++u) p[u] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < 32; u += 8) {
        uint4 pk;
        pk.x = pack_bf16x2((o[u] * f0 + p[u] * f1) * inv, (o[u + 1] * f0 + p[u + 1] * f1) * inv);
        pk.y = pack_bf16x2((o[u + 2] * f0 + p[u + 2] * f1) * inv, (o[u + 3] * f0 + p[u + 3] * f1) * inv);
        pk.z = pack_bf16x2((o[u + 4] * f0 + p[u + 4] * f1) * inv, (o[u + 5] * f0 + p[u + 5] * f1) * inv);
        pk.w = pack_bf16x2((o[u + 6] * f0 + p[u + 6] * f1) * inv, (o[u + 7] * f0 + p[u + 7] * f1) * inv);
        *reinterpret_cast<uint4*>(sm.q + sw128_offset(r, (64 * w + 32 * c2 + u) >> 3, 128)) = pk;
      }
    }
    if (w == 0 && t < a.BCP) {
      const int64_t orow = ((int64_t)bi * a.nq + h) * a.BCP + t;
      if (part)
        a.lse_parts[(int64_t)split * a.b * a.nq * a.BCP + orow] =
            L > 0.f ? (M + __log2f(L)) * 0.6931471805599453f : -INFINITY;
      else if (a.lse != nullptr)
        a.lse[orow] = (M + __log2f(L)) * 0.6931471805599453f;
    }
    // rows past the chunk are clipped by the store
    fence_proxy_async_smem();
    named_barrier_sync(1, 256);
    // (after a timeout the tile is not stored: the status word reports it)
    if (tid == 0 && !*reinterpret_cast<volatile int*>(&sm.abort)) {
      const CUtensorMap* om = part ? &maps.op : &maps.o;
      const int zb = part ? split * a.b + bi : bi;
      tma_store_4d(om, smem_u32(sm.q), 0, t0, h, zb);
      tma_store_4d(om, smem_u32(sm.q) + ATOM_BYTES, 64, t0, h, zb);
      bulk_commit_group();
      bulk_wait_group_read_0();  // the staging may go once the copy has read it
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// The merge of the key ranges of split tiles: one thread per 8 output
// elements of a row. Ranges that saw no visible key (lse = -inf) weigh 0; a
// row with none gives O = 0, lse = -inf.
constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
attn_split_merge_kernel(const bf16* __restrict__ O_parts, const float* __restrict__ lse_parts, int nsplit,
                        int64_t rows, bf16* __restrict__ O, float* __restrict__ lse) {
  pdl_wait();  // the partials come from the attention kernel
  const int64_t g = (int64_t)blockIdx.x * kMergeThreads + threadIdx.x;
  if (g >= rows * (D / 8)) return;
  const int64_t row = g / (D / 8);
  const int c0 = (int)(g % (D / 8)) * 8;
  float ls[4];
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    ls[s] = s < nsplit ? __ldcg(lse_parts + (int64_t)s * rows + row) : -INFINITY;
    M = fmaxf(M, ls[s]);
  }
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float L = 0.f;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    if (ls[s] == -INFINITY) continue;
    const float wgt = __expf(ls[s] - M);
    L += wgt;
    const uint4 raw = __ldcg(reinterpret_cast<const uint4*>(O_parts + ((int64_t)s * rows + row) * D + c0));
    const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc[2 * u] = fmaf(wgt, __uint_as_float(wd[u] << 16), acc[2 * u]);
      acc[2 * u + 1] = fmaf(wgt, __uint_as_float(wd[u] & 0xFFFF0000u), acc[2 * u + 1]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint4 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(O + row * D + c0) = pk;
  if (c0 == 0 && lse != nullptr) lse[row] = L > 0.f ? M + __logf(L) : -INFINITY;
}

}  // namespace

int attn_splits(int64_t tiles, int nt) {
  if (tiles < 1 || 2 * tiles > kAttnWaveCTAs) return 1;
  int s = (int)std::min<int64_t>(4, kAttnWaveCTAs / tiles);
  s = std::min(s, nt / 2);
  return s < 2 ? 1 : s;
}

cudaError_t launch_attn_tc(const AttnArgs& args, bool pdl, cudaStream_t stream) {
  if (args.d != D) return cudaErrorNotSupported;
  // rows gathered by index while loading: the other kernel
  if (args.kv_idx != nullptr && args.bsa > 0) return launch_attn_tc_gather(args, stream);
  AttnArgs a = args;
  if (a.nsplit < 1 || a.nsplit > 4 || (a.nsplit > 1 && (a.O_parts == nullptr || a.lse_parts == nullptr)))
    return cudaErrorInvalidValue;
  const WaitHooks hooks = wait_hooks();
  a.wait_ns = hooks.wait_ns;
  a.inject = hooks.inject == INJECT_ATTN_TMA ? 1 : 0;
  Maps maps;
  const int64_t oh = (int64_t)a.BCP * D, ob = (int64_t)a.nq * oh;  // O is contiguous
  if (!encode_bf16_4d(&maps.q, a.Q.data, D, a.BCP, a.nq, a.b, a.Q.st, a.Q.sh, a.Q.sb, 128) ||
      !encode_bf16_4d(&maps.kc, a.Kc.data, D, a.BCP, a.nkv, a.b, a.Kc.st, a.Kc.sh, a.Kc.sb, 128) ||
      !encode_bf16_4d(&maps.vc, a.Vc.data, D, a.BCP, a.nkv, a.b, a.Vc.st, a.Vc.sh, a.Vc.sb, 128) ||
      !encode_bf16_4d(&maps.o, a.O, D, a.BCP, a.nq, a.b, D, oh, ob, 128))
    return cudaErrorNotSupported;
  if (a.nsplit > 1) {
    if (!encode_bf16_4d(&maps.op, a.O_parts, D, a.BCP, a.nq, (uint64_t)a.nsplit * a.b, D, oh, ob, 128))
      return cudaErrorNotSupported;
  } else {
    maps.op = maps.o;  // never written
  }
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G * ((a.BCP + 127) / 128) * a.nsplit, a.nkv, a.b);  // one query tile (range) per CTA
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, attn_tma_kernel, maps, a);
  if (e != cudaSuccess || a.nsplit == 1) return e;
  const int64_t rows = (int64_t)a.b * a.nq * a.BCP;
  cudaLaunchConfig_t mc = {};
  mc.gridDim = dim3((unsigned)((rows * (D / 8) + kMergeThreads - 1) / kMergeThreads));
  mc.blockDim = dim3(kMergeThreads);
  mc.stream = stream;
  mc.attrs = attr;
  mc.numAttrs = 1;  // waits for the attention inside
  return cudaLaunchKernelEx(&mc, attn_split_merge_kernel, static_cast<const bf16*>(a.O_parts),
                            static_cast<const float*>(a.lse_parts), a.nsplit, rows, static_cast<bf16*>(a.O),
                            a.lse);
}

}  // namespace quoka
