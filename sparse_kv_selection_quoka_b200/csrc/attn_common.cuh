// Pieces shared by the two tcgen05 attention kernels (the one that streams
// gathered K/V tiles with TMA and the one that gathers rows while loading).
//
// Layout shared by both: TMEM holds S0 | S1 | O0 | O1 (128 fp32 columns
// each, 512 in all), S_w and O_w belonging to softmax warpgroup w, whose
// thread r owns query row r (TMEM lane r) of its query tile. In the
// gathering kernel the two warpgroups own two query tiles of one KV head;
// in the streaming kernel they share one query tile and take alternate key
// tiles.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace quoka {
namespace attn {

using namespace sm100;

constexpr int D = 128;                    // head dim
constexpr int N = 128;                    // keys per tile
constexpr int TILE_BYTES = 128 * D * 2;   // one 128-row bf16 tile
constexpr int ATOM_BYTES = 128 * 128;     // one 64-column swizzle atom of a 128-row tile
constexpr uint32_t TMEM_COLS = 512;
constexpr int SOFTMAX_THREADS = 256;      // warps 0-7
constexpr float RESCALE_THRESHOLD = 8.f;  // log2 units

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, N, 0, 0);  // A = Q K-major, B = K K-major
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);  // A = P (TMEM), B = V MN-major

struct TileInfo {
  int valid, h, t0;
};

// Query tiles of pair `pair` of KV head j: row tile r = 2 * pair + w is query
// head j * G + r / ntt, chunk rows [128 * (r % ntt), +128).
__device__ __forceinline__ void pair_tiles(int pair, int j, int G, int ntt, TileInfo (&ti)[2]) {
  const int R = G * ntt;
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int r = 2 * pair + w;
    ti[w].valid = r < R;
    ti[w].h = j * G + (r < R ? r / ntt : 0);
    ti[w].t0 = (r < R ? r % ntt : 0) * 128;
  }
}

// A wait gave up: stop the CTA's other roles and record the fault and the
// waiting site (a small code naming the barrier).
template <class Smem>
__device__ __forceinline__ void record_abort(Smem& sm, int* status, int where) {
  sm.abort = 1;
  latch_status(status, 5 /* QUOKA_ERR_TIMEOUT */);
  latch_where(status, where);
}

// Warp-uniform bounded wait (every lane polls; all lanes agree on the
// result), bounded by the kernel's wait limit sm.wait_ns.
template <class Smem>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Smem& sm, int* status, int where) {
  const bool ok = mbar_wait(bar, parity, &sm.abort, sm.wait_ns);
  const bool all_ok = __all_sync(0xffffffffu, ok);
  if (!all_ok && (threadIdx.x & 31) == 0) record_abort(sm, status, where);
  return all_ok;
}

// Bounded wait on a local barrier that another CTA of the cluster completes.
__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity) {
  bool ok = mbar_try_wait_cluster(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    while (!ok && globaltimer_ns() - t0 < kWaitLimitNs) ok = mbar_try_wait_cluster(bar, parity);
  }
  return ok;
}

template <class Smem>
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity, Smem& sm, int* status, int where) {
  const bool all_ok = __all_sync(0xffffffffu, wait_cluster(bar, parity));
  if (!all_ok && (threadIdx.x & 31) == 0) record_abort(sm, status, where);
  return all_ok;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// The MMA issue helpers below are called by every lane of the (converged)
// MMA warp; one elected lane issues.

// S[:, 0:128) = Q K^T for a 128-row Q tile and a 128-key K tile, both in
// shared memory in the 128-byte-swizzled K-major layout (two 64-column atoms).
__device__ __forceinline__ void issue_qk(uint32_t tmem_s, uint32_t q_smem, uint32_t k_smem) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t koff = (kk >> 2) * ATOM_BYTES + (kk & 3) * 32;
    umma_bf16_ss_warp(tmem_s, sw128_desc(q_smem + koff, 16, 1024), sw128_desc(k_smem + koff, 16, 1024), IDESC_QK,
                 kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V with P (bf16, packed two per column) in TMEM over the S columns
// and V in shared memory in the 128-byte-swizzled MN-major layout.
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_smem, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < N / 16; ++kk)
    umma_bf16_ts_warp(tmem_o, tmem_p + kk * 8, sw128_desc(v_smem + kk * 2048, ATOM_BYTES, 1024), IDESC_PV,
                 (accumulate || kk > 0) ? 1u : 0u);
}

// Part `part` of O (+)= P V when the 128 keys are released in PARTS
// equal parts: the K = 16 steps of keys [part * N / PARTS, (part + 1) * N / PARTS).
template <int PARTS>
__device__ __forceinline__ void issue_pv_part(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_smem, int part,
                                              bool accumulate) {
  constexpr int KK = N / 16 / PARTS;
#pragma unroll
  for (int q = 0; q < KK; ++q) {
    const int kk = part * KK + q;
    umma_bf16_ts_warp(tmem_o, tmem_p + kk * 8, sw128_desc(v_smem + kk * 2048, ATOM_BYTES, 1024), IDESC_PV,
                 (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One key tile of the online softmax of this thread's query row, single
// pass: the row's 128 scores are read from TMEM once into registers. Key c
// of the tile (key number base_n + c) is visible when base_n + c < lim. Then
// the row max (3-input max tree), and P = 2^(s * qscale - m) in bf16 over
// the first 64 S columns (packed two per column), with the products and row
// sums in paired fp32 arithmetic and the exp2 on the MUFU. The running max m moves only when it
// grows by more than RESCALE_THRESHOLD, in which case the O accumulator
// (complete for the previous tiles) is rescaled in TMEM before any P of the
// tile is released. P is released to the MMA issuer in PARTS equal key
// ranges as soon as each is in TMEM: after the part's stores complete, each
// warp arrives once on p_part[part] (4 arrivals per part), so the P V
// product of the first keys runs while the later ones are still being
// exponentiated. Updates m and l. TMEM accesses are warp-collective: no
// per-row branch surrounds one.
template <int PARTS>
__device__ __forceinline__ void softmax_tile_split(uint32_t S, uint32_t O, bool have_o, int base_n, int lim,
                                                   float qscale, float& m, float& l, uint64_t* p_part) {
  constexpr int CPP = 4 / PARTS;  // 32-key chunks per part
  float v[128];
  __syncwarp();
  tmem_ld64(S, v);
  tmem_ld64(S + 64, v + 64);
  tmem_wait_ld();
  if (base_n + N > lim) {
#pragma unroll
    for (int u = 0; u < 128; ++u) v[u] = (base_n + u < lim) ? v[u] : -INFINITY;
  }
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(v[k], v[k + 8]);
#pragma unroll
  for (int u = 16; u < 128; u += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], v[u + k], v[u + 8 + k]);
  const float mx = fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7])) * qscale;
  const float m_cand = fmaxf(m, mx);
  const float m_new = (m_cand > m + RESCALE_THRESHOLD || m == -INFINITY) ? m_cand : m;
  const float corr = (m_new == m) ? 1.f : ex2(m - m_new);
  const float m_use = m_new == -INFINITY ? 0.f : m_new;
  // warp-uniform condition: the rescale's TMEM traffic is collective
  if (have_o && __any_sync(0xffffffffu, corr != 1.f)) {
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
  const uint64_t qs2 = f2_pack(qscale, qscale), nm2 = f2_pack(-m_use, -m_use);
  uint64_t acc[4] = {0, 0, 0, 0};  // paired row sums (+0.0f halves)
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int u = 0; u < 32; u += 2) {
      const int e = 32 * c + u;
      const uint64_t x = f2_fma(f2_pack(v[e], v[e + 1]), qs2, nm2);
      float x0, x1;
      f2_unpack(x, x0, x1);
      const float p0 = ex2(x0), p1 = ex2(x1);
      acc[(u >> 1) & 3] = f2_add(acc[(u >> 1) & 3], f2_pack(p0, p1));
      pk[u >> 1] = pack_bf16x2(p0, p1);
    }
    __syncwarp();
    tmem_st16(S + 16 * c, pk);
    if (c % CPP == CPP - 1) {
      // this part's P (and any O rescale) is in TMEM: release it
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&p_part[c / CPP]);
    }
  }
  float r[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) f2_unpack(acc[k], r[2 * k], r[2 * k + 1]);
  l = l * corr + (((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7])));
  m = m_new;
}

// One key tile of the online softmax of this thread's query row, on S in
// TMEM (this warp's lanes): key c of the tile (key number base_n + c) is
// visible when base_n + c < lim. Two passes over the row (max, then
// P = 2^(s * qscale - m) in bf16 over the consumed S columns); the running
// max m moves only when it grows by more than RESCALE_THRESHOLD, in which
// case the O accumulator (complete for the previous tiles) is rescaled in
// TMEM. Updates m and l. Every TMEM access is warp-collective: no per-row
// branch surrounds one.
__device__ __forceinline__ void softmax_tile(uint32_t S, uint32_t O, bool have_o, int base_n, int lim, float qscale,
                                             float& m, float& l) {
  const bool all_vis = base_n + N <= lim;
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
  l = l * corr + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
  m = m_new;
  // warp-uniform condition: the rescale's TMEM traffic is collective
  if (have_o && __any_sync(0xffffffffu, corr != 1.f)) {
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
}

}  // namespace attn
}  // namespace quoka
