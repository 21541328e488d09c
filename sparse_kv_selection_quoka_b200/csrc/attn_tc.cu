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
// One CTA per 128 query rows of one head. The key list is the selected prior
// rows (read in place through the sorted index list: a fused gather) followed
// by the chunk's keys, in tiles of 128 keys. Warp roles:
//   warps 0-3  softmax: thread r owns query row r (= TMEM lane r); reads its
//              S row from TMEM, applies the causal mask, online softmax in
//              fp32 (exp2 on the MUFU), rescales the O accumulator in TMEM
//              when the running max moves, writes P (bf16) to shared memory;
//              final normalisation and store.
//   warp 4     TMEM allocation and the single-thread MMA issue:
//              S = Q K^T (M=128, N=128, K=128) into a double-buffered TMEM S,
//              O += P V (M=128, N=128, K=128) into the TMEM O accumulator.
//   warps 5-8  loaders: cp.async 16-byte row chunks (gathered by index) into
//              a 2-stage K/V ring laid out in the 128-byte-swizzled UMMA
//              layout; zero-fill past the end of the key list. Warps 5-6
//              load the even tiles (and Q), warps 7-8 the odd tiles.
// Every wait is bounded: a wait that gives up records QUOKA_ERR_TIMEOUT and
// the CTA unwinds (waits for its in-flight copies and MMAs, frees TMEM).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace quoka {

using namespace sm100;

namespace {

constexpr int AT_M = 128;      // query rows per CTA
constexpr int AT_N = 128;      // keys per tile
constexpr int AT_D = 128;      // head dim
constexpr int AT_STAGES = 2;   // K/V ring depth
constexpr int AT_SM_WARPS = 4;
constexpr int AT_MMA_WARP = 4;
constexpr int AT_LD_WARPS = 4;
constexpr int AT_LD_THREADS = AT_LD_WARPS * 32 / AT_STAGES;  // threads of one loader group
constexpr int AT_THREADS = (AT_SM_WARPS + 1 + AT_LD_WARPS) * 32;
constexpr int TILE_BYTES = 128 * AT_D * 2;  // 128 rows x 256 B
constexpr int ATOM_BYTES = 128 * 128;       // one 64-column swizzle atom of a 128-row tile
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256;

constexpr uint32_t IDESC_QK = idesc_bf16_f32(AT_M, AT_N, 0, 0);  // A=Q K-major, B=K K-major
constexpr uint32_t IDESC_PV = idesc_bf16_f32(AT_M, AT_D, 0, 1);  // A=P K-major, B=V MN-major

struct __align__(1024) AttnSmem {
  uint8_t q[TILE_BYTES];
  uint8_t k[AT_STAGES][TILE_BYTES];
  uint8_t v[AT_STAGES][TILE_BYTES];
  uint8_t p[TILE_BYTES];
  uint64_t q_full;
  uint64_t kv_full[AT_STAGES];
  uint64_t kv_empty[AT_STAGES];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t p_full;
  uint64_t o_done;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void record_abort(AttnSmem& sm, int* status) {
  sm.abort = 1;
  latch_status(status, 5 /* QUOKA_ERR_TIMEOUT */);
}

// Warp-uniform bounded wait (every lane polls; all lanes agree on the result).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, AttnSmem& sm, int* status) {
  const bool ok = mbar_wait(bar, parity, &sm.abort);
  const bool all_ok = __all_sync(0xffffffffu, ok);
  if (!all_ok && (threadIdx.x & 31) == 0) record_abort(sm, status);
  return all_ok;
}

__global__ void __launch_bounds__(AT_THREADS, 1)
attn_tc_kernel(const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, bi = blockIdx.z;
  const int G = a.nq / a.nkv, j = h / G;
  const int t0 = blockIdx.x * AT_M;
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int nsel = a.bsa > 0 ? max(0, min(a.kv_count[kvrow], a.bsa)) : 0;
  const int nchunk = min(a.BCP, t0 + AT_M);
  const int total = nsel + nchunk;
  const int nT = (total + AT_N - 1) / AT_N;

  if (tid == 0) {
    mbar_init(&sm.q_full, AT_LD_THREADS);
    for (int s = 0; s < AT_STAGES; ++s) {
      mbar_init(&sm.kv_full[s], AT_LD_THREADS);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_empty[s], AT_SM_WARPS * 32);
    }
    mbar_init(&sm.p_full, AT_SM_WARPS * 32);
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == AT_MMA_WARP) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp >= AT_MMA_WARP + 1) {
    // ------------------------------------------------------------ loaders
    // Two groups of 64 threads own alternating tiles (group g loads tiles
    // i = g, g + 2, ... into stage g). Each group publishes a tile as soon as
    // it has landed, so a group never waits for a free stage while holding
    // back a tile the MMA needs first.
    const int grp = (warp - (AT_MMA_WARP + 1)) / 2;
    const int lt = tid - (AT_MMA_WARP + 1 + 2 * grp) * 32;  // 0..63
    const int c = lt & 15;        // 16-byte chunk of a row (fixed per thread)
    const int rsub = lt >> 4;     // row within a group of 4
    const bf16* Qb = static_cast<const bf16*>(a.Q.data) + bi * a.Q.sb + h * a.Q.sh;
    const bf16* Kb = static_cast<const bf16*>(a.K.data) + bi * a.K.sb + j * a.K.sh;
    const bf16* Vb = static_cast<const bf16*>(a.V.data) + bi * a.V.sb + j * a.V.sh;
    const bf16* Kcb = static_cast<const bf16*>(a.Kc.data) + bi * a.Kc.sb + j * a.Kc.sh;
    const bf16* Vcb = static_cast<const bf16*>(a.Vc.data) + bi * a.Vc.sb + j * a.Vc.sh;
    const int32_t* idx = a.kv_idx + kvrow * a.bsa;
    bool bad_index = false;

    if (grp == 0) {
      const uint32_t q_s = smem_u32(sm.q);
#pragma unroll 4
      for (int it = 0; it < 32; ++it) {
        const int r = it * 4 + rsub;
        const int t = t0 + r;
        const bool ok = t < a.BCP;
        const bf16* src = ok ? Qb + (int64_t)t * a.Q.st + c * 8 : Kcb;
        cp_async_16(q_s + sw128_offset(r, c, 128), src, ok ? 16u : 0u);
      }
      cp_async_commit();
    }

    bool alive = true;
    for (int i = grp; i < nT && alive; i += AT_STAGES) {
      const int s = grp;
      if (i >= AT_STAGES) alive = warp_wait(&sm.kv_empty[s], ((i / AT_STAGES) - 1) & 1, sm, a.status);
      if (!alive) break;
      const uint32_t k_s = smem_u32(sm.k[s]), v_s = smem_u32(sm.v[s]);
#pragma unroll 4
      for (int it = 0; it < 32; ++it) {
        const int r = it * 4 + rsub;
        const int n = i * AT_N + r;
        const bf16* ks = Kcb;
        const bf16* vs = Vcb;
        uint32_t bytes = 0u;
        if (n < nsel) {
          const int32_t tau = __ldg(idx + n);
          if (tau >= 0 && (int64_t)tau < a.T) {
            ks = Kb + (int64_t)tau * a.K.st + c * 8;
            vs = Vb + (int64_t)tau * a.V.st + c * 8;
            bytes = 16u;
          } else {
            bad_index = true;
          }
        } else if (n < total) {
          const int p = n - nsel;
          ks = Kcb + (int64_t)p * a.Kc.st + c * 8;
          vs = Vcb + (int64_t)p * a.Vc.st + c * 8;
          bytes = 16u;
        }
        const uint32_t off = sw128_offset(r, c, 128);
        cp_async_16(k_s + off, ks, bytes);
        cp_async_16(v_s + off, vs, bytes);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      if (i == 0) mbar_arrive(&sm.q_full);
      mbar_arrive(&sm.kv_full[s]);
    }
    cp_async_wait<0>();
    if (bad_index) latch_status(a.status, 6 /* QUOKA_ERR_BOUNDS */);
  } else if (warp == AT_MMA_WARP) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t q_s = smem_u32(sm.q), p_s = smem_u32(sm.p);
      bool alive = mbar_wait(&sm.q_full, 0, &sm.abort);
      auto issue_pv = [&](int jt) -> bool {
        const int s = jt % AT_STAGES;
        if (!mbar_wait(&sm.p_full, jt & 1, &sm.abort)) return false;
        tc_fence_after();
        const uint32_t v_s = smem_u32(sm.v[s]);
#pragma unroll
        for (int kk = 0; kk < AT_N / 16; ++kk) {
          const uint64_t ad = sw128_desc(p_s + (kk >> 2) * ATOM_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(v_s + kk * 2048, ATOM_BYTES, 1024);
          umma_bf16_ss(tmem + TM_O, ad, bd, IDESC_PV, (jt > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&sm.kv_empty[s]);
        umma_commit(&sm.o_done);
        return true;
      };
      for (int i = 0; i < nT && alive; ++i) {
        const int s = i % AT_STAGES, sb = i & 1;
        alive = mbar_wait(&sm.kv_full[s], (i / AT_STAGES) & 1, &sm.abort);
        if (alive && i >= 2) alive = mbar_wait(&sm.s_empty[sb], ((i >> 1) - 1) & 1, &sm.abort);
        if (!alive) break;
        tc_fence_after();
        const uint32_t k_s = smem_u32(sm.k[s]);
#pragma unroll
        for (int kk = 0; kk < AT_D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * ATOM_BYTES + (kk & 3) * 32;
          const uint64_t ad = sw128_desc(q_s + koff, 16, 1024);
          const uint64_t bd = sw128_desc(k_s + koff, 16, 1024);
          umma_bf16_ss(tmem + (sb ? TM_S1 : TM_S0), ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.s_full[sb]);
        if (i >= 1) alive = issue_pv(i - 1);
      }
      if (alive && nT > 0) alive = issue_pv(nT - 1);
      if (!alive) record_abort(sm, a.status);
      // every MMA this thread issued has completed before TMEM is freed
      umma_commit(&sm.mma_done);
      if (!mbar_drain(&sm.mma_done, 0)) latch_status(a.status, 5 /* QUOKA_ERR_TIMEOUT */);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = tid;  // query row within the tile == TMEM lane
    const int t = t0 + r;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float qscale = a.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    uint8_t* prow = sm.p;
    bool alive = true;
    for (int i = 0; i < nT && alive; ++i) {
      const int sb = i & 1;
      alive = warp_wait(&sm.s_full[sb], (i >> 1) & 1, sm, a.status);
      if (!alive) break;
      tc_fence_after();
      float x[AT_N];
#pragma unroll
      for (int q4 = 0; q4 < AT_N / 32; ++q4)
        tmem_ld32(lane_base + (sb ? TM_S1 : TM_S0) + q4 * 32, *reinterpret_cast<float(*)[32]>(&x[q4 * 32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sm.s_empty[sb]);

      // mask (keys past the list, and chunk keys after this row), scale, max
      const int base_n = i * AT_N;
      float mx = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < AT_N; ++cc) {
        const int n = base_n + cc;
        const bool vis = n < nsel || (n < total && n - nsel <= t);
        x[cc] = vis ? x[cc] * qscale : -INFINITY;
        mx = fmaxf(mx, x[cc]);
      }
      const float m_new = fmaxf(m, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float corr = ex2(m - m_use);
      float rs = 0.f;
#pragma unroll
      for (int cc = 0; cc < AT_N; ++cc) {
        x[cc] = ex2(x[cc] - m_use);
        rs += x[cc];
      }
      l = l * corr + rs;
      m = m_new;

      if (i > 0) {
        // PV of the previous tile must be done before O is rescaled and the
        // P buffer is overwritten
        alive = warp_wait(&sm.o_done, (i - 1) & 1, sm, a.status);
        if (!alive) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll 1
          for (int q4 = 0; q4 < AT_D / 32; ++q4) {
            float o[32];
            tmem_ld32(lane_base + TM_O + q4 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] *= corr;
            tmem_st32(lane_base + TM_O + q4 * 32, o);
          }
          tmem_wait_st();
        }
      }
      // P row (bf16) into the swizzled K-major A-operand tile
#pragma unroll
      for (int c = 0; c < AT_N / 8; ++c) {
        uint4 pk;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(x[8 * c + 0], x[8 * c + 1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(x[8 * c + 2], x[8 * c + 3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(x[8 * c + 4], x[8 * c + 5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(x[8 * c + 6], x[8 * c + 7]);
        pk.x = *reinterpret_cast<uint32_t*>(&h0);
        pk.y = *reinterpret_cast<uint32_t*>(&h1);
        pk.z = *reinterpret_cast<uint32_t*>(&h2);
        pk.w = *reinterpret_cast<uint32_t*>(&h3);
        *reinterpret_cast<uint4*>(prow + sw128_offset(r, c, 128)) = pk;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
    }
    if (alive && nT > 0) alive = warp_wait(&sm.o_done, (nT - 1) & 1, sm, a.status);
    if (alive) {
      tc_fence_after();
      const float inv = 1.f / l;
      bf16* orow = static_cast<bf16*>(a.O) + (((int64_t)bi * a.nq + h) * a.BCP + t) * AT_D;
#pragma unroll 1
      for (int q4 = 0; q4 < AT_D / 32; ++q4) {
        float o[32];
        tmem_ld32(lane_base + TM_O + q4 * 32, o);
        tmem_wait_ld();
        if (t < a.BCP) {
#pragma unroll
          for (int u = 0; u < 32; u += 8) {
            uint4 pk;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(o[u + 0] * inv, o[u + 1] * inv);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(o[u + 2] * inv, o[u + 3] * inv);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(o[u + 4] * inv, o[u + 5] * inv);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(o[u + 6] * inv, o[u + 7] * inv);
            pk.x = *reinterpret_cast<uint32_t*>(&h0);
            pk.y = *reinterpret_cast<uint32_t*>(&h1);
            pk.z = *reinterpret_cast<uint32_t*>(&h2);
            pk.w = *reinterpret_cast<uint32_t*>(&h3);
            *reinterpret_cast<uint4*>(orow + q4 * 32 + u) = pk;
          }
        }
      }
      if (t < a.BCP && a.lse != nullptr)
        a.lse[((int64_t)bi * a.nq + h) * a.BCP + t] = (m + __log2f(l)) * 0.6931471805599453f;
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
  const size_t smem = sizeof(AttnSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.BCP + AT_M - 1) / AT_M, a.nq, a.b);
  attn_tc_kernel<<<grid, AT_THREADS, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace quoka
