// Sparse GQA attention for short chunks: a decode step (BCP = 1) or a short
// block of speculative tokens, where the G * BCP query rows of a KV head are
// far fewer than a 128-row tensor-core tile.
//
// [QUOKA §4.2, problem 3] the same attention as the prefill path:
//   O[b,h,t] = sum_k softmax_k(scale * q . k) v,
//   k over {K[b, j, kv_idx[b, j, n]] : n < kv_count[b, j]} U {Kc[b, j, s] : s <= t},
//   j = floor(h / G),
// (QUOKA = the technical write-up "QUOKA: how it reshapes LLM prefill
// efficiency", bqwf.cn news item 915859; its decode-time use is the
// generation-speed experiment of §4.)
//
// With so few query rows the step is bound by reading the selected K / V
// rows, each of which is needed by one KV head only. The keys of a KV head
// (its nsel selected rows, then its BCP chunk keys) are cut into slices of
// 64; one CTA takes one slice for all G * BCP query rows of the head, reads
// its rows by index straight from the cache (no gathered copy: every row is
// read once), and writes the slice's softmax-normalised partial output and
// its log-sum-exp in fp32. A second kernel merges the slices of every query
// row: O = sum_s exp(lse_s - LSE) O_s, LSE = log sum_s exp(lse_s).
// Arithmetic in fp32 on the CUDA cores (bf16 or fp32 inputs).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace quoka {

namespace {

constexpr int kThreads = 128;
constexpr int KS = 64;  // keys per slice (one CTA)
constexpr int kMergeThreads = 256;

template <typename T>
__device__ __forceinline__ void to_f32x(const uint4& v, float* out);
template <>
__device__ __forceinline__ void to_f32x<float>(const uint4& v, float* out) {
  out[0] = __uint_as_float(v.x);
  out[1] = __uint_as_float(v.y);
  out[2] = __uint_as_float(v.z);
  out[3] = __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void to_f32x<__nv_bfloat16>(const uint4& v, float* out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(w[i] << 16);
    out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Shared memory of a slice, in this order: Q rows [R][D] fp32 (pre-scaled),
// K rows [KS] of D elements of the input type with a 16-byte pad each (which
// makes the per-key 16-byte reads of the score loop conflict-free; the same
// space later holds the warps' P V sums), V rows
// [KS][D] of the input type, scores / probabilities [R][KS] fp32, (m, l) per
// row [R][2] fp32.
template <typename T, int D>
struct SliceSmem {
  static constexpr int KROW = D * (int)sizeof(T) + 16;  // bytes per K row
  static constexpr int VROW = D * (int)sizeof(T);       // bytes per V row
  __host__ __device__ static constexpr size_t q_off() { return 0; }
  __host__ __device__ static constexpr size_t k_off(int R) { return (size_t)R * D * 4; }
  // (the K rows' space later holds the 4 warps' P V sums, [4][R][D] fp32)
  __host__ __device__ static constexpr size_t k_bytes(int R) {
    return (size_t)KS * KROW > (size_t)16 * R * D ? (size_t)KS * KROW : (size_t)16 * R * D;
  }
  __host__ __device__ static constexpr size_t v_off(int R) { return k_off(R) + k_bytes(R); }
  __host__ __device__ static constexpr size_t p_off(int R) { return v_off(R) + (size_t)KS * VROW; }
  __host__ __device__ static constexpr size_t ml_off(int R) { return p_off(R) + (size_t)R * KS * 4; }
  __host__ __device__ static constexpr size_t bytes(int R) { return ml_off(R) + (size_t)R * 2 * 4; }
};

// grid (nsplit, nkv, b). Slice s covers key numbers [64 s, 64 s + 64) of the
// head's list (selected keys 0 .. nsel - 1, then chunk keys).
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) decode_slice_kernel(const DecodeArgs a) {
  using L = SliceSmem<T, D>;
  constexpr int EPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  constexpr int CPR = D / EPC;              // chunks per row
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ const T* kp[KS];
  __shared__ const T* vp[KS];
  __shared__ int nsel_s;
  const int G = a.nq / a.nkv, R = G * a.BCP;
  float* Qs = reinterpret_cast<float*>(dsm + L::q_off());
  uint8_t* Ksb = dsm + L::k_off(R);
  const T* Vs = reinterpret_cast<const T*>(dsm + L::v_off(R));
  float* Ps = reinterpret_cast<float*>(dsm + L::p_off(R));
  float* ml = reinterpret_cast<float*>(dsm + L::ml_off(R));
  const int s = blockIdx.x, j = blockIdx.y, bi = blockIdx.z, tid = threadIdx.x;
  const float qscale = a.scale * 1.4426950408889634f;  // scores in log2 units
  const T* Q = static_cast<const T*>(a.Q.data);

  pdl_trigger();
  // the query rows (not written by any earlier kernel of the step): row r is
  // head j * G + r / BCP, chunk position r % BCP
  for (int e = tid; e < R * CPR; e += kThreads) {
    const int r = e / CPR, c = e % CPR;
    const int h = j * G + r / a.BCP, t = r % a.BCP;
    const uint4 v = *reinterpret_cast<const uint4*>(Q + bi * a.Q.sb + h * a.Q.sh + t * a.Q.st + c * EPC);
    float f[EPC];
    to_f32x<T>(v, f);
#pragma unroll
    for (int i = 0; i < EPC; ++i) Qs[r * D + c * EPC + i] = f[i] * qscale;
  }

  pdl_wait();  // the indices and counts may come from the previous kernel
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int n0 = s * KS;
  if (tid < KS) {
    // the count and this slice's index entries at once (an index is read
    // whenever it lies in the list's storage; it counts only below nsel)
    const int n = n0 + tid;
    const int cnt = a.bsa > 0 ? __ldcg(a.kv_count + kvrow) : 0;
    const int32_t tau = n < a.bsa ? __ldcg(a.kv_idx + kvrow * a.bsa + n) : -1;
    const int nsel = max(0, min(cnt, a.bsa));
    const T* kr = nullptr;
    const T* vr = nullptr;
    if (n < nsel) {
      if (tau >= 0 && (int64_t)tau < a.T) {
        kr = static_cast<const T*>(a.K.data) + bi * a.K.sb + j * a.K.sh + tau * a.K.st;
        vr = static_cast<const T*>(a.V.data) + bi * a.V.sb + j * a.V.sh + tau * a.V.st;
      } else if (a.status != nullptr) {
        latch_status(a.status, 6 /* QUOKA_ERR_BOUNDS */);  // the key reads as zeros
      }
    } else if (n - nsel < a.BCP) {
      const int c = n - nsel;
      kr = static_cast<const T*>(a.Kc.data) + bi * a.Kc.sb + j * a.Kc.sh + c * a.Kc.st;
      vr = static_cast<const T*>(a.Vc.data) + bi * a.Vc.sb + j * a.Vc.sh + c * a.Vc.st;
    }
    kp[tid] = kr;
    vp[tid] = vr;
    if (tid == 0) nsel_s = nsel;
  }
  __syncthreads();
  const int nsel = nsel_s;
  const int nk = max(0, min(KS, nsel + a.BCP - n0));  // keys of this slice

  // K and V rows of the slice, copied asynchronously in their input type;
  // rows without a key are zero-filled (the source is then not read: a
  // chunk row of this head stands in as its address)
  {
    const T* dummy = static_cast<const T*>(a.Kc.data) + bi * a.Kc.sb + j * a.Kc.sh;
    const uint32_t kbase = sm100::smem_u32(Ksb), vbase = sm100::smem_u32(Vs);
    for (int e = tid; e < KS * CPR; e += kThreads) {
      const int k = e / CPR, c = e % CPR;
      const T* kr = kp[k];
      const T* vr = vp[k];
      sm100::cp_async_16(kbase + k * L::KROW + c * 16, kr ? kr + c * EPC : dummy, kr ? 16u : 0u);
      sm100::cp_async_16(vbase + k * L::VROW + c * 16, vr ? vr + c * EPC : dummy, vr ? 16u : 0u);
    }
    sm100::cp_async_commit();
    sm100::cp_async_wait<0>();
  }
  __syncthreads();

  // scores: two threads per key (lanes 2k, 2k + 1 of the key's pair), each
  // over half of d, 4 query rows at a time in independent accumulators, the
  // halves summed by one shuffle; key n0 + k is visible to row r when it is
  // a selected key, or a chunk key at a position not after the row's
  {
    static_assert(KS * 2 == kThreads, "two threads per key");
    constexpr int HALF = CPR / 2;  // 16-byte chunks per half row
    const int k = tid >> 1, half = tid & 1;
    const int n = n0 + k;
    const uint4* krow = reinterpret_cast<const uint4*>(Ksb + k * L::KROW) + half * HALF;
    for (int r0 = 0; r0 < R; r0 += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
      for (int c = 0; c < HALF; ++c) {
        float kf[EPC];
        to_f32x<T>(krow[c], kf);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = min(r0 + i, R - 1);  // (rows past R: computed, not stored)
          const float4* qr = reinterpret_cast<const float4*>(Qs + r * D + (half * HALF + c) * EPC);
#pragma unroll
          for (int e4 = 0; e4 < EPC / 4; ++e4) {
            const float4 qq = qr[e4];
            acc[i] = fmaf(qq.x, kf[4 * e4], acc[i]);
            acc[i] = fmaf(qq.y, kf[4 * e4 + 1], acc[i]);
            acc[i] = fmaf(qq.z, kf[4 * e4 + 2], acc[i]);
            acc[i] = fmaf(qq.w, kf[4 * e4 + 3], acc[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 1);
      if (half == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = r0 + i;
          if (r < R) {
            const bool vis = k < nk && (n < nsel || n - nsel <= r % a.BCP);
            Ps[r * KS + k] = vis ? acc[i] : -INFINITY;
          }
        }
      }
    }
  }
  __syncthreads();

  // per row: max, probabilities 2^(s - m), their sum (one warp per row)
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < R; r += kThreads / 32) {
      float* pr = Ps + r * KS;
      const float s0 = pr[lane], s1 = pr[lane + 32];
      float m = fmaxf(s0, s1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float p0 = m == -INFINITY ? 0.f : exp2f(s0 - m);
      const float p1 = m == -INFINITY ? 0.f : exp2f(s1 - m);
      pr[lane] = p0;
      pr[lane + 32] = p1;
      float l = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) {
        ml[2 * r] = m;
        ml[2 * r + 1] = l;
      }
    }
  }
  __syncthreads();

  // P V: warp w takes keys [16 w, 16 w + 16); a lane accumulates a block of
  // 4 rows x 4 columns (one 4-element V read and 4 probabilities per 16
  // FMAs); the warps' sums are added in shared memory (over the K rows, free
  // now). p = 0 past the slice's keys, whose V rows are zero.
  float* Osum = reinterpret_cast<float*>(Ksb);  // [4 warps][R][D]
  {
    const int warp = tid >> 5, lane = tid & 31;
    constexpr int NCG = D / 4;  // 4-column groups
    const int nblk = ((R + 3) / 4) * NCG;
    float acc[4][4];
    for (int blk = lane; blk < nblk; blk += 32) {
      const int rg = blk / NCG, cg = blk % NCG;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < KS / 4; ++kk) {
        const int k = warp * (KS / 4) + kk;
        float v[4];
        if constexpr (sizeof(T) == 2) {
          const uint2 raw = *reinterpret_cast<const uint2*>(Vs + k * D + 4 * cg);
          v[0] = __uint_as_float(raw.x << 16);
          v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
          v[2] = __uint_as_float(raw.y << 16);
          v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
        } else {
          const float4 raw = *reinterpret_cast<const float4*>(Vs + k * D + 4 * cg);
          v[0] = raw.x;
          v[1] = raw.y;
          v[2] = raw.z;
          v[3] = raw.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 4 * rg + i;
          const float p = r < R ? Ps[r * KS + k] : 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[i][c] = fmaf(p, v[c], acc[i][c]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * rg + i;
        if (r < R)
          *reinterpret_cast<float4*>(Osum + ((size_t)warp * R + r) * D + 4 * cg) =
              make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      }
    }
  }
  __syncthreads();

  // the slice's output rows, normalised by their own sums, and their lse
  const int64_t rows = (int64_t)a.b * a.nq * a.BCP;
  for (int e = tid; e < R * D / 4; e += kThreads) {
    const int r = e / (D / 4), c4 = e % (D / 4);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
      const float4 x = *reinterpret_cast<const float4*>(Osum + ((size_t)w * R + r) * D + 4 * c4);
      o.x += x.x;
      o.y += x.y;
      o.z += x.z;
      o.w += x.w;
    }
    const float m = ml[2 * r], l = ml[2 * r + 1];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int h = j * G + r / a.BCP, t = r % a.BCP;
    const int64_t row = ((int64_t)bi * a.nq + h) * a.BCP + t;
    *reinterpret_cast<float4*>(a.O_parts + ((int64_t)s * rows + row) * D + 4 * c4) =
        make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    if (c4 == 0) a.lse_parts[(int64_t)s * rows + row] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// bf16 inputs: the same slice on the tensor cores (mma.sync m16n8k16, bf16 x
// bf16 -> fp32). With only R = G * BCP <= 64 query rows the slice is bound
// by its loads, not by arithmetic; what the tensor cores remove is the
// instruction stream of the CUDA-core dot products (thousands of shared
// memory reads and FMAs per thread), which kept the SMs issuing long after
// the slice's rows had arrived. The query rows are padded to Rp, a multiple
// of 16 (padding rows are zero and their results unused).
//   S (Rp x 64) = Q K^T: warp w takes keys [16 w, 16 w + 16);
//   softmax per row in fp32 (one warp per row), P rounded to bf16;
//   O (Rp x D) = P V: warp w takes columns [w D / 4, (w + 1) D / 4).
// Q, K and V rows sit in shared memory with a 16-byte pad each, P rows with
// one too, so that every 8-row ldmatrix phase hits 32 distinct banks.

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// c (16 x 8, fp32) += a (16 x 16, bf16, row-major) * b (16 x 8, bf16, column-major)
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared memory of a tensor-core slice, in this order: Q rows [Rp], K rows
// [KS], V rows [KS] (bf16, ROWB bytes each), scores [R][KS] fp32, P rows [Rp]
// (bf16, PROWB bytes each), (m, l) per row [R][2] fp32.
template <int D>
struct MmaSliceSmem {
  static constexpr int ROWB = D * 2 + 16;
  static constexpr int PROWB = KS * 2 + 16;
  __host__ __device__ static constexpr size_t k_off(int Rp) { return (size_t)Rp * ROWB; }
  __host__ __device__ static constexpr size_t v_off(int Rp) { return k_off(Rp) + (size_t)KS * ROWB; }
  __host__ __device__ static constexpr size_t s_off(int Rp) { return v_off(Rp) + (size_t)KS * ROWB; }
  __host__ __device__ static constexpr size_t p_off(int Rp) { return s_off(Rp) + (size_t)Rp * KS * 4; }
  __host__ __device__ static constexpr size_t ml_off(int Rp) { return p_off(Rp) + (size_t)Rp * PROWB; }
  __host__ __device__ static constexpr size_t bytes(int Rp) { return ml_off(Rp) + (size_t)Rp * 2 * 4; }
};

template <int D>
__global__ void __launch_bounds__(kThreads) decode_slice_mma_kernel(const DecodeArgs a) {
  using L = MmaSliceSmem<D>;
  using T = __nv_bfloat16;
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  static_assert(KS == 64 && kThreads == 128, "four warps of 16 keys");
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ const T* kp[KS];
  __shared__ const T* vp[KS];
  __shared__ int nsel_s;
  const int G = a.nq / a.nkv, R = G * a.BCP, Rp = (R + 15) & ~15;
  const uint32_t qbase = sm100::smem_u32(dsm), kbase = qbase + (uint32_t)L::k_off(Rp);
  const uint32_t vbase = qbase + (uint32_t)L::v_off(Rp), pbase = qbase + (uint32_t)L::p_off(Rp);
  float* Ss = reinterpret_cast<float*>(dsm + L::s_off(Rp));
  float* ml = reinterpret_cast<float*>(dsm + L::ml_off(Rp));
  const int s = blockIdx.x, j = blockIdx.y, bi = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, grp = lane >> 2, tig = lane & 3;
  const float qscale = a.scale * 1.4426950408889634f;  // scores in log2 units
  const T* Q = static_cast<const T*>(a.Q.data);

  pdl_trigger();
  // the query rows (not written by any earlier kernel of the step): row r is
  // head j * G + r / BCP, chunk position r % BCP; padding rows are zeroed
  for (int e = tid; e < Rp * CPR; e += kThreads) {
    const int r = e / CPR, c = e % CPR;
    const T* src = Q;
    uint32_t n = 0u;
    if (r < R) {
      src = Q + bi * a.Q.sb + (j * G + r / a.BCP) * a.Q.sh + (r % a.BCP) * a.Q.st + c * 8;
      n = 16u;
    }
    sm100::cp_async_16(qbase + r * L::ROWB + c * 16, src, n);
  }
  sm100::cp_async_commit();

  pdl_wait();  // the indices and counts may come from the previous kernel
  const int64_t kvrow = (int64_t)bi * a.nkv + j;
  const int n0 = s * KS;
  if (tid < KS) {
    const int n = n0 + tid;
    const int cnt = a.bsa > 0 ? __ldcg(a.kv_count + kvrow) : 0;
    const int32_t tau = n < a.bsa ? __ldcg(a.kv_idx + kvrow * a.bsa + n) : -1;
    const int nsel = max(0, min(cnt, a.bsa));
    const T* kr = nullptr;
    const T* vr = nullptr;
    if (n < nsel) {
      if (tau >= 0 && (int64_t)tau < a.T) {
        kr = static_cast<const T*>(a.K.data) + bi * a.K.sb + j * a.K.sh + tau * a.K.st;
        vr = static_cast<const T*>(a.V.data) + bi * a.V.sb + j * a.V.sh + tau * a.V.st;
      } else if (a.status != nullptr) {
        latch_status(a.status, 6 /* QUOKA_ERR_BOUNDS */);  // the key reads as zeros
      }
    } else if (n - nsel < a.BCP) {
      const int c = n - nsel;
      kr = static_cast<const T*>(a.Kc.data) + bi * a.Kc.sb + j * a.Kc.sh + c * a.Kc.st;
      vr = static_cast<const T*>(a.Vc.data) + bi * a.Vc.sb + j * a.Vc.sh + c * a.Vc.st;
    }
    kp[tid] = kr;
    vp[tid] = vr;
    if (tid == 0) nsel_s = nsel;
  }
  __syncthreads();
  const int nsel = nsel_s;
  const int nk = max(0, min(KS, nsel + a.BCP - n0));  // keys of this slice
  for (int e = tid; e < KS * CPR; e += kThreads) {
    const int k = e / CPR, c = e % CPR;
    const T* kr = kp[k];
    const T* vr = vp[k];
    sm100::cp_async_16(kbase + k * L::ROWB + c * 16, kr ? kr + c * 8 : Q, kr ? 16u : 0u);
    sm100::cp_async_16(vbase + k * L::ROWB + c * 16, vr ? vr + c * 8 : Q, vr ? 16u : 0u);
  }
  sm100::cp_async_commit();
  sm100::cp_async_wait<0>();
  __syncthreads();

  // S = Q K^T for keys [16 warp, 16 warp + 16), scaled, masked, into Ss
  for (int mt = 0; mt < Rp / 16; ++mt) {
    float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int arow = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int k0 = 0; k0 < D; k0 += 32) {
      uint32_t a0[4], a1[4];
      ldsm_x4(qbase + arow * L::ROWB + (k0 + 8 * (lane >> 4)) * 2, a0);
      ldsm_x4(qbase + arow * L::ROWB + (k0 + 16 + 8 * (lane >> 4)) * 2, a1);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t b[4];
        const int key = 16 * warp + 8 * nt + (lane & 7);
        ldsm_x4(kbase + key * L::ROWB + (k0 + 8 * (lane >> 3)) * 2, b);
        mma_bf16_16816(c[nt], a0, b[0], b[1]);
        mma_bf16_16816(c[nt], a1, b[2], b[3]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = mt * 16 + grp + 8 * hf;
        if (r >= R) continue;
        const int k = 16 * warp + 8 * nt + 2 * tig;
        float v[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int n = n0 + k + u;
          const bool vis = k + u < nk && (n < nsel || n - nsel <= r % a.BCP);
          v[u] = vis ? c[nt][2 * hf + u] * qscale : -INFINITY;
        }
        *reinterpret_cast<float2*>(Ss + r * KS + k) = make_float2(v[0], v[1]);
      }
    }
  }
  __syncthreads();

  // per row: max, probabilities 2^(s - m) (bf16 into P), their sum, and the
  // slice's log-sum-exp (one warp per row)
  const int64_t rows = (int64_t)a.b * a.nq * a.BCP;
  for (int r = warp; r < R; r += kThreads / 32) {
    const float s0 = Ss[r * KS + lane], s1 = Ss[r * KS + lane + 32];
    float m = fmaxf(s0, s1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float p0 = m == -INFINITY ? 0.f : exp2f(s0 - m);
    const float p1 = m == -INFINITY ? 0.f : exp2f(s1 - m);
    T* pr = reinterpret_cast<T*>(dsm + L::p_off(Rp) + (size_t)r * L::PROWB);
    pr[lane] = __float2bfloat16_rn(p0);
    pr[lane + 32] = __float2bfloat16_rn(p1);
    float l = p0 + p1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      ml[2 * r] = m;
      ml[2 * r + 1] = l;
      const int h = j * G + r / a.BCP, t = r % a.BCP;
      const int64_t row = ((int64_t)bi * a.nq + h) * a.BCP + t;
      a.lse_parts[(int64_t)s * rows + row] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }
  __syncthreads();

  // O = P V for columns [warp D / 4, (warp + 1) D / 4), normalised by l
  constexpr int NTO = D / 32;  // 8-column tiles per warp
  for (int mt = 0; mt < Rp / 16; ++mt) {
    float o[NTO][4];
#pragma unroll
    for (int nt = 0; nt < NTO; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    const int arow = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int k0 = 0; k0 < KS; k0 += 16) {
      uint32_t pa[4];
      ldsm_x4(pbase + arow * L::PROWB + (k0 + 8 * (lane >> 4)) * 2, pa);
      const int key = k0 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int nt = 0; nt < NTO; nt += 2) {
        uint32_t b[4];
        const int col = warp * (D / 4) + 8 * nt + 8 * (lane >> 4);
        ldsm_x4_trans(vbase + key * L::ROWB + col * 2, b);
        mma_bf16_16816(o[nt], pa, b[0], b[1]);
        mma_bf16_16816(o[nt + 1], pa, b[2], b[3]);
      }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int r = mt * 16 + grp + 8 * hf;
      if (r >= R) continue;
      const float l = ml[2 * r + 1];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int h = j * G + r / a.BCP, t = r % a.BCP;
      const int64_t row = ((int64_t)bi * a.nq + h) * a.BCP + t;
      float* dst = a.O_parts + ((int64_t)s * rows + row) * D + warp * (D / 4) + 2 * tig;
#pragma unroll
      for (int nt = 0; nt < NTO; ++nt)
        *reinterpret_cast<float2*>(dst + 8 * nt) = make_float2(o[nt][2 * hf] * inv, o[nt][2 * hf + 1] * inv);
    }
  }
}

// O = sum_s w_s O_s, w_s = exp(lse_s - LSE), LSE = log sum_s exp(lse_s) over
// the slices of a query row; rows without a visible key (all lse = -inf)
// give O = 0, LSE = -inf. One CTA per query row: the slices are spread over
// groups of threads that each own a 4-column chunk; a thread merges its
// slices in one pass (a running max, sum and output, each slice's lse and
// partial loaded together), then the groups' states are merged in shared
// memory.
template <typename T>
__global__ void __launch_bounds__(kMergeThreads)
decode_merge_kernel(const float* __restrict__ O_parts, const float* __restrict__ lse_parts, int nsplit,
                    int64_t rows, int d, T* __restrict__ O, float* __restrict__ lse) {
  __shared__ float4 part[kMergeThreads];
  __shared__ float pm[kMergeThreads], pl[kMergeThreads];
  pdl_wait();  // the partials come from the slice kernel
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int ncg = d / 4, nsl = kMergeThreads / ncg;
  const int cg = tid % ncg, sl = tid / ncg;
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int BATCH = 8;  // slices whose loads are in flight together
  for (int s0 = sl; s0 < nsplit; s0 += BATCH * nsl) {
    float ls[BATCH];
    float4 x[BATCH];
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const int s = s0 + i * nsl;
      ls[i] = -INFINITY;
      x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s < nsplit) {
        ls[i] = __ldcg(lse_parts + (int64_t)s * rows + row);
        x[i] = __ldcg(reinterpret_cast<const float4*>(O_parts + ((int64_t)s * rows + row) * d) + cg);
      }
    }
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      if (ls[i] > m) {
        const float f = m == -INFINITY ? 0.f : expf(m - ls[i]);
        acc.x *= f;
        acc.y *= f;
        acc.z *= f;
        acc.w *= f;
        l *= f;
        m = ls[i];
      }
      const float w = ls[i] == -INFINITY ? 0.f : expf(ls[i] - m);
      acc.x = fmaf(w, x[i].x, acc.x);
      acc.y = fmaf(w, x[i].y, acc.y);
      acc.z = fmaf(w, x[i].z, acc.z);
      acc.w = fmaf(w, x[i].w, acc.w);
      l += w;
    }
  }
  part[tid] = acc;
  pm[tid] = m;
  pl[tid] = l;
  __syncthreads();
  if (tid < ncg) {
    float M = -INFINITY;
    for (int g = 0; g < nsl; ++g) M = fmaxf(M, pm[g * ncg + tid]);
    float L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < nsl; ++g) {
      const float mg = pm[g * ncg + tid];
      const float f = mg == -INFINITY ? 0.f : expf(mg - M);
      const float4 x = part[g * ncg + tid];
      L = fmaf(f, pl[g * ncg + tid], L);
      o.x = fmaf(f, x.x, o.x);
      o.y = fmaf(f, x.y, o.y);
      o.z = fmaf(f, x.z, o.z);
      o.w = fmaf(f, x.w, o.w);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    T* dst = O + row * d + 4 * tid;
    dst[0] = from_f32<T>(o.x * inv);
    dst[1] = from_f32<T>(o.y * inv);
    dst[2] = from_f32<T>(o.z * inv);
    dst[3] = from_f32<T>(o.w * inv);
    if (tid == 0 && lse != nullptr) lse[row] = L > 0.f ? M + logf(L) : -INFINITY;
  }
}

template <typename T, int D>
cudaError_t launch_typed(const DecodeArgs& a, bool pdl, cudaStream_t stream) {
  const int R = (a.nq / a.nkv) * a.BCP;
  constexpr bool kMma = sizeof(T) == 2;
  auto* kern = kMma ? decode_slice_mma_kernel<D> : decode_slice_kernel<T, D>;
  const size_t smem = kMma ? MmaSliceSmem<D>::bytes((R + 15) & ~15) : SliceSmem<T, D>::bytes(R);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.nsplit, a.nkv, a.b);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)a.b * a.nq * a.BCP;
  cudaLaunchConfig_t mc = {};
  mc.gridDim = dim3((unsigned)rows);  // one CTA per query row
  mc.blockDim = dim3(kMergeThreads);
  mc.stream = stream;
  mc.attrs = attr;
  mc.numAttrs = 1;  // waits for the slices inside
  return cudaLaunchKernelEx(&mc, decode_merge_kernel<T>, static_cast<const float*>(a.O_parts),
                            static_cast<const float*>(a.lse_parts), a.nsplit, rows, D, static_cast<T*>(a.O),
                            a.lse);
}

}  // namespace

int decode_splits(int bsa, int BCP) { return (bsa + BCP + KS - 1) / KS; }

cudaError_t launch_decode_attn(bool bf16, const DecodeArgs& a, bool pdl, cudaStream_t stream) {
  const int R = (a.nq / a.nkv) * a.BCP;
  if (R < 1 || R > kDecodeMaxRows || a.nsplit != decode_splits(a.bsa, a.BCP)) return cudaErrorInvalidValue;
  if (a.d == 128)
    return bf16 ? launch_typed<__nv_bfloat16, 128>(a, pdl, stream) : launch_typed<float, 128>(a, pdl, stream);
  if (a.d == 64)
    return bf16 ? launch_typed<__nv_bfloat16, 64>(a, pdl, stream) : launch_typed<float, 64>(a, pdl, stream);
  return cudaErrorNotSupported;
}

}  // namespace quoka
