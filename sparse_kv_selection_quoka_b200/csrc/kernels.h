// Host-side launchers of the QUOKA kernels (internal to libquoka.so).
// Every launcher only enqueues work on `stream` and returns the launch
// error (cudaSuccess when the launch was accepted).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace quoka {

// Test hooks, set through quoka_debug_set_wait_hooks and read by the
// launchers of the tensor-core scoring and attention kernels: the bound of
// every wait in those kernels (2 s by default), and an optional fault
// injection that makes one barrier expect one arrival more than it ever
// receives, so that the timeout path (give up, latch QUOKA_ERR_TIMEOUT and a
// fault site, drain, free TMEM, exit) runs without hanging the GPU.
enum : uint32_t { INJECT_NONE = 0u, INJECT_SCORE_TC = 1u, INJECT_ATTN_TMA = 2u };
struct WaitHooks {
  uint64_t wait_ns;
  uint32_t inject;
};
WaitHooks wait_hooks();

// Element-stride description of a (b, heads, rows, d) tensor.
struct Strided {
  const void* data;
  int64_t sb, sh, st;  // strides of batch, head and row, in elements
};

// Step (a)+(b)+(c, first half): one CTA per (batch, query head). Writes the
// chosen chunk positions in rank order and the chosen queries Qhat
// (b, nq, NQ, d) fp32, L2-normalised when `normalize` (the cosine score;
// raw for the dot-product score).
cudaError_t launch_qsel(bool bf16, int d, Strided Q, int b, int nq, int BCP, int NQ,
                        float* Qhat, int32_t* q_idx, bool normalize, cudaStream_t stream);

// Step (c, second half): Q_group (b, nkv, NQ, d) fp32 = mean over the G
// heads of each group of Qhat at the same rank; optionally also the bf16
// hi/lo split (b, nkv, 2*NQ, d): rows [0, NQ) hi, rows [NQ, 2NQ) lo.
// When `hist` is given, also zeroes the (b * nkv, TOPK_HIST_BINS) score
// histogram that the tensor-core scoring kernel fills. When `status` is
// given, clears the call's two status words (the first kernel of a call
// that may latch nothing runs before it).
constexpr int TOPK_HIST_BINS = 4096;
cudaError_t launch_qgroup(int d, const float* Qhat, int b, int nq, int nkv, int NQ,
                          float* Qg, uint16_t* Qg_hilo, uint32_t* hist, int* status, cudaStream_t stream);

// Steps (a)-(c) fused (query selection and group mean in one kernel) for
// bf16, d = 128, BCP <= 512, NQ <= 32, G <= 8, or a one-query chunk
// (BCP = 1, G <= 32): writes q_idx (rank order, when not null), Qg and
// Qg_hilo as launch_qgroup does, zeroes `hist` and clears the status words
// when given; `normalize` as for launch_qsel. Returns
// cudaErrorNotSupported for other shapes.
cudaError_t launch_qsel_group_fast(Strided Q, int b, int nq, int nkv, int BCP, int NQ, int32_t* q_idx,
                                   float* Qg, uint16_t* Qg_hilo, uint32_t* hist, int* status, bool normalize,
                                   cudaStream_t stream);

// Step (d) on the CUDA cores (fp32 arithmetic; any input dtype). key_norm:
// divide by |k| (cosine score) or not (dot-product score).
cudaError_t launch_score_simt(bool bf16, int d, Strided K, int b, int nkv, int64_t T,
                              const float* Qg, int NQ, float* S_agg, bool key_norm, cudaStream_t stream);

// Step (d) on the tcgen05 tensor cores (bf16 K, Q_group as bf16 hi + lo).
// Also accumulates, per (batch, KV head), the histogram of the scores'
// 12-bit value buckets (score_bin) into `hist` (zeroed beforehand), the
// first digit of the top-k select.
// Returns cudaErrorNotSupported when the shape has no tensor-core variant.
// pdl: launch with programmatic stream serialisation (the kernel starts its
// K stream while the previous kernel in the stream still runs). key_norm:
// divide by |k| (cosine score) or not (dot-product score; the histogram is
// then of little use and the caller does not hand it to the top-k).
cudaError_t launch_score_tc(int d, Strided K, int b, int nkv, int64_t T,
                            const uint16_t* Qg_hilo, int NQ, float* S_agg, uint32_t* hist,
                            int* status, bool pdl, bool key_norm, cudaStream_t stream);

// Step (e): per (batch, KV head) cluster radix select of the BSA_eff
// largest scores, ties to the lower index, written in ascending key order.
// Requires 1 <= bsa <= T and T <= topk_max_T().
int64_t topk_max_T();
// `hist`, when not null, is the (b * nkv, TOPK_HIST_BINS) histogram of the
// scores' value buckets made by the scoring kernel; the first pass is then
// skipped.
cudaError_t launch_topk(const float* S_agg, int b, int nkv, int64_t T, int bsa,
                        const uint32_t* hist, int32_t* kv_idx, int32_t* kv_count, int* status,
                        bool pdl, cudaStream_t stream);

// Step (f): gather of the selected K and V rows into contiguous
// (b, nkv, bsa, d) buffers. Rows past kv_count, and rows whose index is out
// of range (latched as QUOKA_ERR_BOUNDS when status is given), are written
// as zeros.
cudaError_t launch_gather(bool bf16, int d, Strided K, Strided V, int b, int nkv, int64_t T,
                          const int32_t* kv_idx, const int32_t* kv_count, int bsa,
                          void* Ksel, void* Vsel, int* status, bool pdl, cudaStream_t stream);

struct AttnArgs {
  Strided Q, K, V, Kc, Vc;
  int b, nq, nkv, d, BCP;
  int64_t T;
  const int32_t* kv_idx;    // (b, nkv, bsa), or null: K/V hold the gathered rows (row n = key n)
  const int32_t* kv_count;  // (b, nkv)
  int bsa;
  float scale;
  void* O;                  // (b, nq, BCP, d) contiguous, dtype of Q
  float* lse;               // (b, nq, BCP) or null
  int* status;
  int no_chunk = 0;         // 1: the chunk's own keys are left out (a shard's partial attention);
                            // rows with no visible key then give O = 0 and lse = -inf
  uint64_t wait_ns = 0;     // bound of every wait (set by the launcher from wait_hooks())
  int inject = 0;           // test hook (set by the launcher from wait_hooks())
  // Split key ranges (tensor-core attention over gathered rows only): with
  // nsplit > 1 every query tile's key tiles are cut into nsplit contiguous
  // ranges, one CTA each; a CTA writes its range's normalised partial output
  // and log-sum-exp, and a merge kernel combines them into O / lse.
  int nsplit = 1;
  void* O_parts = nullptr;     // (nsplit * b, nq, BCP, d) bf16, contiguous
  float* lse_parts = nullptr;  // (nsplit, b, nq, BCP) fp32
};

// Key-range splits of the tensor-core attention for a launch of `tiles`
// 128-row query tiles with at most `nt` key tiles each: 1 when the tiles
// already fill the GPU, else as many ranges (<= 4, each of >= 2 key tiles)
// as keep the CTAs within one wave of kAttnWaveCTAs.
constexpr int kAttnWaveCTAs = 148;  // SMs of a B200: one attention CTA per SM
int attn_splits(int64_t tiles, int nt);

// Steps (f)+(g) in fp32 on the CUDA cores (any input dtype).
cudaError_t launch_attn_simt(bool bf16, const AttnArgs& a, cudaStream_t stream);

// Steps (f)+(g) on the tcgen05 tensor cores (bf16, d = 128; O contiguous).
// With a.kv_idx null (or bsa = 0), a.K / a.V are the gathered selected rows
// (b, nkv, >= bsa, d) and every K/V tile is a TMA box (attn_tma.cu);
// otherwise launch_attn_tc_gather runs, which gathers the rows by index
// while loading them (attn_tc.cu).
// Return cudaErrorNotSupported when the shape has no tensor-core variant.
cudaError_t launch_attn_tc(const AttnArgs& a, bool pdl, cudaStream_t stream);
cudaError_t launch_attn_tc_gather(const AttnArgs& a, cudaStream_t stream);

// Steps (f)+(g) for short chunks (decode steps, short speculative blocks):
// the G * BCP query rows of a KV head together, its keys in slices of 64 (one
// CTA each, rows read by index from the cache), fp32 partial outputs and
// log-sum-exps merged by a second kernel (decode_attn.cu).
constexpr int kDecodeMaxRows = 64;  // G * BCP
struct DecodeArgs {
  Strided Q, K, V, Kc, Vc;  // K, V: the full cache (b, nkv, T, d)
  int b, nq, nkv, d, BCP;
  int64_t T;
  const int32_t* kv_idx;    // (b, nkv, bsa)
  const int32_t* kv_count;  // (b, nkv)
  int bsa;
  float scale;
  float* O_parts;           // (nsplit, b, nq, BCP, d) fp32
  float* lse_parts;         // (nsplit, b, nq, BCP) fp32
  int nsplit;               // decode_splits(bsa, BCP)
  void* O;                  // (b, nq, BCP, d) contiguous, dtype of Q
  float* lse;               // (b, nq, BCP) or null
  int* status;
};
int decode_splits(int bsa, int BCP);
cudaError_t launch_decode_attn(bool bf16, const DecodeArgs& a, bool pdl, cudaStream_t stream);

}  // namespace quoka
