// C ABI of libquoka.so: argument validation, workspace carving and the launch
// sequence of the QUOKA step. See include/quoka.h for the contract of every
// entry point.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "nvtx_range.h"
#include "kernels.h"
#include "quoka.h"

namespace quoka {

namespace {
// Test hooks of quoka_debug_set_wait_hooks (process-wide).
std::atomic<uint64_t> g_wait_ns{0};
std::atomic<uint32_t> g_inject{INJECT_NONE};
}  // namespace

WaitHooks wait_hooks() {
  const uint64_t ns = g_wait_ns.load(std::memory_order_relaxed);
  return WaitHooks{ns == 0 ? 2000000000ull : ns, g_inject.load(std::memory_order_relaxed)};
}

// Device address of quoka_select_static's fixed scratch (select_static.cu).
quoka_status static_scratch_address(void** out);

namespace {

// The status words of a call whose first kernel can itself latch a fault
// are cleared by this one-thread kernel. It lets the call's next kernel
// (launched with programmatic stream serialisation) start at once; that
// kernel's latches wait for this grid to complete first (latch_status).
__global__ void clear_status_kernel(int* status) {
  pdl_trigger();
  status[0] = 0;
  status[1] = 0;
}

}  // namespace

cudaError_t clear_status_async(int* status, cudaStream_t stream) {
  clear_status_kernel<<<1, 1, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace quoka

namespace {

using quoka::Strided;

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Workspace layout. Every region starts on a 256-byte boundary.
struct WsLayout {
  size_t status = 0;    // int32 device status word
  size_t qhat = 0;      // (b, nq, NQ, d) fp32: normalised chosen queries
  size_t qgroup = 0;    // (b, nkv, NQ, d) fp32: group means
  size_t qhilo = 0;     // (b, nkv, 2*NQ, d) bf16: hi / lo split of the group means
  size_t qidx = 0;      // (b, nq, NQ) int32
  size_t sagg = 0;      // (b, nkv, T) fp32
  size_t kvidx = 0;     // (b, nkv, BSA_eff) int32
  size_t kvcount = 0;   // (b, nkv) int32
  size_t hist = 0;      // (b, nkv, 4096) uint32: first-digit histogram of the score keys
  size_t select_total = 0;  // end of what quoka_select needs
  size_t ksel = 0;      // (b, nkv, BSA_eff, d) bf16: gathered selected K (tensor-core attention)
  size_t vsel = 0;      // (b, nkv, BSA_eff, d) bf16: gathered selected V
  size_t aparts = 0;    // split key ranges of the tensor-core attention: partials
  size_t aparts_bytes = 0;
  size_t dparts = 0;    // short chunks: (nsplit, b, nq, BCP, d) fp32 partial outputs
  size_t dlse = 0;      // short chunks: (nsplit, b, nq, BCP) fp32 partial log-sum-exps
  size_t total = 0;
};

// Key-range splits of the tensor-core attention over the gathered rows
// (bf16, d = 128) for a chunk of b * nq * ceil(BCP / 128) query tiles and
// BSA_eff selected keys (with the chunk's own keys unless no_chunk).
int attn_nsplit(int64_t b, int64_t nq, int64_t BCP, int64_t d, int64_t bsa_eff, bool bf16, bool no_chunk) {
  if (!bf16 || d != 128) return 1;
  const int64_t tiles = b * nq * ((BCP + 127) / 128);
  const int64_t nt = (bsa_eff + 127) / 128 + (no_chunk ? 0 : 1);
  return quoka::attn_splits(tiles, (int)std::min<int64_t>(nt, 1 << 20));
}

// Bytes of the partials of `nsplit` key ranges: (nsplit * b, nq, BCP, d)
// bf16 outputs, then (nsplit, b, nq, BCP) fp32 log-sum-exps.
size_t attn_parts_bytes(int64_t b, int64_t nq, int64_t BCP, int64_t d, int nsplit) {
  if (nsplit <= 1) return 0;
  const int64_t rows = (int64_t)nsplit * b * nq * BCP;
  return align_up((size_t)(rows * d) * 2) + align_up((size_t)rows * 4);
}

// Chunks whose G * BCP query rows per KV head fit one CTA of the decode
// attention take it (its fp32 partials live in the workspace).
bool short_chunk(int64_t nq, int64_t nkv, int64_t BCP, int64_t d) {
  return nkv > 0 && nq % nkv == 0 && (nq / nkv) * BCP <= quoka::kDecodeMaxRows && (d == 64 || d == 128);
}

// The tensor-core attention (bf16, d = 128) streams the selected rows from a
// contiguous gathered copy when the workspace holds one.
bool uses_gather_buffers(quoka_dtype dtype, int64_t d, int64_t bsa_eff) {
  return dtype == QUOKA_BF16 && d == 128 && bsa_eff > 0;
}

WsLayout ws_layout(int64_t b, int64_t nq, int64_t nkv, int64_t d, int64_t T, int64_t NQ,
                   int64_t bsa_eff, bool gather_buffers, int64_t BCP = 0, bool decode = false) {
  // (gather_buffers implies bf16, d = 128)
  WsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  L.status = take(kAlign);
  L.qhat = take((size_t)(b * nq * NQ * d) * 4);
  L.qgroup = take((size_t)(b * nkv * NQ * d) * 4);
  L.qhilo = take((size_t)(b * nkv * 2 * NQ * d) * 2);
  L.qidx = take((size_t)(b * nq * NQ) * 4);
  L.sagg = take((size_t)(b * nkv * T) * 4);
  L.kvidx = take((size_t)(b * nkv * bsa_eff) * 4);
  L.kvcount = take((size_t)(b * nkv) * 4);
  L.hist = take((size_t)(b * nkv) * quoka::TOPK_HIST_BINS * 4);
  L.select_total = off;
  if (gather_buffers) {
    L.ksel = take((size_t)(b * nkv * bsa_eff * d) * 2);
    L.vsel = take((size_t)(b * nkv * bsa_eff * d) * 2);
    if (BCP > 0) {
      L.aparts_bytes = attn_parts_bytes(b, nq, BCP, d, attn_nsplit(b, nq, BCP, d, bsa_eff, true, false));
      if (L.aparts_bytes > 0) L.aparts = take(L.aparts_bytes);
    }
  }
  if (decode) {
    const int64_t rows = (int64_t)quoka::decode_splits((int)bsa_eff, (int)BCP) * b * nq * BCP;
    L.dparts = take((size_t)(rows * d) * 4);
    L.dlse = take((size_t)rows * 4);
  }
  L.total = off;
  return L;
}

// Workspace of quoka_decode_attn: the status words, then the partials.
size_t decode_ws_bytes(int64_t b, int64_t nq, int64_t d, int64_t BCP, int64_t bsa_eff) {
  const int64_t rows = (int64_t)quoka::decode_splits((int)bsa_eff, (int)BCP) * b * nq * BCP;
  return kAlign + align_up((size_t)(rows * d) * 4) + align_up((size_t)rows * 4);
}

// Workspace of quoka_sparse_gqa_attn alone: the status words, then (when
// used) the gathered selected K and V.
size_t attn_ws_bytes(int64_t b, int64_t nkv, int64_t d, int64_t bsa_eff, bool gather_buffers) {
  size_t n = kAlign;
  if (gather_buffers) n += 2 * align_up((size_t)(b * nkv * bsa_eff * d) * 2);
  return n;
}

size_t elt_size(quoka_dtype t) { return t == QUOKA_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Checks a tensor's dtype, shape and strides. Extents equal to -1 in `want`
// are free and returned through `want`.
bool check_tensor(const quoka_tensor* t, quoka_dtype dtype, int64_t want[4]) {
  if (t == nullptr) return false;
  if (t->dtype != dtype) return false;
  for (int i = 0; i < 4; ++i) {
    if (t->shape[i] < 0) return false;
    if (want[i] >= 0 && t->shape[i] != want[i]) return false;
    want[i] = t->shape[i];
  }
  int64_t n = 1;
  for (int i = 0; i < 4; ++i) n *= t->shape[i];
  if (n == 0) return true;  // nothing is read: pointer and strides are irrelevant
  if (t->stride[3] != 1) return false;
  const int64_t es = (int64_t)elt_size(dtype);
  for (int i = 0; i < 3; ++i) {
    if (t->stride[i] < 0) return false;
    if ((t->stride[i] * es) % 16 != 0) return false;
  }
  if (t->data == nullptr || !aligned16(t->data)) return false;
  return true;
}

Strided strided(const quoka_tensor* t) {
  return Strided{t->data, t->stride[0], t->stride[1], t->stride[2]};
}

bool supported_d(int64_t d) { return d == 64 || d == 128; }

constexpr int64_t kMaxBCP = 16384;
constexpr int64_t kMaxHeads = 65535;

quoka_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QUOKA_OK;
  if (e == cudaErrorNotSupported) return QUOKA_ERR_UNSUPPORTED;
  return QUOKA_ERR_CUDA;
}

struct SelectShapes {
  int64_t b, nq, nkv, d, T, BCP;
};

quoka_status validate_select(const quoka_tensor* Q, const quoka_tensor* K, int NQ, int BSA,
                             SelectShapes* s) {
  if (Q == nullptr || K == nullptr) return QUOKA_ERR_INVALID_ARG;
  int64_t qs[4] = {-1, -1, -1, -1};
  if (!check_tensor(Q, Q->dtype, qs)) return QUOKA_ERR_INVALID_ARG;
  if (Q->dtype != QUOKA_F32 && Q->dtype != QUOKA_BF16) return QUOKA_ERR_INVALID_ARG;
  int64_t ks[4] = {qs[0], -1, -1, qs[3]};
  if (!check_tensor(K, Q->dtype, ks)) return QUOKA_ERR_INVALID_ARG;
  s->b = qs[0];
  s->nq = qs[1];
  s->BCP = qs[2];
  s->d = qs[3];
  s->nkv = ks[1];
  s->T = ks[2];
  if (s->b < 1 || s->nq < 1 || s->nkv < 1 || s->BCP < 1) return QUOKA_ERR_INVALID_ARG;
  if (s->nq % s->nkv != 0) return QUOKA_ERR_INVALID_ARG;
  if (NQ < 1 || NQ > s->BCP || BSA < 0) return QUOKA_ERR_INVALID_ARG;
  if (!supported_d(s->d)) return QUOKA_ERR_UNSUPPORTED;
  if (s->BCP > kMaxBCP || s->nq > kMaxHeads || s->nkv > kMaxHeads || s->b > kMaxHeads)
    return QUOKA_ERR_UNSUPPORTED;
  if (s->T > quoka::topk_max_T()) return QUOKA_ERR_UNSUPPORTED;
  return QUOKA_OK;
}

quoka_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < need) return QUOKA_ERR_WORKSPACE;
  return QUOKA_OK;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

// Steps (a)-(e) after validation. kv_idx / kv_count / q_idx / s_agg are the
// final destinations (workspace regions when the caller passed none).
// `flags`: QUOKA_SCORE_DOT_PRODUCT selects the plain dot-product score (no
// L2 normalisation of the chosen queries or of the keys).
quoka_status run_select(const quoka_tensor* Q, const quoka_tensor* K, const SelectShapes& s, int NQ,
                        int bsa_eff, int32_t* kv_idx, int32_t* kv_count, int32_t* q_idx,
                        float* s_agg, void* ws, const WsLayout& L, cudaStream_t stream, uint32_t flags = 0u) {
  const bool cosine = (flags & QUOKA_SCORE_DOT_PRODUCT) == 0u;
  const bool bf = Q->dtype == QUOKA_BF16;
  const int b = (int)s.b, nq = (int)s.nq, nkv = (int)s.nkv, d = (int)s.d, BCP = (int)s.BCP;
  float* qhat = at<float>(ws, L.qhat);
  float* qg = at<float>(ws, L.qgroup);
  uint16_t* qhilo = at<uint16_t>(ws, L.qhilo);
  int32_t* qidx = q_idx != nullptr ? q_idx : at<int32_t>(ws, L.qidx);
  float* sagg = s_agg != nullptr ? s_agg : at<float>(ws, L.sagg);
  int* status = at<int>(ws, L.status);
  uint32_t* hist = at<uint32_t>(ws, L.hist);

  cudaError_t e = cudaErrorNotSupported;
  if (bf && d == 128)
    e = quoka::launch_qsel_group_fast(strided(Q), b, nq, nkv, BCP, NQ, qidx, qg, qhilo, hist, status, cosine,
                                      stream);
  if (e == cudaErrorNotSupported) {
    e = quoka::launch_qsel(bf, d, strided(Q), b, nq, BCP, NQ, qhat, qidx, cosine, stream);
    if (e != cudaSuccess) return cuda_status(e);
    e = quoka::launch_qgroup(d, qhat, b, nq, nkv, NQ, qg, bf ? qhilo : nullptr, bf ? hist : nullptr, status,
                             stream);
  }
  if (e != cudaSuccess) return cuda_status(e);
  bool hist_made = false;
  if (s.T > 0) {
    e = cudaErrorNotSupported;
    if (bf) {
      e = quoka::launch_score_tc(d, strided(K), b, nkv, s.T, qhilo, NQ, sagg, hist, status, true, cosine,
                                 stream);
      // the value-bucket histogram spans the cosine range [-1, 1]
      hist_made = e == cudaSuccess && cosine;
    }
    if (e == cudaErrorNotSupported)
      e = quoka::launch_score_simt(bf, d, strided(K), b, nkv, s.T, qg, NQ, sagg, cosine, stream);
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (bsa_eff > 0) {
    e = quoka::launch_topk(sagg, b, nkv, s.T, bsa_eff, hist_made ? hist : nullptr, kv_idx, kv_count, status,
                           true, stream);
    if (e != cudaSuccess) return cuda_status(e);
  } else {
    e = cudaMemsetAsync(kv_count, 0, sizeof(int32_t) * b * nkv, stream);
    if (e != cudaSuccess) return QUOKA_ERR_CUDA;
  }
  return QUOKA_OK;
}

struct AttnShapes {
  int64_t b, nq, nkv, d, T, BCP;
};

quoka_status validate_attn(const quoka_tensor* Q, const quoka_tensor* K, const quoka_tensor* V,
                           const quoka_tensor* Kc, const quoka_tensor* Vc, AttnShapes* s) {
  if (Q == nullptr || K == nullptr || V == nullptr || Kc == nullptr || Vc == nullptr)
    return QUOKA_ERR_INVALID_ARG;
  int64_t qs[4] = {-1, -1, -1, -1};
  if (!check_tensor(Q, Q->dtype, qs)) return QUOKA_ERR_INVALID_ARG;
  if (Q->dtype != QUOKA_F32 && Q->dtype != QUOKA_BF16) return QUOKA_ERR_INVALID_ARG;
  int64_t ks[4] = {qs[0], -1, -1, qs[3]};
  if (!check_tensor(K, Q->dtype, ks)) return QUOKA_ERR_INVALID_ARG;
  int64_t vs[4] = {ks[0], ks[1], ks[2], ks[3]};
  if (!check_tensor(V, Q->dtype, vs)) return QUOKA_ERR_INVALID_ARG;
  int64_t kcs[4] = {qs[0], ks[1], qs[2], qs[3]};
  if (!check_tensor(Kc, Q->dtype, kcs)) return QUOKA_ERR_INVALID_ARG;
  int64_t vcs[4] = {qs[0], ks[1], qs[2], qs[3]};
  if (!check_tensor(Vc, Q->dtype, vcs)) return QUOKA_ERR_INVALID_ARG;
  s->b = qs[0];
  s->nq = qs[1];
  s->BCP = qs[2];
  s->d = qs[3];
  s->nkv = ks[1];
  s->T = ks[2];
  if (s->b < 1 || s->nq < 1 || s->nkv < 1 || s->BCP < 1) return QUOKA_ERR_INVALID_ARG;
  if (s->nq % s->nkv != 0) return QUOKA_ERR_INVALID_ARG;
  if (!supported_d(s->d)) return QUOKA_ERR_UNSUPPORTED;
  if (s->BCP > kMaxBCP || s->nq > kMaxHeads || s->nkv > kMaxHeads || s->b > kMaxHeads)
    return QUOKA_ERR_UNSUPPORTED;
  if (s->T > (int64_t)INT32_MAX) return QUOKA_ERR_UNSUPPORTED;
  return QUOKA_OK;
}

// Step (g) (with step (f) fused into the loads when kv_idx is given; with
// kv_idx null, K / V are the gathered selected rows and T their row count).
quoka_status run_attn(const quoka_tensor* Q, Strided K, Strided V, const quoka_tensor* Kc,
                      const quoka_tensor* Vc, const AttnShapes& s, int64_t T, const int32_t* kv_idx,
                      const int32_t* kv_count, int bsa_eff, float scale, void* O, float* lse,
                      int* status, cudaStream_t stream, bool pdl = false, bool no_chunk = false,
                      void* parts = nullptr, size_t parts_bytes = 0) {
  quoka::AttnArgs a;
  a.no_chunk = no_chunk ? 1 : 0;
  a.Q = strided(Q);
  a.K = K;
  a.V = V;
  a.Kc = strided(Kc);
  a.Vc = strided(Vc);
  a.b = (int)s.b;
  a.nq = (int)s.nq;
  a.nkv = (int)s.nkv;
  a.d = (int)s.d;
  a.BCP = (int)s.BCP;
  a.T = T;
  a.kv_idx = kv_idx;
  a.kv_count = kv_count;
  a.bsa = bsa_eff;
  a.scale = scale;
  a.O = O;
  a.lse = lse;
  a.status = status;
  if (kv_idx == nullptr && parts != nullptr) {
    // split key ranges when the query tiles leave most SMs idle and the
    // workspace holds the partials
    const int ns = attn_nsplit(s.b, s.nq, s.BCP, s.d, bsa_eff, Q->dtype == QUOKA_BF16, no_chunk);
    if (ns > 1 && parts_bytes >= attn_parts_bytes(s.b, s.nq, s.BCP, s.d, ns)) {
      const int64_t rows = (int64_t)ns * s.b * s.nq * s.BCP;
      a.nsplit = ns;
      a.O_parts = parts;
      a.lse_parts = reinterpret_cast<float*>(static_cast<char*>(parts) + align_up((size_t)(rows * s.d) * 2));
    }
  }
  cudaError_t e = cudaErrorNotSupported;
  if (Q->dtype == QUOKA_BF16) e = quoka::launch_attn_tc(a, pdl, stream);
  if (e == cudaErrorNotSupported) e = quoka::launch_attn_simt(Q->dtype == QUOKA_BF16, a, stream);
  return cuda_status(e);
}

// Steps (f)+(g) on the full cache K / V: when `gathered` (the workspace's
// Ksel / Vsel buffers) is given, step (f) runs as its own kernel into it and
// the attention streams the copy; otherwise the attention gathers in place.
quoka_status gather_then_attn(const quoka_tensor* Q, const quoka_tensor* K, const quoka_tensor* V,
                              const quoka_tensor* Kc, const quoka_tensor* Vc, const AttnShapes& s,
                              const int32_t* kv_idx, const int32_t* kv_count, int bsa_eff, float scale,
                              void* O, float* lse, void* ksel, void* vsel, int* status,
                              cudaStream_t stream, bool no_chunk = false, void* parts = nullptr,
                              size_t parts_bytes = 0) {
  if (ksel == nullptr || vsel == nullptr || bsa_eff == 0)
    return run_attn(Q, strided(K), strided(V), Kc, Vc, s, s.T, kv_idx, kv_count, bsa_eff, scale, O, lse,
                    status, stream, false, no_chunk);
  cudaError_t e = quoka::launch_gather(Q->dtype == QUOKA_BF16, (int)s.d, strided(K), strided(V), (int)s.b,
                                       (int)s.nkv, s.T, kv_idx, kv_count, bsa_eff, ksel, vsel, status, true,
                                       stream);
  if (e != cudaSuccess) return cuda_status(e);
  const int64_t sh = (int64_t)bsa_eff * s.d, sb = s.nkv * sh;
  // the attention may launch while the gather finishes (it waits for it)
  return run_attn(Q, Strided{ksel, sb, sh, s.d}, Strided{vsel, sb, sh, s.d}, Kc, Vc, s, bsa_eff, nullptr,
                  kv_count, bsa_eff, scale, O, lse, status, stream, true, no_chunk, parts, parts_bytes);
}

// Steps (f)+(g) for a short chunk (short_chunk()): the slice kernel reads the
// selected rows by index from the cache, then the merge kernel.
quoka_status run_decode(const quoka_tensor* Q, const quoka_tensor* K, const quoka_tensor* V,
                        const quoka_tensor* Kc, const quoka_tensor* Vc, const AttnShapes& s,
                        const int32_t* kv_idx, const int32_t* kv_count, int bsa_eff, float scale, void* O,
                        float* lse, float* O_parts, float* lse_parts, int* status, cudaStream_t stream,
                        bool pdl) {
  quoka::DecodeArgs a;
  a.Q = strided(Q);
  a.K = strided(K);
  a.V = strided(V);
  a.Kc = strided(Kc);
  a.Vc = strided(Vc);
  a.b = (int)s.b;
  a.nq = (int)s.nq;
  a.nkv = (int)s.nkv;
  a.d = (int)s.d;
  a.BCP = (int)s.BCP;
  a.T = s.T;
  a.kv_idx = kv_idx;
  a.kv_count = kv_count;
  a.bsa = bsa_eff;
  a.scale = scale;
  a.O_parts = O_parts;
  a.lse_parts = lse_parts;
  a.nsplit = quoka::decode_splits(bsa_eff, (int)s.BCP);
  a.O = O;
  a.lse = lse;
  a.status = status;
  return cuda_status(quoka::launch_decode_attn(Q->dtype == QUOKA_BF16, a, pdl, stream));
}

}  // namespace

extern "C" {

size_t quoka_workspace_size(int b, int nq, int nkv, int d, int64_t T, int BCP, int NQ, int BSA,
                            quoka_dtype dtype) {
  if (b < 1 || nq < 1 || nkv < 1 || d < 1 || T < 0 || BCP < 1 || NQ < 1 || BSA < 0) return 0;
  if (nq % nkv != 0 || (dtype != QUOKA_F32 && dtype != QUOKA_BF16)) return 0;
  const int64_t bsa_eff = std::min<int64_t>(BSA, T);
  const bool dec = short_chunk(nq, nkv, BCP, d);
  // (a short chunk's layout keeps the gather buffers too: the same workspace
  // then also gives quoka_sparse_gqa_attn its fastest path)
  return ws_layout(b, nq, nkv, d, T, NQ, bsa_eff, uses_gather_buffers(dtype, d, bsa_eff), BCP, dec).total;
}

size_t quoka_select_workspace_size(int b, int nq, int nkv, int d, int64_t T, int BCP, int NQ, int BSA,
                                   quoka_dtype dtype) {
  if (quoka_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, dtype) == 0) return 0;
  const int64_t bsa_eff = std::min<int64_t>(BSA, T);
  return ws_layout(b, nq, nkv, d, T, NQ, bsa_eff, false).select_total;
}

size_t quoka_attn_workspace_size(int b, int nkv, int d, int BSA_eff, quoka_dtype dtype) {
  if (b < 1 || nkv < 1 || d < 1 || BSA_eff < 0) return 0;
  if (dtype != QUOKA_F32 && dtype != QUOKA_BF16) return 0;
  return attn_ws_bytes(b, nkv, d, BSA_eff, uses_gather_buffers(dtype, d, BSA_eff));
}

quoka_status quoka_select(const quoka_tensor* Q, const quoka_tensor* K, int NQ, int BSA,
                          int32_t* kv_idx, int32_t* kv_count, int32_t* q_idx, float* s_agg,
                          void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_select");
  return quoka_select_ex(Q, K, NQ, BSA, kv_idx, kv_count, q_idx, s_agg, 0u, ws, ws_bytes, stream);
}

quoka_status quoka_select_ex(const quoka_tensor* Q, const quoka_tensor* K, int NQ, int BSA,
                             int32_t* kv_idx, int32_t* kv_count, int32_t* q_idx, float* s_agg,
                             uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_select_ex");
  if ((flags & ~QUOKA_SCORE_DOT_PRODUCT) != 0u) return QUOKA_ERR_INVALID_ARG;
  SelectShapes s;
  quoka_status st = validate_select(Q, K, NQ, BSA, &s);
  if (st != QUOKA_OK) return st;
  const int64_t bsa_eff = std::min<int64_t>(BSA, s.T);
  if (kv_count == nullptr || (bsa_eff > 0 && kv_idx == nullptr)) return QUOKA_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(s.b, s.nq, s.nkv, s.d, s.T, NQ, bsa_eff, false);
  st = check_ws(ws, ws_bytes, L.select_total);
  if (st != QUOKA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // (the status words are cleared by the first kernel)
  return run_select(Q, K, s, NQ, (int)bsa_eff, kv_idx, kv_count, q_idx, s_agg, ws, L, cs, flags);
}

quoka_status quoka_gather_kv(const quoka_tensor* K, const quoka_tensor* V, const int32_t* kv_idx,
                             const int32_t* kv_count, int BSA_eff, void* Ksel, void* Vsel,
                             void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_gather_kv");
  if (K == nullptr || V == nullptr || kv_count == nullptr || BSA_eff < 0) return QUOKA_ERR_INVALID_ARG;
  int64_t ks[4] = {-1, -1, -1, -1};
  if (!check_tensor(K, K->dtype, ks)) return QUOKA_ERR_INVALID_ARG;
  if (K->dtype != QUOKA_F32 && K->dtype != QUOKA_BF16) return QUOKA_ERR_INVALID_ARG;
  int64_t vs[4] = {ks[0], ks[1], ks[2], ks[3]};
  if (!check_tensor(V, K->dtype, vs)) return QUOKA_ERR_INVALID_ARG;
  if (!supported_d(ks[3])) return QUOKA_ERR_UNSUPPORTED;
  if (ks[0] < 1 || ks[1] < 1 || ks[0] > kMaxHeads || ks[1] > kMaxHeads) return QUOKA_ERR_INVALID_ARG;
  if (BSA_eff > 0 && (kv_idx == nullptr || Ksel == nullptr || Vsel == nullptr || !aligned16(Ksel) ||
                      !aligned16(Vsel)))
    return QUOKA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = nullptr;
  if (ws != nullptr) {
    if (((uintptr_t)ws % kAlign) != 0 || ws_bytes < 2 * sizeof(int)) return QUOKA_ERR_WORKSPACE;
    status = static_cast<int*>(ws);
    if (quoka::clear_status_async(status, cs) != cudaSuccess) return QUOKA_ERR_CUDA;
  }
  cudaError_t e = quoka::launch_gather(K->dtype == QUOKA_BF16, (int)ks[3], strided(K), strided(V),
                                       (int)ks[0], (int)ks[1], ks[2], kv_idx, kv_count, BSA_eff, Ksel,
                                       Vsel, status, true, cs);
  return cuda_status(e);
}

quoka_status quoka_sparse_gqa_attn(const quoka_tensor* Q, const quoka_tensor* K,
                                   const quoka_tensor* V, const int32_t* kv_idx,
                                   const int32_t* kv_count, int BSA_eff, const quoka_tensor* Kc,
                                   const quoka_tensor* Vc, float scale, void* O, float* lse,
                                   void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_sparse_gqa_attn");
  return quoka_sparse_gqa_attn_ex(Q, K, V, kv_idx, kv_count, BSA_eff, Kc, Vc, scale, O, lse, 0u, ws, ws_bytes,
                                  stream);
}

quoka_status quoka_sparse_gqa_attn_ex(const quoka_tensor* Q, const quoka_tensor* K,
                                      const quoka_tensor* V, const int32_t* kv_idx,
                                      const int32_t* kv_count, int BSA_eff, const quoka_tensor* Kc,
                                      const quoka_tensor* Vc, float scale, void* O, float* lse,
                                      uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_sparse_gqa_attn_ex");
  if ((flags & ~QUOKA_ATTN_NO_CHUNK_KEYS) != 0u) return QUOKA_ERR_INVALID_ARG;
  const bool no_chunk = (flags & QUOKA_ATTN_NO_CHUNK_KEYS) != 0u;
  AttnShapes s;
  quoka_status st = validate_attn(Q, K, V, Kc, Vc, &s);
  if (st != QUOKA_OK) return st;
  if (BSA_eff < 0 || kv_count == nullptr || (BSA_eff > 0 && kv_idx == nullptr)) return QUOKA_ERR_INVALID_ARG;
  if (O == nullptr || !aligned16(O)) return QUOKA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return QUOKA_ERR_INVALID_ARG;
  if (ws == nullptr || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < kAlign) return QUOKA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  // (a memset here: launched early behind a clear kernel, the attention measured ~2 us slower)
  if (cudaMemsetAsync(status, 0, 2 * sizeof(int), cs) != cudaSuccess) return QUOKA_ERR_CUDA;
  // with room for the gathered copy, the selected rows are gathered first
  void* ksel = nullptr;
  void* vsel = nullptr;
  void* parts = nullptr;
  size_t parts_bytes = 0;
  const bool gb = uses_gather_buffers(Q->dtype, s.d, BSA_eff);
  const size_t gb_end = attn_ws_bytes(s.b, s.nkv, s.d, BSA_eff, true);
  if (gb && ws_bytes >= gb_end) {
    ksel = static_cast<char*>(ws) + kAlign;
    vsel = static_cast<char*>(ksel) + align_up((size_t)(s.b * s.nkv * BSA_eff * s.d) * 2);
    // (room past the gathered copy takes the split ranges' partials)
    parts = static_cast<char*>(ws) + gb_end;
    parts_bytes = ws_bytes - gb_end;
  }
  return gather_then_attn(Q, K, V, Kc, Vc, s, kv_idx, kv_count, BSA_eff, scale, O, lse, ksel, vsel, status,
                          cs, no_chunk, parts, parts_bytes);
}

quoka_status quoka_sparse_gqa_attn_gathered(const quoka_tensor* Q, const quoka_tensor* Ksel,
                                            const quoka_tensor* Vsel, const int32_t* kv_count,
                                            const quoka_tensor* Kc, const quoka_tensor* Vc, float scale,
                                            void* O, float* lse, void* ws, size_t ws_bytes,
                                            void* stream) {
  quoka::NvtxRange nvtx_range("quoka_sparse_gqa_attn_gathered");
  AttnShapes s;
  quoka_status st = validate_attn(Q, Ksel, Vsel, Kc, Vc, &s);
  if (st != QUOKA_OK) return st;
  if (kv_count == nullptr) return QUOKA_ERR_INVALID_ARG;
  if (O == nullptr || !aligned16(O)) return QUOKA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return QUOKA_ERR_INVALID_ARG;
  if (ws == nullptr || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < kAlign) return QUOKA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  // (a memset here: launched early behind a clear kernel, the attention measured ~2 us slower)
  if (cudaMemsetAsync(status, 0, 2 * sizeof(int), cs) != cudaSuccess) return QUOKA_ERR_CUDA;
  // the rows of Ksel / Vsel are the selected keys in list order: BSA_eff = T
  // (room past the status words takes the split ranges' partials)
  return run_attn(Q, strided(Ksel), strided(Vsel), Kc, Vc, s, s.T, nullptr, kv_count, (int)s.T, scale, O,
                  lse, status, cs, true, false, static_cast<char*>(ws) + kAlign, ws_bytes - kAlign);
}

size_t quoka_decode_workspace_size(int b, int nq, int nkv, int d, int BCP, int BSA_eff, quoka_dtype dtype) {
  if (b < 1 || nq < 1 || nkv < 1 || BCP < 1 || BSA_eff < 0) return 0;
  if (dtype != QUOKA_F32 && dtype != QUOKA_BF16) return 0;
  if (!short_chunk(nq, nkv, BCP, d)) return 0;
  return decode_ws_bytes(b, nq, d, BCP, BSA_eff);
}

quoka_status quoka_decode_attn(const quoka_tensor* Q, const quoka_tensor* K, const quoka_tensor* V,
                               const int32_t* kv_idx, const int32_t* kv_count, int BSA_eff,
                               const quoka_tensor* Kc, const quoka_tensor* Vc, float scale, void* O,
                               float* lse, void* ws, size_t ws_bytes, void* stream) {
  quoka::NvtxRange nvtx_range("quoka_decode_attn");
  AttnShapes s;
  quoka_status st = validate_attn(Q, K, V, Kc, Vc, &s);
  if (st != QUOKA_OK) return st;
  if (!short_chunk(s.nq, s.nkv, s.BCP, s.d)) return QUOKA_ERR_UNSUPPORTED;
  if (BSA_eff < 0 || kv_count == nullptr || (BSA_eff > 0 && kv_idx == nullptr)) return QUOKA_ERR_INVALID_ARG;
  if (O == nullptr || !aligned16(O)) return QUOKA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return QUOKA_ERR_INVALID_ARG;
  const size_t need = decode_ws_bytes(s.b, s.nq, s.d, s.BCP, BSA_eff);
  if (ws == nullptr || ((uintptr_t)ws % kAlign) != 0 || ws_bytes < need) return QUOKA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  if (quoka::clear_status_async(status, cs) != cudaSuccess) return QUOKA_ERR_CUDA;
  const int64_t rows = (int64_t)quoka::decode_splits(BSA_eff, (int)s.BCP) * s.b * s.nq * s.BCP;
  float* O_parts = reinterpret_cast<float*>(static_cast<char*>(ws) + kAlign);
  float* lse_parts = reinterpret_cast<float*>(reinterpret_cast<char*>(O_parts) + align_up((size_t)(rows * s.d) * 4));
  return run_decode(Q, K, V, Kc, Vc, s, kv_idx, kv_count, BSA_eff, scale, O, lse, O_parts, lse_parts, status, cs,
                    true);
}

quoka_status quoka_prefill_chunk(const quoka_tensor* Q, const quoka_tensor* K,
                                 const quoka_tensor* V, const quoka_tensor* Kc,
                                 const quoka_tensor* Vc, int NQ, int BSA, float scale, void* O,
                                 float* lse, int32_t* kv_idx_out, void* ws, size_t ws_bytes,
                                 void* stream) {
  quoka::NvtxRange nvtx_range("quoka_prefill_chunk");
  AttnShapes as;
  quoka_status st = validate_attn(Q, K, V, Kc, Vc, &as);
  if (st != QUOKA_OK) return st;
  SelectShapes s;
  st = validate_select(Q, K, NQ, BSA, &s);
  if (st != QUOKA_OK) return st;
  if (O == nullptr || !aligned16(O)) return QUOKA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return QUOKA_ERR_INVALID_ARG;
  const int64_t bsa_eff = std::min<int64_t>(BSA, s.T);
  const bool dec = short_chunk(s.nq, s.nkv, s.BCP, s.d);
  const bool gb = uses_gather_buffers(Q->dtype, s.d, bsa_eff);
  const WsLayout L = ws_layout(s.b, s.nq, s.nkv, s.d, s.T, NQ, bsa_eff, gb, s.BCP, dec);
  st = check_ws(ws, ws_bytes, L.total);
  if (st != QUOKA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int* status = at<int>(ws, L.status);  // cleared by the selection's first kernel
  int32_t* kv_idx = kv_idx_out != nullptr ? kv_idx_out : at<int32_t>(ws, L.kvidx);
  int32_t* kv_count = at<int32_t>(ws, L.kvcount);
  st = run_select(Q, K, s, NQ, (int)bsa_eff, kv_idx, kv_count, nullptr, nullptr, ws, L, cs);
  if (st != QUOKA_OK) return st;
  if (dec)  // a short chunk: the decode attention (waits for the selection's last kernel)
    return run_decode(Q, K, V, Kc, Vc, as, kv_idx, kv_count, (int)bsa_eff, scale, O, lse, at<float>(ws, L.dparts),
                      at<float>(ws, L.dlse), status, cs, true);
  return gather_then_attn(Q, K, V, Kc, Vc, as, kv_idx, kv_count, (int)bsa_eff, scale, O, lse,
                          gb ? at<void>(ws, L.ksel) : nullptr, gb ? at<void>(ws, L.vsel) : nullptr, status, cs,
                          false, L.aparts_bytes > 0 ? at<void>(ws, L.aparts) : nullptr, L.aparts_bytes);
}

quoka_status quoka_get_device_status(const void* ws, void* stream, int32_t* device_status) {
  quoka::NvtxRange nvtx_range("quoka_get_device_status");
  if (device_status == nullptr) return QUOKA_ERR_INVALID_ARG;
  if (ws == nullptr) {  // the fixed scratch of quoka_select_static
    void* p = nullptr;
    const quoka_status st = quoka::static_scratch_address(&p);
    if (st != QUOKA_OK) return st;
    ws = p;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return QUOKA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return QUOKA_ERR_CUDA;
  *device_status = v;
  return QUOKA_OK;
}

quoka_status quoka_get_device_fault_site(const void* ws, void* stream, int32_t* site) {
  quoka::NvtxRange nvtx_range("quoka_get_device_fault_site");
  if (site == nullptr) return QUOKA_ERR_INVALID_ARG;
  if (ws == nullptr) {  // the fixed scratch of quoka_select_static
    void* p = nullptr;
    const quoka_status st = quoka::static_scratch_address(&p);
    if (st != QUOKA_OK) return st;
    ws = p;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, static_cast<const int32_t*>(ws) + 1, sizeof(int32_t), cudaMemcpyDeviceToHost, cs) !=
      cudaSuccess)
    return QUOKA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return QUOKA_ERR_CUDA;
  *site = v;
  return QUOKA_OK;
}

quoka_status quoka_debug_set_wait_hooks(uint64_t wait_limit_ns, uint32_t inject) {
  if (inject > QUOKA_DEBUG_INJECT_ATTN) return QUOKA_ERR_INVALID_ARG;
  quoka::g_wait_ns.store(wait_limit_ns, std::memory_order_relaxed);
  quoka::g_inject.store(inject, std::memory_order_relaxed);
  return QUOKA_OK;
}

const char* quoka_status_string(quoka_status status) {
  switch (status) {
    case QUOKA_OK: return "QUOKA_OK";
    case QUOKA_ERR_INVALID_ARG: return "QUOKA_ERR_INVALID_ARG";
    case QUOKA_ERR_UNSUPPORTED: return "QUOKA_ERR_UNSUPPORTED";
    case QUOKA_ERR_WORKSPACE: return "QUOKA_ERR_WORKSPACE";
    case QUOKA_ERR_CUDA: return "QUOKA_ERR_CUDA";
    case QUOKA_ERR_TIMEOUT: return "QUOKA_ERR_TIMEOUT";
    case QUOKA_ERR_BOUNDS: return "QUOKA_ERR_BOUNDS";
  }
  return "QUOKA_ERR_UNKNOWN";
}

}  // extern "C"
