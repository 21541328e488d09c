/*
 * quoka.h - C ABI of libquoka.so, the sm_100a (NVIDIA B200) implementation of
 * the QUOKA query-oriented KV-selection step for chunked prefill.
 *
 * Source of the method: the QUOKA technical write-up "QUOKA: how it reshapes
 * LLM prefill efficiency" (bqwf.cn, news item 915859), cited as [QUOKA §x]:
 *   §2.1 Algorithm 1  query subselection: MQ = mean(Q over the chunk's
 *                     tokens), SQ = -cos(Q, MQ), keep the top-NQ queries
 *   §2.2              cosine score S_ij = Q_i.K_j / (|Q_i| |K_j|)
 *   §2.3              GQA-aware aggregation: L2-normalise the chosen queries
 *                     and the keys, mean the queries over each KV head's
 *                     query-head group, score every key against those group
 *                     means (b,nkv,NQ,T), keep each key's largest score over
 *                     the NQ queries (b,nkv,T), and select the BSA keys with
 *                     the highest such score per KV head
 *   §4.2 problem 3    the selected KV is the attention's input KV, with the
 *                     causal mask off for it
 *
 * Shapes and notation: b batch, nq query heads, nkv KV heads, G = nq / nkv,
 * d head dim (64 or 128), BCP chunk length, T prior keys, NQ chosen queries
 * (1 <= NQ <= BCP), BSA key budget, BSA_eff = min(BSA, T). Query head h reads
 * KV head floor(h / G).
 *
 * Conventions shared by every call:
 *   - All tensor data pointers are DEVICE pointers on the current CUDA device;
 *     the caller owns all memory. The library never allocates or frees
 *     device memory; scratch space is the caller's workspace `ws`
 *     (device pointer, at least quoka_workspace_size() bytes, 256-byte
 *     aligned). The one exception is quoka_select_static, whose scratch is a
 *     fixed device array inside the library (see its declaration).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call only enqueues work on it and returns; nothing
 *     synchronises with the host.
 *   - Arguments are validated on the host before anything is enqueued; on an
 *     error return nothing has been enqueued.
 *   - Faults that only the device can see (a key index outside [0, T), a
 *     bounded wait that gave up) are latched into a status word at the start
 *     of `ws` and read back with quoka_get_device_status(). Every call that
 *     takes `ws` clears that word (and the fault-site word after it) on
 *     `stream` before any of its kernels can latch a fault: quoka_select,
 *     quoka_select_ex and quoka_prefill_chunk in their first kernel,
 *     quoka_gather_kv and quoka_decode_attn in a one-thread kernel of their
 *     own, the other calls with an 8-byte memset; a kernel latches only
 *     after the kernel before it in the call has completed. The word
 *     reports the faults of the latest call.
 *   - Calls on different streams with different workspaces may run
 *     concurrently. Two calls sharing one workspace must be ordered.
 */
#ifndef QUOKA_H
#define QUOKA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QUOKA_OK = 0,
  QUOKA_ERR_INVALID_ARG = 1, /* bad shape, stride, pointer or parameter */
  QUOKA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d not 64/128) */
  QUOKA_ERR_WORKSPACE = 3,   /* ws is NULL, misaligned or too small */
  QUOKA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  QUOKA_ERR_TIMEOUT = 5,     /* device: a bounded wait gave up */
  QUOKA_ERR_BOUNDS = 6       /* device: an index was out of range (access skipped) */
} quoka_status;

typedef enum { QUOKA_F32 = 0, QUOKA_BF16 = 1 } quoka_dtype;

/* A strided 4-D view of device memory. Strides are in ELEMENTS; stride[3]
 * must be 1, every other stride must keep each row 16-byte aligned
 * (stride * element size a multiple of 16), and `data` must be 16-byte
 * aligned. Dimensions of extent 0 are allowed where stated; a view with no
 * elements is never read, so its pointer and strides are not checked. */
typedef struct {
  const void* data;
  quoka_dtype dtype;
  int64_t shape[4];
  int64_t stride[4];
} quoka_tensor;

/* Bytes of workspace any call below needs for these sizes (the maximum over
 * the calls, so one workspace serves all of them at their fastest, split
 * key ranges of the attention included; quoka_prefill_chunk needs exactly
 * this much). Returns 0 only for invalid sizes. */
size_t quoka_workspace_size(int b, int nq, int nkv, int d, int64_t T, int BCP,
                            int NQ, int BSA, quoka_dtype dtype);

/* Bytes of workspace quoka_select (and quoka_select_static's scratch) needs
 * for these sizes; at most quoka_workspace_size(). Returns 0 only for
 * invalid sizes. */
size_t quoka_select_workspace_size(int b, int nq, int nkv, int d, int64_t T,
                                   int BCP, int NQ, int BSA, quoka_dtype dtype);

/* Bytes of workspace with which quoka_sparse_gqa_attn takes its fastest path
 * for these sizes: 256 (the status words) plus, for bf16 with d = 128 and
 * BSA_eff > 0, two 256-byte-aligned buffers of b * nkv * BSA_eff * d bf16
 * (the gathered selected K and V). Returns 0 only for invalid sizes. */
size_t quoka_attn_workspace_size(int b, int nkv, int d, int BSA_eff,
                                 quoka_dtype dtype);

/* Steps (a)-(e), [QUOKA §2.1 Algorithm 1, §2.2, §2.3]:
 *   Q (b, nq, BCP, d), K (b, nkv, T, d), same dtype.
 *   kv_idx   out (b, nkv, BSA_eff) int32, contiguous: for each (batch, KV
 *            head) the BSA_eff keys with the largest S_agg, ties to the lower
 *            key index, in ASCENDING key order. This sorted format is the one
 *            quoka_gather_kv and quoka_sparse_gqa_attn read.
 *   kv_count out (b, nkv) int32: number of valid entries per row (BSA_eff).
 *   q_idx    out (b, nq, NQ) int32 or NULL: chosen chunk positions per query
 *            head in rank order (descending SQ, ties to the lower position).
 *   s_agg    out (b, nkv, T) float or NULL: the aggregated key scores.
 * T may be 0 (nothing is selected). */
quoka_status quoka_select(const quoka_tensor* Q, const quoka_tensor* K, int NQ,
                          int BSA, int32_t* kv_idx, int32_t* kv_count,
                          int32_t* q_idx, float* s_agg, void* ws,
                          size_t ws_bytes, void* stream);

/* Score variants of quoka_select_ex (bit flags). */
#define QUOKA_SCORE_DOT_PRODUCT 1u

/* quoka_select with score variants. flags = 0 is quoka_select exactly.
 * QUOKA_SCORE_DOT_PRODUCT: the ablation the write-up compares the cosine
 * score against ([QUOKA §2.2], "standard dot-product attention", its Table
 * 9): the chosen queries are not L2-normalised before the group mean, the
 * keys are not normalised, and S_agg[j, tau] = max_i Q_group[j, i] . K[tau]
 * with Q_group the mean over the G heads of the raw chosen queries. The
 * query choice (steps (a), (b)) is the same. S_agg is then unbounded; the
 * top-k (same ties and output format) runs without the scoring kernel's
 * value-bucket histogram.
 * Other flag bits are rejected with QUOKA_ERR_INVALID_ARG. Arguments
 * otherwise as quoka_select. */
quoka_status quoka_select_ex(const quoka_tensor* Q, const quoka_tensor* K,
                             int NQ, int BSA, int32_t* kv_idx,
                             int32_t* kv_count, int32_t* q_idx, float* s_agg,
                             uint32_t flags, void* ws, size_t ws_bytes,
                             void* stream);

/* Size of the fixed device scratch array behind quoka_select_static. */
#define QUOKA_STATIC_SCRATCH_BYTES (8u << 20)

/* quoka_select without a workspace argument, for callers that cannot
 * allocate device memory: for example a plugin hosted by a framework whose
 * own allocator owns all device memory and forbids raw cudaMalloc, or code on
 * a latency-critical path where cudaMalloc (which may synchronise the device)
 * is not acceptable. The QUOKA write-up has no counterpart of this call; it
 * only changes where the scratch lives.
 *   Arguments, outputs and results are those of quoka_select, minus ws.
 *   Scratch comes from a file-scope device array of
 *   QUOKA_STATIC_SCRATCH_BYTES per device, held by every GPU that loads the
 *   library until the process exits. Shapes whose
 *   quoka_select_workspace_size() exceeds it are rejected with QUOKA_ERR_WORKSPACE before anything is
 *   enqueued. Nothing is allocated (no cudaMalloc or cudaFree, no allocating
 *   library call).
 *   Every call looks up the array's device address in the context current
 *   at the call (cudaGetSymbolAddress), so nothing goes stale after a
 *   cudaDeviceReset or under another context.
 *   All calls on a device share the array and it keeps the last call's
 *   contents (each call clears its status words first; everything else is
 *   rewritten before it is read). Calls that overlap on the GPU race on the
 *   array: order them (one stream, or events between streams).
 *   The device faults of the latest call are read with
 *   quoka_get_device_status(NULL, ...) / quoka_get_device_fault_site(NULL,
 *   ...). */
quoka_status quoka_select_static(const quoka_tensor* Q, const quoka_tensor* K, int NQ,
                                 int BSA, int32_t* kv_idx, int32_t* kv_count,
                                 int32_t* q_idx, float* s_agg, void* stream);

/* Step (f), [QUOKA §4.2 problem 3]: Ksel[b, j, n] = K[b, j, kv_idx[b, j, n]]
 * and the same for V, for n < kv_count[b, j]. Rows past the count, and rows
 * whose index is out of range, are written as zeros (so the output can be
 * handed to quoka_sparse_gqa_attn_gathered as it is).
 *   K, V (b, nkv, T, d); kv_idx (b, nkv, BSA_eff) int32; kv_count (b, nkv).
 *   Ksel, Vsel out (b, nkv, BSA_eff, d), contiguous, dtype of K.
 * An index outside [0, T) is not read and is latched as QUOKA_ERR_BOUNDS in
 * `ws` (which may be NULL, in which case it is only skipped). */
quoka_status quoka_gather_kv(const quoka_tensor* K, const quoka_tensor* V,
                             const int32_t* kv_idx, const int32_t* kv_count,
                             int BSA_eff, void* Ksel, void* Vsel, void* ws,
                             size_t ws_bytes, void* stream);

/* Steps (f)+(g), [QUOKA §4.2 problem 3]: for every query head h, token t,
 *   O[b,h,t] = sum_k softmax_k(scale * Q[b,h,t].k) v
 * over the selected prior keys k = K[b, j, kv_idx[b, j, n]] (n < kv_count,
 * no mask) and the chunk's own keys Kc[b, j, s] with s <= t (causal),
 * j = floor(h / G).
 *   Q (b, nq, BCP, d); K, V (b, nkv, T, d); Kc, Vc (b, nkv, BCP, d).
 *   ws  at least 256 bytes. With ws_bytes >= quoka_attn_workspace_size()
 *       (bf16, d = 128) the selected rows are first gathered into ws (step
 *       (f) as its own kernel, the copy staying in L2) and the attention
 *       streams them as dense tiles; with less, the bf16 attention gathers
 *       the rows itself while loading them (slower, same results). When
 *       the chunk has few 128-row query tiles (b * nq * ceil(BCP / 128) at
 *       most 74) and ws has room past the gathered copy for their partials
 *       (quoka_workspace_size() includes it), each tile's key tiles are
 *       split into 2-4 ranges run side by side and merged by a second
 *       kernel (same results up to rounding).
 *   O   out (b, nq, BCP, d), contiguous, dtype of Q.
 *   lse out (b, nq, BCP) float or NULL: natural-log partition function
 *       log sum_k exp(scale * q.k).
 * bf16 inputs run on the tcgen05 tensor cores (fp32 accumulation and
 * softmax); fp32 inputs run in fp32 on the CUDA cores. */
quoka_status quoka_sparse_gqa_attn(const quoka_tensor* Q, const quoka_tensor* K,
                                   const quoka_tensor* V, const int32_t* kv_idx,
                                   const int32_t* kv_count, int BSA_eff,
                                   const quoka_tensor* Kc, const quoka_tensor* Vc,
                                   float scale, void* O, float* lse, void* ws,
                                   size_t ws_bytes, void* stream);

/* Options of quoka_sparse_gqa_attn_ex (bit flags). */
#define QUOKA_ATTN_NO_CHUNK_KEYS 1u

/* quoka_sparse_gqa_attn with options; flags = 0 is quoka_sparse_gqa_attn
 * exactly. QUOKA_ATTN_NO_CHUNK_KEYS leaves the chunk's own keys (Kc, Vc) out:
 * the softmax runs over the selected keys only. This is one rank's partial
 * attention when the prior keys are split over ranks (only one rank adds the
 * chunk's keys); rows with no visible key give O = 0 and lse = -inf, and
 * quoka_combine_partials merges the ranks' (O, lse). Kc and Vc must still
 * be valid tensors of their usual shape (they are not read). Other flag
 * bits are rejected with QUOKA_ERR_INVALID_ARG. */
quoka_status quoka_sparse_gqa_attn_ex(const quoka_tensor* Q, const quoka_tensor* K,
                                      const quoka_tensor* V,
                                      const int32_t* kv_idx,
                                      const int32_t* kv_count, int BSA_eff,
                                      const quoka_tensor* Kc,
                                      const quoka_tensor* Vc, float scale,
                                      void* O, float* lse, uint32_t flags,
                                      void* ws, size_t ws_bytes, void* stream);

/* Step (g) on a selected KV that is already gathered, [QUOKA §4.2 problem 3]:
 * the attention of quoka_sparse_gqa_attn with key n of KV head j being row
 * n of Ksel[b, j] / Vsel[b, j] (n < kv_count[b, j]) instead of an indexed
 * row of the cache. quoka_sparse_gqa_attn with a full workspace is exactly
 * quoka_gather_kv followed by this call.
 *   Ksel, Vsel (b, nkv, BSA_eff, d), dtype of Q, any 16-byte-aligned row
 *   strides. Rows from kv_count to BSA_eff are masked out but are read: they
 *   must hold finite values (quoka_gather_kv writes zeros there).
 *   kv_count (b, nkv) int32, values above BSA_eff are clamped to it.
 *   ws at least 256 bytes (the status words); room past them for the
 *   partials of split key ranges lets a chunk with few query tiles split
 *   them as quoka_sparse_gqa_attn does. Other arguments as in
 *   quoka_sparse_gqa_attn. */
quoka_status quoka_sparse_gqa_attn_gathered(const quoka_tensor* Q,
                                            const quoka_tensor* Ksel,
                                            const quoka_tensor* Vsel,
                                            const int32_t* kv_count,
                                            const quoka_tensor* Kc,
                                            const quoka_tensor* Vc, float scale,
                                            void* O, float* lse, void* ws,
                                            size_t ws_bytes, void* stream);

/* Steps (f)+(g) for a short chunk: a decode step (BCP = 1) or a short block
 * of speculative tokens, [QUOKA §4.2 problem 3] and its generation-speed use
 * in §4. The same attention as quoka_sparse_gqa_attn (same arguments and
 * layouts; results equal up to rounding), computed for chunks whose G * BCP
 * query rows per KV head are at most 64 (G = nq / nkv), d = 64 or 128: the
 * keys of each KV head (its kv_count selected rows, then its BCP chunk keys)
 * are cut into slices of 64, each slice read by index straight from the
 * cache and attended by all G * BCP query rows of the head in fp32 (bf16 or
 * fp32 inputs), and the slices' partial outputs are merged by their
 * log-sum-exps. quoka_prefill_chunk takes this path by itself for such
 * chunks.
 *   ws  at least quoka_decode_workspace_size() bytes, 256-byte aligned: the
 *       status words, then the fp32 partials.
 * Returns QUOKA_ERR_UNSUPPORTED when G * BCP > 64 or d is not 64 / 128. */
size_t quoka_decode_workspace_size(int b, int nq, int nkv, int d, int BCP,
                                   int BSA_eff, quoka_dtype dtype);
quoka_status quoka_decode_attn(const quoka_tensor* Q, const quoka_tensor* K,
                               const quoka_tensor* V, const int32_t* kv_idx,
                               const int32_t* kv_count, int BSA_eff,
                               const quoka_tensor* Kc, const quoka_tensor* Vc,
                               float scale, void* O, float* lse, void* ws,
                               size_t ws_bytes, void* stream);

/* The whole step (a)-(g), [QUOKA §2.1 Algorithm 1, §2.2, §2.3, §4.2 problem
 * 3]: quoka_select followed by quoka_sparse_gqa_attn on
 * one stream, with no host synchronisation in between; for a short chunk
 * (G * BCP <= 64 query rows per KV head, d = 64 or 128) the attention is
 * quoka_decode_attn's. ws must hold quoka_workspace_size() bytes.
 *   kv_idx_out (b, nkv, BSA_eff) int32 or NULL: the selected set (else kept
 *   in ws). lse may be NULL. */
quoka_status quoka_prefill_chunk(const quoka_tensor* Q, const quoka_tensor* K,
                                 const quoka_tensor* V, const quoka_tensor* Kc,
                                 const quoka_tensor* Vc, int NQ, int BSA,
                                 float scale, void* O, float* lse,
                                 int32_t* kv_idx_out, void* ws, size_t ws_bytes,
                                 void* stream);

/* ---- Prior keys split over ranks (context parallelism) -----------------
 * The T prior keys of every (batch, KV head) are split into contiguous
 * shards, shard r on rank r in ascending order. Each rank runs
 * quoka_select (or quoka_select_ex) on its shard with the global BSA, then:
 *   1. quoka_shard_candidate_scores: its candidates (key indices) and their
 *      scores, padded to C = min(BSA, T_max) (T_max the largest shard;
 *      padding: index -1, score -inf);
 *   2. the ranks exchange the scores (an all-gather: (N, b, nkv, C) floats)
 *      and quoka_shard_interleave lays them out rank-major per row;
 *   3. quoka_topk over the concatenated lists ((b, nkv, N * C) scores) with
 *      BSA_eff = min(BSA, T_total): positions into that list;
 *   4. quoka_shard_take: this rank's share of the selection as key indices
 *      of its shard (ascending) and their count;
 *   5. quoka_sparse_gqa_attn_ex over them (rank 0 alone without
 *      QUOKA_ATTN_NO_CHUNK_KEYS, so the chunk's own keys count once) with
 *      lse;
 *   6. the ranks exchange (O, lse) and quoka_combine_partials merges them.
 * The selection equals the single-device one: every key of the global
 * top-BSA is among its shard's top-BSA, and ties at the BSA-th score go to
 * the lower global index as on one device. The package module
 * sparse_kv_selection_quoka_b200.sharded runs these steps with
 * torch.distributed. */

/* This rank's candidate list padded to length C >= Cl: for
 * n < kv_count[b, j] (clamped to Cl) cand_idx[b, j, n] = kv_idx[b, j, n] and
 * scores[b, j, n] = s_agg[b, j, that index]; for the rest of [0, C)
 * cand_idx = -1 and scores = -inf. s_agg (b, nkv, T) float; kv_idx
 * (b, nkv, Cl) int32 (quoka_select's output); outs (b, nkv, C); all
 * contiguous. An index outside [0, T) is not read (-inf, -1) and latches
 * QUOKA_ERR_BOUNDS in ws (may be NULL). */
quoka_status quoka_shard_candidate_scores(const float* s_agg, int b, int nkv,
                                          int64_t T, const int32_t* kv_idx,
                                          const int32_t* kv_count, int Cl, int C,
                                          float* scores, int32_t* cand_idx,
                                          void* ws, size_t ws_bytes,
                                          void* stream);

/* out[row, r, :] = in[r, row, :] for 32-bit elements: in (N, rows, C) (an
 * all-gather's output), out (rows, N * C), both contiguous and 4-byte
 * aligned. */
quoka_status quoka_shard_interleave(const void* in, int N, int64_t rows,
                                    int64_t C, void* out, void* stream);

/* Step (e) alone, [QUOKA §2.3]: the min(BSA, T) largest of scores (b, nkv, T)
 * float (contiguous) per row, ties to the lower index, ascending, into
 * kv_idx (b, nkv, BSA_eff) and kv_count (b, nkv). ws (may be NULL): the
 * status word. T <= the top-k's limit (QUOKA_ERR_UNSUPPORTED beyond). */
quoka_status quoka_topk(const float* scores, int b, int nkv, int64_t T, int BSA,
                        int32_t* kv_idx, int32_t* kv_count, void* ws,
                        size_t ws_bytes, void* stream);

/* This rank's share of a selection over the ranks' concatenated candidate
 * lists: sel_pos (b, nkv, S) int32 ascending positions in [0, N * C),
 * sel_count (b, nkv) entries valid; cand_idx (b, nkv, C) int32 this rank's
 * candidate key indices (its list is positions [rank * C, (rank + 1) * C)).
 * Out: kv_idx (b, nkv, C) int32, ascending key indices of this rank's
 * picks (entries past the count left as written), kv_count (b, nkv). A pick
 * whose candidate index is negative latches QUOKA_ERR_BOUNDS in ws (may be
 * NULL). */
quoka_status quoka_shard_take(const int32_t* sel_pos, const int32_t* sel_count,
                              int b, int nkv, int S, const int32_t* cand_idx,
                              int C, int rank, int32_t* kv_idx,
                              int32_t* kv_count, void* ws, size_t ws_bytes,
                              void* stream);

/* Merge of N partial attentions over disjoint key sets:
 * O = sum_r exp(lse_r - LSE) O_r, LSE = log sum_r exp(lse_r) per row.
 * O_parts (N, b, nq, BCP, d) of dtype, lse_parts (N, b, nq, BCP) float,
 * O out (b, nq, BCP, d) of dtype, lse out (b, nq, BCP) float or NULL; all
 * contiguous, O_parts and O 16-byte aligned, d in {64, 128}. Rows that every
 * rank saw empty give O = 0, LSE = -inf. */
quoka_status quoka_combine_partials(const void* O_parts, const float* lse_parts,
                                    int N, int b, int nq, int BCP, int d,
                                    quoka_dtype dtype, void* O, float* lse,
                                    void* stream);

/* Synchronises `stream`, then reads the device status word of `ws` into
 * *device_status (a quoka_status value; QUOKA_OK if the latest call that
 * used ws latched no device fault). ws = NULL reads the status word of
 * quoka_select_static's fixed scratch on the current device. Returns
 * QUOKA_ERR_CUDA if the copy or the synchronisation failed,
 * QUOKA_ERR_INVALID_ARG if device_status is NULL. */
quoka_status quoka_get_device_status(const void* ws, void* stream,
                                     int32_t* device_status);

/* Synchronises `stream`, then reads the fault-site word of `ws` (the word
 * after the status word) into *site: 0 when the latest call that used ws
 * latched no device fault, else a small code naming the kernel and the wait
 * or check where the first fault happened (diagnostic only; the codes of
 * the scoring kernel are 51-57, those of the attention 11-15, 21-27 and
 * 31-33). ws = NULL as for quoka_get_device_status. Returns as
 * quoka_get_device_status. */
quoka_status quoka_get_device_fault_site(const void* ws, void* stream,
                                         int32_t* site);

/* Test hooks of the tensor-core scoring and attention kernels (bf16,
 * d = 128). The QUOKA write-up has no counterpart: they exist so that a test
 * can run the timeout path of those kernels without hanging the GPU.
 *   wait_limit_ns  bound of every wait inside those kernels for the launches
 *                  that follow (0 restores the default of 2 s).
 *   inject         QUOKA_DEBUG_INJECT_NONE, or one barrier made to expect
 *                  one arrival more than it ever receives in every launch
 *                  that follows: QUOKA_DEBUG_INJECT_SCORE (the scoring
 *                  kernel's release of its first TMEM accumulator) or
 *                  QUOKA_DEBUG_INJECT_ATTN (the attention's first release
 *                  of P to the P V product). The waiting warp gives up after
 *                  wait_limit_ns, latches QUOKA_ERR_TIMEOUT and a fault site
 *                  in ws, and the kernel unwinds (in-flight copies and
 *                  products drained, TMEM freed); the outputs of that call
 *                  are unspecified.
 * Process-wide and read at launch time: set them only while no other
 * thread launches this library's kernels, and reset them with (0, NONE).
 * Returns QUOKA_ERR_INVALID_ARG for an unknown `inject`. */
#define QUOKA_DEBUG_INJECT_NONE 0u
#define QUOKA_DEBUG_INJECT_SCORE 1u
#define QUOKA_DEBUG_INJECT_ATTN 2u
quoka_status quoka_debug_set_wait_hooks(uint64_t wait_limit_ns, uint32_t inject);

/* A static, human-readable name of a status code. */
const char* quoka_status_string(quoka_status status);

#ifdef __cplusplus
}
#endif

#endif /* QUOKA_H */
