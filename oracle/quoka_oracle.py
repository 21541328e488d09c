"""CPU oracle of the QUOKA prefill-chunk step, in float64 numpy.

TEST INFRASTRUCTURE ONLY. This module is a plain, slow, obviously correct
restatement of what the method computes. Only the test suite, the smoke check
and the benchmark's CPU-baseline leg may import it. The product path (the CUDA
library and its Python binding) never imports, calls or links it, and this
module imports nothing from the product.

Source: the QUOKA technical write-up "QUOKA: how it reshapes LLM prefill
efficiency" (bqwf.cn, news item 915859), cited below as [QUOKA §x]:
  §1.1   key idea: queries with low cosine to the mean query matter most
  §2.1   query subselection (Algorithm 1): MQ = mean(Q), SQ = -cos(Q, MQ),
         keep the top-NQ queries by SQ
  §2.2   cosine score S_ij = Q_i.K_j / (|Q_i| |K_j|)
  §2.3   GQA-aware aggregation: L2-normalise the chosen queries and the keys,
         mean the queries over each KV head's query-head group, score with a
         matmul, take the max over the chosen queries, keep the top-BSA keys
  §4.2   the selected KV is handed to FlashAttention as its input KV with the
         causal mask switched off for it (problem 3)
  §2.2   also: the cosine score is compared against the standard dot-product
         score (its Table 9); the dot_product=True variant below drops both
         L2 normalisations (chosen queries and keys) and keeps everything else

Readings where the article is silent or garbled (each is listed in the design
notes too):
  * The queries are the chunk (BCP of them); the keys are the T prior keys of
    the cache. The chunk's own keys are not scored; they join the attention
    causally.
  * cos(Q, MQ) is taken along the head dimension d, with MQ broadcast over the
    chunk's tokens; the norm product is clamped below at 1e-8.
  * topk returns its picks in descending score order; ties go to the lower
    index. Position i of every query head of a group is averaged with
    position i of the group's other heads (the reshape + mean over the group
    axis in §2.3).
  * Query head h belongs to KV head floor(h / G), G = nq / nkv.
  * BSA_eff = min(BSA, T); T = 0 selects nothing. Ties at the BSA-th score go
    to the lower key index. Selected indices are returned in ascending order.
  * Attention: scale 1/sqrt(d); no mask over the selected prior keys; causal
    (key s <= query t) over the chunk's own keys.

Parity unpinned: nothing in the article prints a worked numeric example, so the
exact values of SQ, S_agg and O are pinned only through the closed forms,
invariants, special cases and brute-force checks in the test suite, not by
printed numbers.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

__all__ = [
    "mean_query",
    "query_scores",
    "select_queries",
    "group_queries",
    "key_scores",
    "select_keys",
    "gather_kv",
    "sparse_attention",
    "sparse_attention_rows",
    "select",
    "prefill_chunk",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Step (a): mean query and query scores  [QUOKA §2.1, Algorithm 1]
# ---------------------------------------------------------------------------

def mean_query(Q) -> np.ndarray:
    """MQ[b, h] = (1/BCP) sum_t Q[b, h, t]   -> (b, nq, d)."""
    Q = _f64(Q)
    return Q.sum(axis=2) / Q.shape[2]


def query_scores(Q) -> np.ndarray:
    """SQ[b, h, t] = -cos(Q[b, h, t], MQ[b, h])   -> (b, nq, BCP).

    [QUOKA §2.1]: the priority of a query is the negative cosine between it
    and the mean query; outliers (low cosine) get the highest priority."""
    Q = _f64(Q)
    MQ = mean_query(Q)
    b, nq, L, d = Q.shape
    SQ = np.empty((b, nq, L))
    for bi in range(b):
        for h in range(nq):
            m = MQ[bi, h]
            m_norm = np.sqrt(np.dot(m, m))
            for t in range(L):
                q = Q[bi, h, t]
                den = max(np.sqrt(np.dot(q, q)) * m_norm, 1e-8)
                SQ[bi, h, t] = -np.dot(q, m) / den
    return SQ


# ---------------------------------------------------------------------------
# Step (b): top-NQ query subselection  [QUOKA §2.1, Algorithm 1]
# ---------------------------------------------------------------------------

def select_queries(SQ, NQ: int) -> np.ndarray:
    """Indices of the NQ largest SQ per (b, h), in rank order (descending SQ,
    ties to the lower position)   -> (b, nq, NQ) int64."""
    SQ = _f64(SQ)
    b, nq, L = SQ.shape
    if not 1 <= NQ <= L:
        raise ValueError("need 1 <= NQ <= BCP")
    out = np.empty((b, nq, NQ), dtype=np.int64)
    pos = np.arange(L)
    for bi in range(b):
        for h in range(nq):
            # primary key -SQ (ascending), secondary key position
            order = np.lexsort((pos, -SQ[bi, h]))
            out[bi, h] = order[:NQ]
    return out


# ---------------------------------------------------------------------------
# Step (c): normalise the chosen queries, mean over each GQA group
# [QUOKA §2.3: each chosen query divided by its L2 norm, then averaged over
#  the query heads of its KV head's group]
# ---------------------------------------------------------------------------

def group_queries(Q, q_idx, nkv: int, normalize: bool = True) -> np.ndarray:
    """Q_group[b, j, i] = (1/G) sum_g Q[b, jG+g, q_idx[b, jG+g, i]] / |.|
       -> (b, nkv, NQ, d). normalize=False: the raw chosen queries are
       averaged (the dot-product variant)."""
    Q = _f64(Q)
    b, nq, L, d = Q.shape
    if nq % nkv:
        raise ValueError("nq must be a multiple of nkv")
    G = nq // nkv
    NQ = q_idx.shape[2]
    out = np.zeros((b, nkv, NQ, d))
    for bi in range(b):
        for j in range(nkv):
            for i in range(NQ):
                acc = np.zeros(d)
                for g in range(G):
                    h = j * G + g
                    q = Q[bi, h, q_idx[bi, h, i]]
                    acc += q / np.sqrt(np.dot(q, q)) if normalize else q
                out[bi, j, i] = acc / G
    return out


# ---------------------------------------------------------------------------
# Step (d): cosine scores, max over the chosen queries
# [QUOKA §2.2 cosine score; §2.3 S = Q_group K_norm^T, S_agg = max over NQ]
# ---------------------------------------------------------------------------

def key_scores(Q_group, K, normalize: bool = True) -> np.ndarray:
    """S_agg[b, j, tau] = max_i Q_group[b, j, i] . K[b, j, tau] / |K[b, j, tau]|
       -> (b, nkv, T). normalize=False: the plain dot product with K (the
       dot-product variant)."""
    Qg = _f64(Q_group)
    b, nkv, T, d = K.shape
    out = np.empty((b, nkv, T))
    for bi in range(b):
        for j in range(nkv):
            Kh = _f64(K[bi, j])           # one head at a time bounds memory
            Kn = Kh / np.linalg.norm(Kh, axis=1, keepdims=True) if normalize else Kh
            S = Qg[bi, j] @ Kn.T          # (NQ, T), the library matmul
            out[bi, j] = S.max(axis=0)
    return out


# ---------------------------------------------------------------------------
# Step (e): top-BSA keys per KV head   [QUOKA §2.3: the BSA keys with the
# highest aggregated score are kept]
# ---------------------------------------------------------------------------

def select_keys(S_agg, BSA: int) -> np.ndarray:
    """The BSA_eff = min(BSA, T) largest scores per (b, j), ties to the lower
    key index, returned as ascending key indices -> (b, nkv, BSA_eff) int64."""
    S = _f64(S_agg)
    b, nkv, T = S.shape
    if BSA < 0:
        raise ValueError("BSA must be >= 0")
    n = min(BSA, T)
    out = np.empty((b, nkv, n), dtype=np.int64)
    pos = np.arange(T)
    for bi in range(b):
        for j in range(nkv):
            order = np.lexsort((pos, -S[bi, j]))
            out[bi, j] = np.sort(order[:n])
    return out


# ---------------------------------------------------------------------------
# Step (f): gather   [QUOKA §4.2 problem 3: the selection becomes the KV input]
# ---------------------------------------------------------------------------

def gather_kv(K, V, sel):
    """Ksel[b, j, n] = K[b, j, sel[b, j, n]] (same for V)."""
    b, nkv = sel.shape[:2]
    Ks = np.stack([np.stack([_f64(K[bi, j][sel[bi, j]]) for j in range(nkv)]) for bi in range(b)])
    Vs = np.stack([np.stack([_f64(V[bi, j][sel[bi, j]]) for j in range(nkv)]) for bi in range(b)])
    return Ks, Vs


# ---------------------------------------------------------------------------
# Step (g): GQA attention over the selected keys plus the chunk's own keys
# [QUOKA §4.2 problem 3: selected KV as attention input, causal mask off for
#  it; the chunk's own keys causally]
# ---------------------------------------------------------------------------

def sparse_attention(Q, K, V, sel, Kc, Vc, scale: Optional[float] = None, include_chunk: bool = True):
    """O[b, h, t] = sum_k softmax_k(scale * Q[b,h,t] . k) v over
    k in {K[b, j, sel[b, j]]} U {Kc[b, j, s] : s <= t}, j = floor(h / G).

    Returns (O (b, nq, BCP, d), LSE (b, nq, BCP)) with
    LSE = log sum_k exp(scale * q . k).

    include_chunk=False leaves the chunk's own keys out (one rank's part
    when the prior keys are split over ranks); a row with no key left gets
    O = 0 and LSE = -inf."""
    Q = _f64(Q)
    Kc = _f64(Kc)
    Vc = _f64(Vc)
    b, nq, L, d = Q.shape
    nkv = Kc.shape[1]
    G = nq // nkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    Ks, Vs = gather_kv(K, V, sel)
    O = np.empty((b, nq, L, d))
    LSE = np.empty((b, nq, L))
    for bi in range(b):
        for h in range(nq):
            j = h // G
            keys = np.concatenate([Ks[bi, j], Kc[bi, j]], axis=0)
            vals = np.concatenate([Vs[bi, j], Vc[bi, j]], axis=0)
            n_sel = Ks.shape[2]
            logits = scale * (Q[bi, h] @ keys.T)             # (L, n_sel + L)
            # chunk key s is visible to query t iff s <= t
            s_idx = np.arange(L)
            hidden = s_idx[None, :] > s_idx[:, None]
            logits[:, n_sel:][hidden] = -np.inf
            if not include_chunk:
                logits[:, n_sel:] = -np.inf
            if logits.shape[1] == 0 or not np.isfinite(logits).any(axis=1).all():
                # rows with no key at all: O = 0, LSE = -inf
                empty = ~np.isfinite(logits).any(axis=1) if logits.shape[1] else np.ones(L, dtype=bool)
                O[bi, h] = 0.0
                LSE[bi, h] = -np.inf
                live = ~empty
                if live.any():
                    lg = logits[live]
                    m = lg.max(axis=1, keepdims=True)
                    p = np.exp(lg - m)
                    denom = p.sum(axis=1, keepdims=True)
                    O[bi, h][live] = (p @ vals) / denom
                    LSE[bi, h][live] = (m + np.log(denom))[:, 0]
                continue
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            denom = p.sum(axis=1, keepdims=True)
            O[bi, h] = (p @ vals) / denom
            LSE[bi, h] = (m + np.log(denom))[:, 0]
    return O, LSE


# ---------------------------------------------------------------------------
# Whole step
# ---------------------------------------------------------------------------

def select(Q, K, NQ: int, BSA: int, *, override_q_idx=None, dot_product: bool = False):
    """Steps (a)-(e). Returns a dict with SQ, q_idx, Q_group, S_agg, sel.

    override_q_idx replaces the top-NQ choice (to check the later steps alone
    on another implementation's choice of queries). dot_product=True scores
    with the plain dot product: no L2 normalisation of the chosen queries in
    step (c) nor of the keys in step (d) ([QUOKA §2.2], the comparison of its
    Table 9); steps (a), (b) and (e) are unchanged."""
    Q = _f64(Q)
    nkv = K.shape[1]
    SQ = query_scores(Q)
    q_idx = select_queries(SQ, NQ) if override_q_idx is None else np.asarray(override_q_idx, dtype=np.int64)
    Qg = group_queries(Q, q_idx, nkv, normalize=not dot_product)
    S_agg = key_scores(Qg, K, normalize=not dot_product)
    sel = select_keys(S_agg, BSA)
    return {"SQ": SQ, "q_idx": q_idx, "Q_group": Qg, "S_agg": S_agg, "sel": sel}


def prefill_chunk(Q, K, V, Kc, Vc, NQ: int, BSA: int, scale: Optional[float] = None,
                  *, override_q_idx=None, override_sel=None):
    """Steps (a)-(g). Returns the select() dict plus O and LSE.

    override_sel replaces the top-BSA choice (to check attention alone on
    another implementation's selected set)."""
    r = select(Q, K, NQ, BSA, override_q_idx=override_q_idx)
    sel = r["sel"] if override_sel is None else np.asarray(override_sel, dtype=np.int64)
    O, LSE = sparse_attention(Q, K, V, sel, Kc, Vc, scale)
    r.update(O=O, LSE=LSE, sel_used=sel)
    return r


def sparse_attention_rows(Q, K, V, sel, Kc, Vc, rows, scale: Optional[float] = None):
    """Step (g) for a list of (b, h, t) rows only, computed one by one:
    returns (O_rows (n, d), LSE_rows (n,)). Same definition as
    sparse_attention; used to check large workloads on a sample of rows."""
    d = Q.shape[-1]
    nq, nkv = Q.shape[1], Kc.shape[1]
    G = nq // nkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((len(rows), d))
    lse = np.empty(len(rows))
    for n, (bi, h, t) in enumerate(rows):
        j = h // G
        idx = np.asarray(sel[bi, j], dtype=np.int64)
        keys = np.concatenate([_f64(K[bi, j][idx]), _f64(Kc[bi, j, :t + 1])], axis=0)
        vals = np.concatenate([_f64(V[bi, j][idx]), _f64(Vc[bi, j, :t + 1])], axis=0)
        logits = scale * (keys @ _f64(Q[bi, h, t]))
        m = logits.max()
        p = np.exp(logits - m)
        out[n] = (p @ vals) / p.sum()
        lse[n] = m + np.log(p.sum())
    return out, lse
