"""Seeded synthetic inputs for the QUOKA prefill-chunk step.

This module only draws random tensors and plants structure in them. It holds
none of the method's arithmetic (no means, cosines, selections or softmax), so
both the CUDA path and the CPU oracle may take their inputs from here.

Every tensor is drawn in float32 from numpy's PCG64 with a fixed seed and a
fixed draw order (noise for Q, K, V, Kc, Vc first, then the planted
structure), and is rounded once to bfloat16 (round-to-nearest-even) for the
bf16 workloads. The shapes are those of the Llama3-3B / Qwen3-4B layers the
QUOKA write-up evaluates on; its evaluation runs on real model activations,
which are not available here, so the value structure is a synthetic stand-in
defined with these workloads: queries share a per-group mean direction, a
fraction of them are outliers with no mean component, and a set of "heavy"
keys is aligned with the outlier directions.

Layouts (row-major, contiguous):
  Q  (b, nq,  BCP, d)   the chunk's queries
  K  (b, nkv, T,   d)   the T prior keys of the cache
  V  (b, nkv, T,   d)
  Kc (b, nkv, BCP, d)   the chunk's own keys
  Vc (b, nkv, BCP, d)
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "ChunkInputs",
    "make_chunk",
    "make_workload",
    "SweepInputs",
    "make_sweep",
    "to_torch",
]


@dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic workload."""

    name: str
    b: int
    nq: int
    nkv: int
    d: int
    T: int
    BCP: int
    NQ: int
    BSA: int
    dtype: str  # "f32" or "bf16"
    structure: str  # "planted_tiny", "llama", "qwen", "long"
    seed: int


# The five workloads. Index order matches the order the workloads are listed
# in the configuration file that defines them (0 tiny, 1 Llama-shaped,
# 2 Qwen-shaped, 3 chunked sweep, 4 long context).
WORKLOADS = [
    Workload("tiny_fp32", 1, 4, 2, 64, 1024, 128, 8, 256, "f32", "planted_tiny", 1000),
    Workload("llama3.2-3b_T8k", 1, 24, 8, 128, 8192, 256, 16, 2048, "bf16", "llama", 1001),
    Workload("qwen3-4b_T32k", 1, 32, 8, 128, 32768, 512, 32, 4096, "bf16", "qwen", 1002),
    # the sweep: T is per chunk (256*c), listed here with the total length
    Workload("sweep_b8_S16k", 8, 32, 8, 128, 16384, 256, 16, 0, "bf16", "llama", 1003),
    Workload("long_T128k_G8", 1, 64, 8, 128, 131072, 512, 32, 16384, "bf16", "long", 1004),
]


@dataclass
class ChunkInputs:
    """One chunk's inputs as numpy float32 arrays (already bf16-representable
    when dtype == "bf16")."""

    Q: np.ndarray
    K: np.ndarray
    V: np.ndarray
    Kc: np.ndarray
    Vc: np.ndarray
    NQ: int
    BSA: int
    dtype: str
    meta: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.Q.shape[-1]))


def _round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 -> bfloat16 -> float32 (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _unit_rows(rng: np.random.Generator, n: int, d: int) -> np.ndarray:
    v = rng.standard_normal((n, d), dtype=np.float32).astype(np.float64)
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    return v.astype(np.float32)


def _plant_queries(rng, Q, nkv, G, kind, n_outlier, W):
    """Add a per-group mean direction to every query and replace a seeded
    subset of chunk positions (shared by the G heads of a group) by outliers
    along the group's outlier directions W[j] (C, d)."""
    b, nq, L, d = Q.shape
    mu = 4.0 * _unit_rows(rng, b * nkv, d).reshape(b, nkv, d)
    out_pos = np.zeros((b, nkv, n_outlier), dtype=np.int64)
    for bi in range(b):
        for j in range(nkv):
            pos = np.sort(rng.choice(L, size=n_outlier, replace=False))
            out_pos[bi, j] = pos
            is_out = np.zeros(L, dtype=bool)
            is_out[pos] = True
            C = W.shape[2]
            for g in range(G):
                h = j * G + g
                Q[bi, h, ~is_out] += mu[bi, j]
                for n, t in enumerate(pos):
                    Q[bi, h, t] += 4.0 * W[bi, j, n % C]
    return mu, out_pos


def _plant_keys(rng, K, W, n_heavy, contiguous):
    """Add 8x an outlier direction to n_heavy keys per (batch, KV head):
    either one contiguous run at a seeded offset or seeded random positions.
    Directions cycle over the C outlier directions of that KV head."""
    b, nkv, T, d = K.shape
    n_heavy = min(n_heavy, T)
    pos_all = np.zeros((b, nkv, n_heavy), dtype=np.int64)
    C = W.shape[2]
    for bi in range(b):
        for j in range(nkv):
            if contiguous:
                start = int(rng.integers(0, T - n_heavy + 1))
                pos = np.arange(start, start + n_heavy)
            else:
                pos = np.sort(rng.choice(T, size=n_heavy, replace=False))
            pos_all[bi, j] = pos
            for n, t in enumerate(pos):
                K[bi, j, t] += 8.0 * W[bi, j, n % C]
    return pos_all


def make_chunk(
    b: int,
    nq: int,
    nkv: int,
    d: int,
    T: int,
    BCP: int,
    NQ: int,
    BSA: int,
    *,
    dtype: str = "bf16",
    structure: str = "llama",
    seed: int = 0,
) -> ChunkInputs:
    """Draw one chunk's inputs.

    structure:
      "iid"          Q, K, V, Kc, Vc all i.i.d. N(0, 1).
      "planted_tiny" i.i.d. N(0,1), plus per KV head j a unit direction u_j:
                     16 prior keys set to exactly 3*u_j, and at 8 chunk
                     positions every query head of group j set to
                     3*u_j + 0.1*noise.
      "llama"        per-group mean direction mu_j (norm 4) + N(0,1) noise;
                     10% of chunk positions are outliers 4*w_{j,c} + noise
                     (C = 4 directions per KV head); 64 heavy keys per KV head
                     in one contiguous run get N(0,1) + 8*w_{j,c}.
      "qwen"         as "llama" with 256 heavy keys at random positions.
      "long"         as "llama" with 12.5% outliers and C = 32 clusters;
                     1024 heavy keys per KV head (32 per cluster) at random
                     positions.
    Heavy-key counts are capped at T.
    """
    assert nq % nkv == 0
    G = nq // nkv
    rng = np.random.Generator(np.random.PCG64(seed))
    Q = rng.standard_normal((b, nq, BCP, d), dtype=np.float32)
    K = rng.standard_normal((b, nkv, T, d), dtype=np.float32)
    V = rng.standard_normal((b, nkv, T, d), dtype=np.float32)
    Kc = rng.standard_normal((b, nkv, BCP, d), dtype=np.float32)
    Vc = rng.standard_normal((b, nkv, BCP, d), dtype=np.float32)
    meta: dict = {"structure": structure, "seed": seed}

    if structure == "iid":
        pass
    elif structure == "planted_tiny":
        u = _unit_rows(rng, b * nkv, d).reshape(b, nkv, d)
        heavy = np.zeros((b, nkv, min(16, T)), dtype=np.int64)
        qpos = np.zeros((b, nkv, min(8, BCP)), dtype=np.int64)
        for bi in range(b):
            for j in range(nkv):
                hp = np.sort(rng.choice(T, size=heavy.shape[2], replace=False)) if T else heavy[bi, j]
                heavy[bi, j] = hp
                K[bi, j, hp] = 3.0 * u[bi, j]
                qp = np.sort(rng.choice(BCP, size=qpos.shape[2], replace=False))
                qpos[bi, j] = qp
                for g in range(G):
                    h = j * G + g
                    Q[bi, h, qp] = 3.0 * u[bi, j] + 0.1 * Q[bi, h, qp]
        meta.update(heavy_pos=heavy, planted_q_pos=qpos, u=u)
    elif structure in ("llama", "qwen", "long"):
        C = 32 if structure == "long" else 4
        frac = 0.125 if structure == "long" else 0.10
        n_out = max(1, int(round(frac * BCP)))
        n_heavy = {"llama": 64, "qwen": 256, "long": 1024}[structure]
        W = _unit_rows(rng, b * nkv * C, d).reshape(b, nkv, C, d)
        mu, out_pos = _plant_queries(rng, Q, nkv, G, structure, n_out, W)
        heavy = _plant_keys(rng, K, W, n_heavy, contiguous=(structure == "llama"))
        meta.update(mu=mu, outlier_pos=out_pos, heavy_pos=heavy, W=W)
    else:
        raise ValueError(f"unknown structure {structure!r}")

    if dtype == "bf16":
        Q, K, V, Kc, Vc = (_round_bf16(x) for x in (Q, K, V, Kc, Vc))
    elif dtype != "f32":
        raise ValueError(dtype)
    return ChunkInputs(Q, K, V, Kc, Vc, NQ, BSA, dtype, meta)


def make_workload(index_or_name) -> ChunkInputs:
    """Inputs of one of the single-chunk workloads (0, 1, 2, 4)."""
    w = _lookup(index_or_name)
    if w.name.startswith("sweep"):
        raise ValueError("the sweep workload is made by make_sweep()")
    return make_chunk(w.b, w.nq, w.nkv, w.d, w.T, w.BCP, w.NQ, w.BSA,
                      dtype=w.dtype, structure=w.structure, seed=w.seed)


def _lookup(index_or_name) -> Workload:
    if isinstance(index_or_name, int):
        return WORKLOADS[index_or_name]
    for w in WORKLOADS:
        if w.name == index_or_name:
            return w
    raise KeyError(index_or_name)


@dataclass
class SweepInputs:
    """A whole sequence processed as consecutive chunks of BCP tokens.

    Qs (b, nq, S, d), Ks/Vs (b, nkv, S, d). Chunk c covers positions
    [c*BCP, (c+1)*BCP); its prior keys are Ks[:, :, :c*BCP]."""

    Qs: np.ndarray
    Ks: np.ndarray
    Vs: np.ndarray
    BCP: int
    NQ: int
    dtype: str

    @property
    def n_chunks(self) -> int:
        return self.Qs.shape[2] // self.BCP

    @staticmethod
    def budget(T: int) -> int:
        """Key budget of a chunk with T prior keys: 25% of T, at least 256,
        never more than T."""
        return min(T, max(256, T // 4))

    def chunk(self, c: int) -> ChunkInputs:
        L = self.BCP
        T = c * L
        return ChunkInputs(
            self.Qs[:, :, T:T + L], self.Ks[:, :, :T], self.Vs[:, :, :T],
            self.Ks[:, :, T:T + L], self.Vs[:, :, T:T + L],
            self.NQ, self.budget(T), self.dtype, {"chunk": c})


def make_sweep(b=8, nq=32, nkv=8, d=128, S=16384, BCP=256, NQ=16, *,
               dtype="bf16", seed=1003, n_heavy=128) -> SweepInputs:
    """Inputs of the chunked-prefill sweep: the "llama" value recipe over a
    whole sequence of S positions (queries for every position, outliers at
    10% of positions, n_heavy heavy keys per KV head at random positions)."""
    G = nq // nkv
    rng = np.random.Generator(np.random.PCG64(seed))
    Qs = rng.standard_normal((b, nq, S, d), dtype=np.float32)
    Ks = rng.standard_normal((b, nkv, S, d), dtype=np.float32)
    Vs = rng.standard_normal((b, nkv, S, d), dtype=np.float32)
    W = _unit_rows(rng, b * nkv * 4, d).reshape(b, nkv, 4, d)
    _plant_queries(rng, Qs, nkv, G, "llama", max(1, int(round(0.1 * S))), W)
    _plant_keys(rng, Ks, W, n_heavy, contiguous=False)
    if dtype == "bf16":
        Qs, Ks, Vs = (_round_bf16(x) for x in (Qs, Ks, Vs))
    return SweepInputs(Qs, Ks, Vs, BCP, NQ, dtype)


def to_torch(x: np.ndarray, dtype: str, device="cpu") -> torch.Tensor:
    """numpy float32 -> torch tensor of the workload dtype (exact for values
    that are already bf16-representable)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.to(device)
