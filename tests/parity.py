"""Parity rules between the CUDA path and the CPU oracle.

  * chosen queries (q_idx): exact, except that entries whose oracle SQ values
    lie within Q_TIE_BAND of each other may swap (fp32 vs fp64 scores);
    when they differ, the oracle is rerun on the CUDA path's choice;
  * aggregated key scores: max-abs S_TOL against the oracle;
  * selected keys: bit-exact, except keys whose oracle score lies within
    KV_TIE_BAND of the BSA-th largest oracle score;
  * attention output: max-abs O_TOL_F32 (fp32 inputs) / O_TOL_BF16 (bf16
    inputs), against the fp64 oracle run on the CUDA path's selected set.
"""
import numpy as np
import torch

from oracle import quoka_oracle as orc

Q_TIE_BAND = 1e-5
KV_TIE_BAND = 1e-3
S_TOL = 2e-5
O_TOL_F32 = 1e-4
O_TOL_BF16 = 2e-2
LSE_TOL = 1e-4


def o_tol(dtype: str) -> float:
    return O_TOL_F32 if dtype == "f32" else O_TOL_BF16


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def to_dev_view(x: np.ndarray, dtype: str, pad: int = 64) -> torch.Tensor:
    """x (b, h, T, d) as the leading T rows of a longer (b, h, T + pad, d)
    device buffer: a strided view (heads T + pad rows apart), as a slice of a
    larger cache would be."""
    b, h, T, d = x.shape
    big = np.zeros((b, h, T + pad, d), dtype=np.float32)
    big[:, :, :T] = x
    return to_dev(big, dtype)[:, :, :T]


def check_q_idx(gpu_q_idx: np.ndarray, SQ: np.ndarray, q_idx: np.ndarray) -> bool:
    """Returns True when identical; False when they differ only inside the
    near-tie band (asserts otherwise)."""
    if np.array_equal(gpu_q_idx, q_idx):
        return True
    b, nq, NQ = q_idx.shape
    for bi in range(b):
        for h in range(nq):
            g, o = gpu_q_idx[bi, h], q_idx[bi, h]
            if np.array_equal(g, o):
                continue
            assert len(set(g.tolist())) == NQ, "duplicate chosen query"
            s = SQ[bi, h]
            diff = np.abs(s[g] - s[o])
            assert diff.max() <= Q_TIE_BAND, (
                f"q_idx differs beyond the near-tie band at b={bi} h={h}: "
                f"max |dSQ| = {diff.max():.3e}")
    return False


def check_kv_sets(gpu_idx: np.ndarray, gpu_count: np.ndarray, S_agg: np.ndarray, bsa_eff: int,
                  sel: np.ndarray, band: float = None) -> int:
    """Checks the CUDA path's selected sets against the oracle's; returns the
    number of (b, j) rows that differ inside the tie band (KV_TIE_BAND, or
    `band` for scores that are not cosines)."""
    band = KV_TIE_BAND if band is None else band
    b, nkv, T = S_agg.shape
    assert np.all(gpu_count == bsa_eff), f"counts {np.unique(gpu_count)} != {bsa_eff}"
    n_diff = 0
    for bi in range(b):
        for j in range(nkv):
            g = gpu_idx[bi, j]
            assert np.all(np.diff(g) > 0), "indices not strictly ascending"
            assert g.min(initial=0) >= 0 and g.max(initial=-1) < T
            if np.array_equal(g, sel[bi, j]):
                continue
            n_diff += 1
            s = S_agg[bi, j]
            thr = np.sort(s)[::-1][bsa_eff - 1]
            sym = np.setxor1d(g, sel[bi, j])
            dev = np.abs(s[sym] - thr)
            assert dev.max() <= band, (
                f"selected keys differ beyond the tie band at b={bi} j={j}: "
                f"{len(sym)} keys, max |S - thr| = {dev.max():.3e}")
    return n_diff


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float -> bfloat16 (round to nearest even) -> float32, on the host."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()
