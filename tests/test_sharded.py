"""The prefill-chunk step with the prior keys split over ranks.

CPU (gloo, world sizes 2 and 3): sparse_kv_selection_quoka_b200.sharded
runs its exchanges through torch.distributed with the per-rank calls done by
OracleOps below (test infrastructure: the fp64 oracle in numpy), and the
result must equal the one-device oracle: the same selected key set and the
same output.

GPU: the library's per-rank calls for several shards in turn in one process
(the exchange is a concatenation, so no kernel waits on another), against
the one-device library selection (bit-exact key sets) and the oracle's
output.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import quoka_oracle as orc
from sparse_kv_selection_quoka_b200 import inputs, sharded
from tests import parity as P


class OracleOps:
    """The per-rank calls of sharded.py on CPU tensors, from the oracle
    (float64 numpy); same shapes, padding and tie rules as the library."""

    def select(self, Q, K, NQ, BSA, dot_product=False):
        r = orc.select(Q.numpy(), K.numpy(), NQ, BSA, dot_product=dot_product)
        sel = torch.from_numpy(r["sel"].astype(np.int32))
        cnt = torch.full(sel.shape[:2], sel.shape[2], dtype=torch.int32)
        return sel, cnt, torch.from_numpy(r["S_agg"])

    def candidates(self, s_agg, kv_idx, kv_count, C):
        b, nkv, _ = s_agg.shape
        scores = torch.full((b, nkv, C), -np.inf, dtype=s_agg.dtype)
        cand = torch.full((b, nkv, C), -1, dtype=torch.int32)
        for bi in range(b):
            for j in range(nkv):
                n = int(kv_count[bi, j])
                cand[bi, j, :n] = kv_idx[bi, j, :n]
                scores[bi, j, :n] = s_agg[bi, j, kv_idx[bi, j, :n].long()]
        return scores, cand

    def interleave(self, gathered):
        N, b, nkv, C = gathered.shape
        return gathered.permute(1, 2, 0, 3).reshape(b, nkv, N * C)

    def topk(self, scores, BSA):
        sel = orc.select_keys(scores.numpy(), BSA).astype(np.int32)
        return torch.from_numpy(sel), torch.full(sel.shape[:2], sel.shape[2], dtype=torch.int32)

    def take(self, sel_pos, sel_count, cand_idx, rank):
        b, nkv, C = cand_idx.shape
        idx = torch.zeros((b, nkv, C), dtype=torch.int32)
        cnt = torch.zeros((b, nkv), dtype=torch.int32)
        for bi in range(b):
            for j in range(nkv):
                p = sel_pos[bi, j, :int(sel_count[bi, j])].long()
                mine = p[(p >= rank * C) & (p < (rank + 1) * C)] - rank * C
                keys = cand_idx[bi, j, mine]
                assert torch.all(keys >= 0), "a padding candidate was selected"
                idx[bi, j, :len(keys)] = keys
                cnt[bi, j] = len(keys)
        return idx, cnt

    def attention(self, Q, K, V, kv_idx, kv_count, Kc, Vc, scale, with_chunk):
        b, nq, L, d = Q.shape
        nkv = K.shape[1]
        G = nq // nkv
        O = np.zeros((b, nq, L, d))
        lse = np.zeros((b, nq, L))
        for bi in range(b):
            for j in range(nkv):
                n = int(kv_count[bi, j])
                sel = kv_idx[bi, j, :n].numpy().astype(np.int64)[None, None]
                hs = slice(j * G, (j + 1) * G)
                o, l = orc.sparse_attention(Q[bi:bi + 1, hs].numpy(), K[bi:bi + 1, j:j + 1].numpy(),
                                            V[bi:bi + 1, j:j + 1].numpy(), sel, Kc[bi:bi + 1, j:j + 1].numpy(),
                                            Vc[bi:bi + 1, j:j + 1].numpy(), scale, include_chunk=with_chunk)
                O[bi, hs] = o[0]
                lse[bi, hs] = l[0]
        return torch.from_numpy(O), torch.from_numpy(lse)

    def combine(self, O_parts, lse_parts):
        ls = lse_parts.numpy()
        lse = np.logaddexp.reduce(ls, axis=0)
        with np.errstate(invalid="ignore"):
            w = np.where(np.isneginf(ls), 0.0, np.exp(ls - lse))
        O = (w[..., None] * O_parts.numpy()).sum(axis=0)
        return torch.from_numpy(O), torch.from_numpy(lse)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(T_shards, seed, BCP=24):
    T = sum(T_shards)
    NQ = min(5, BCP)
    x = inputs.make_chunk(1, 4, 2, 32, T, BCP, NQ, 20, dtype="f32", structure="llama", seed=seed)
    return x


def _gloo_rank(rank, world, port, T_shards, seed, out_dir, BCP=24):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        x = _case(T_shards, seed, BCP)
        offs = np.cumsum([0] + list(T_shards))
        sl = slice(offs[rank], offs[rank + 1])
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
        O, lse, kv_idx, kv_count = sharded.prefill_chunk_sharded(
            t(x.Q), t(x.K[:, :, sl]), t(x.V[:, :, sl]), t(x.Kc), t(x.Vc), x.NQ, x.BSA, T_shards,
            ops=OracleOps())
        # this rank's share, as global key indices
        b, nkv = kv_count.shape
        shares = {f"share_{bi}_{j}": kv_idx[bi, j, :int(kv_count[bi, j])].numpy().astype(np.int64) + offs[rank]
                  for bi in range(b) for j in range(nkv)}
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), O=O.numpy(), lse=lse.numpy(), **shares)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T_shards,BCP", [((90, 60), 24), ((50, 0, 77), 24), ((70, 45), 1)],
                         ids=["two_ranks", "three_ranks_one_empty", "two_ranks_decode_step"])
def test_sharded_exchange_gloo(T_shards, BCP, tmp_path):
    world = len(T_shards)
    port = _free_port()
    mp.start_processes(_gloo_rank, args=(world, port, T_shards, 81, str(tmp_path), BCP), nprocs=world, join=True,
                       start_method="spawn")
    x = _case(T_shards, 81, BCP)
    ref = orc.prefill_chunk(x.Q, x.K, x.V, x.Kc, x.Vc, x.NQ, x.BSA)
    sel = [[set() for _ in range(x.K.shape[1])] for _ in range(x.K.shape[0])]
    for r in range(world):
        z = np.load(tmp_path / f"rank{r}.npz")
        # every rank ends with the whole merged output
        np.testing.assert_allclose(z["O"], ref["O"], atol=1e-10)
        np.testing.assert_allclose(z["lse"], ref["LSE"], atol=1e-10)
        for bi in range(len(sel)):
            for j in range(len(sel[bi])):
                sel[bi][j] |= set(z[f"share_{bi}_{j}"].tolist())
    for bi in range(len(sel)):
        for j in range(len(sel[bi])):
            assert sorted(sel[bi][j]) == ref["sel"][bi, j].tolist()


@pytest.mark.gpu
@pytest.mark.parametrize("T_shards,dt", [((1500, 900, 600), "bf16"), ((2000, 0, 1000), "bf16"),
                                         ((300, 200), "f32")],
                         ids=["bf16_three", "bf16_empty_shard", "f32_two"])
def test_sharded_library_matches_one_device(T_shards, dt):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_selection_quoka_b200 as q
    T = sum(T_shards)
    d = 128 if dt == "bf16" else 64
    x = inputs.make_chunk(1, 8, 2, d, T, 200 if dt == "bf16" else 40, 8 if dt == "bf16" else 4,
                          600 if dt == "bf16" else 100, dtype=dt, structure="llama", seed=83)
    dev = [P.to_dev(a, dt) for a in (x.Q, x.K, x.V, x.Kc, x.Vc)]
    Q, K, V, Kc, Vc = dev
    plan = sharded.ShardPlan(tuple(T_shards), x.BSA)
    offs = np.cumsum([0] + list(T_shards))
    shards = [(K[:, :, offs[r]:offs[r + 1]], V[:, :, offs[r]:offs[r + 1]]) for r in range(plan.N)]
    cands = [sharded.local_candidates(plan, Q, Ks, x.NQ) for Ks, _ in shards]
    all_scores = torch.stack([c[0] for c in cands])            # the exchange, in one process
    shares = [sharded.select_share(plan, all_scores, cands[r][1], r) for r in range(plan.N)]
    parts = [sharded.partial_attention(plan, r, Q, shards[r][0], shards[r][1], Kc, Vc, *shares[r])
             for r in range(plan.N)]
    O, lse = sharded.combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    torch.cuda.synchronize()
    # the merged selection is the one-device selection, key for key
    one_idx, one_cnt, _, _ = q.quoka_select(Q, K, x.NQ, x.BSA)
    for j in range(K.shape[1]):
        merged = np.sort(np.concatenate([shares[r][0][0, j, :int(shares[r][1][0, j])].cpu().numpy() + offs[r]
                                         for r in range(plan.N)]))
        np.testing.assert_array_equal(merged, one_idx[0, j, :int(one_cnt[0, j])].cpu().numpy())
    ref_O, ref_L = orc.sparse_attention(x.Q, x.K, x.V, one_idx.cpu().numpy().astype(np.int64), x.Kc, x.Vc)
    err = np.abs(O.float().cpu().numpy().astype(np.float64) - ref_O).max()
    lerr = np.abs(lse.cpu().numpy().astype(np.float64) - ref_L).max()
    assert err <= P.o_tol(dt), f"O max-abs error {err:.3e}"
    assert lerr <= max(P.LSE_TOL, P.o_tol(dt)), f"lse max-abs error {lerr:.3e}"
