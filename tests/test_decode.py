"""The attention for short chunks (decode steps and short speculative
blocks, G * BCP <= 64 query rows per KV head): quoka_decode_attn against the
oracle on given selections, its edge cases, and its host-side validation.
quoka_prefill_chunk routes such chunks to it; those runs are checked in
test_gpu_parity.py (the BCP = 1 and short-chunk rows of SMALL) and in
test_decode_step_through_prefill_chunk below."""
import numpy as np
import pytest
import torch

from oracle import quoka_oracle as orc
from sparse_kv_selection_quoka_b200 import inputs
from tests import parity as P


def q():
    import sparse_kv_selection_quoka_b200 as m
    return m


def oracle_attention(x, sel, counts):
    """fp64 attention of every query row over its KV head's first counts[b, j]
    selected keys plus the chunk's keys (causal)."""
    b, nq, L, d = x.Q.shape
    nkv = x.K.shape[1]
    G = nq // nkv
    O = np.zeros((b, nq, L, d))
    lse = np.zeros((b, nq, L))
    for bi in range(b):
        for j in range(nkv):
            n = int(counts[bi, j])
            hs = slice(j * G, (j + 1) * G)
            s = sel[bi, j, :n].astype(np.int64)[None, None]
            o, l = orc.sparse_attention(x.Q[bi:bi + 1, hs], x.K[bi:bi + 1, j:j + 1], x.V[bi:bi + 1, j:j + 1], s,
                                        x.Kc[bi:bi + 1, j:j + 1], x.Vc[bi:bi + 1, j:j + 1])
            O[bi, hs] = o[0]
            lse[bi, hs] = l[0]
    return O, lse


CASES = [
    # b, nq, nkv, d, T, BCP, BSA, dtype, counts ("full" or a list per (b, j)), strided views
    (1, 32, 8, 128, 8192, 1, 2048, "bf16", "full", False),         # a decode step, Qwen-shaped heads
    (2, 16, 2, 128, 3000, 8, 700, "bf16", [[700, 333], [1, 0]], True),  # G * BCP = 64 rows, partial counts
    (1, 6, 3, 64, 900, 3, 200, "f32", [[200, 0, 17]], False),      # fp32, d = 64, a head with chunk keys only
    (1, 4, 4, 128, 129, 2, 128, "bf16", "full", False),            # G = 1, BSA_eff = T
    (1, 8, 2, 128, 0, 1, 0, "bf16", "full", False),                # T = 0: the chunk's own key only
    (2, 12, 2, 64, 1500, 5, 400, "bf16", [[400, 3], [0, 399]], True),  # d = 64, 30 rows (two 16-row tiles)
]


@pytest.mark.gpu
@pytest.mark.parametrize("k", range(len(CASES)),
                         ids=[f"b{c[0]}_nq{c[1]}_nkv{c[2]}_d{c[3]}_T{c[4]}_L{c[5]}_BSA{c[6]}_{c[7]}" for c in CASES])
def test_decode_attention_on_given_selection(k):
    b, nq, nkv, d, T, BCP, BSA, dt, counts, strided = CASES[k]
    x = inputs.make_chunk(b, nq, nkv, d, T, BCP, 1, BSA, dtype=dt, structure="llama" if T >= 64 else "iid",
                          seed=300 + k)
    rng = np.random.default_rng(300 + k)
    bsa = min(BSA, T)
    sel = np.stack([[np.sort(rng.choice(T, bsa, replace=False)) if bsa else np.zeros(0, np.int64)
                     for _ in range(nkv)] for _ in range(b)]).reshape(b, nkv, bsa)
    cnt = np.full((b, nkv), bsa, dtype=np.int32) if counts == "full" else np.array(counts, dtype=np.int32)
    idx = sel.copy()
    for bi in range(b):
        for j in range(nkv):
            idx[bi, j, cnt[bi, j]:] = 10 ** 6  # past the count: never read
    if strided:
        Q = P.to_dev_view(x.Q, dt)
        K, V = P.to_dev_view(x.K, dt), P.to_dev_view(x.V, dt)
    else:
        Q, K, V = (P.to_dev(a, dt) for a in (x.Q, x.K, x.V))
    Kc, Vc = P.to_dev(x.Kc, dt), P.to_dev(x.Vc, dt)
    n = q().quoka_decode_workspace_size(b, nq, nkv, d, BCP, bsa, torch.bfloat16 if dt == "bf16" else torch.float32)
    assert n > 0
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")  # garbage partials must not matter
    O, lse = q().quoka_decode_attn(Q, K, V, torch.from_numpy(idx.astype(np.int32)).cuda(),
                                   torch.from_numpy(cnt).cuda(), Kc, Vc, want_lse=True, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    O_ref, L_ref = oracle_attention(x, sel, cnt)
    err = np.abs(O.float().cpu().numpy() - O_ref).max()
    lerr = np.abs(lse.cpu().numpy() - L_ref).max()
    tol = P.o_tol(dt)
    assert err <= tol, f"O max-abs error {err:.3e}"
    assert lerr <= max(P.LSE_TOL, tol), f"lse max-abs error {lerr:.3e}"


@pytest.mark.gpu
def test_decode_out_of_range_index_is_latched_not_read():
    x = inputs.make_chunk(1, 4, 1, 128, 300, 1, 1, 10, dtype="bf16", structure="iid", seed=19)
    Q, K, V, Kc, Vc = (P.to_dev(a, "bf16") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    idx = torch.tensor([[[1, 5, 99, 300, 2000]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[5]], dtype=torch.int32, device="cuda")
    ws = torch.zeros(q().quoka_decode_workspace_size(1, 4, 1, 128, 1, 5, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    O, _ = q().quoka_decode_attn(Q, K, V, idx, cnt, Kc, Vc, ws=ws)
    assert q().quoka_get_device_status(ws) == 6
    assert torch.isfinite(O.float()).all()
    # the next valid call on the same workspace clears the status first
    good = torch.tensor([[[1, 5, 99, 250, 299]]], dtype=torch.int32, device="cuda")
    q().quoka_decode_attn(Q, K, V, good, cnt, Kc, Vc, ws=ws)
    assert q().quoka_get_device_status(ws) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("BCP", [1, 4])
def test_decode_step_through_prefill_chunk(BCP):
    """The whole step on a Qwen-shaped decode (or 4-token speculative) chunk:
    selection vs the oracle (bit-exact up to the tie band) and the output vs
    the oracle on the selected set, through quoka_prefill_chunk."""
    x = inputs.make_chunk(1, 32, 8, 128, 16384, BCP, BCP, 2048, dtype="bf16", structure="qwen", seed=310 + BCP)
    from tests.test_gpu_parity import run_prefill_and_check, run_select_and_check
    ref, gi, _ = run_select_and_check(x)
    run_prefill_and_check(x, ref, gi)


ONE_TOKEN = [
    # b, nq, nkv, T, BSA, strided Q, dot-product score
    (2, 48, 3, 5000, 900, True, False),   # G = 16 query heads per KV head
    (1, 32, 1, 3000, 3000, False, False),  # G = 32, BSA_eff = T
    (1, 8, 8, 1000, 100, False, True),     # G = 1, the dot-product score
]


@pytest.mark.gpu
@pytest.mark.parametrize("k", range(len(ONE_TOKEN)), ids=[f"b{c[0]}_nq{c[1]}_nkv{c[2]}_T{c[3]}" for c in ONE_TOKEN])
def test_one_token_selection(k):
    """A one-query chunk: every head keeps its only query (q_idx = 0, the one
    candidate of Algorithm 1), and S_agg / the selected keys follow from the
    group mean of the G normalised (or raw) queries. Against the oracle."""
    b, nq, nkv, T, BSA, strided, dot = ONE_TOKEN[k]
    x = inputs.make_chunk(b, nq, nkv, 128, T, 1, 1, BSA, dtype="bf16", structure="llama", seed=330 + k)
    Q = P.to_dev_view(x.Q, "bf16") if strided else P.to_dev(x.Q, "bf16")
    K = P.to_dev(x.K, "bf16")
    kv_idx, kv_count, q_idx, s_agg = q().quoka_select(Q, K, 1, BSA, want_q_idx=True, want_s_agg=True,
                                                      dot_product=dot)
    torch.cuda.synchronize()
    assert torch.equal(q_idx.cpu(), torch.zeros((b, nq, 1), dtype=torch.int32))
    ref = orc.select(x.Q, x.K, 1, BSA, dot_product=dot)
    assert np.array_equal(ref["q_idx"], np.zeros((b, nq, 1)))
    scale = max(1.0, float(np.abs(ref["S_agg"]).max())) if dot else 1.0
    err = np.abs(s_agg.cpu().numpy().astype(np.float64) - ref["S_agg"]).max()
    assert err <= P.S_TOL * scale, f"S_agg max-abs error {err:.3e}"
    P.check_kv_sets(kv_idx.cpu().numpy().astype(np.int64), kv_count.cpu().numpy(), ref["S_agg"], min(BSA, T),
                    ref["sel"], band=P.KV_TIE_BAND * scale)


# ---------------------------------------------------------------- host side

def test_decode_workspace_size_counts_the_slices():
    """Partials: ceil((BSA_eff + BCP) / 64) slices of b * nq * BCP rows, d + 1
    floats each (the outputs and the log-sum-exps), after the 256-byte status
    block, each region 256-byte aligned."""
    m = q()
    al = lambda n: (n + 255) // 256 * 256
    for b, nq, nkv, d, BCP, bsa in [(1, 32, 8, 128, 1, 4096), (2, 16, 2, 64, 8, 700), (1, 4, 4, 128, 3, 0)]:
        ns = (bsa + BCP + 63) // 64
        rows = ns * b * nq * BCP
        want = 256 + al(rows * d * 4) + al(rows * 4)
        assert m.quoka_decode_workspace_size(b, nq, nkv, d, BCP, bsa, torch.bfloat16) == want
