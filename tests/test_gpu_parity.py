"""CUDA path vs the CPU oracle, element by element, on seeded inputs.

Every call goes through the C ABI of libquoka.so (via the ctypes binding).
Small shapes span several tiles and ragged tails and cover the degenerate
cases (T = 0, BSA = 0, BSA >= T, NQ = 1, NQ = BCP, G = 1, d = 64, batch > 1);
the full-size workloads are checked in the launch configuration the
benchmark times, on every output the oracle can afford and on sampled rows
otherwise.
"""
import numpy as np
import pytest
import torch

from oracle import quoka_oracle as orc
from sparse_kv_selection_quoka_b200 import inputs
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_selection_quoka_b200 as q
    q.load()
    return q


def q():
    import sparse_kv_selection_quoka_b200 as m
    return m


def run_select_and_check(x: inputs.ChunkInputs, dev=None):
    """quoka_select vs the oracle; returns (oracle result on the GPU's query
    choice, GPU kv_idx, GPU kv_count). `dev` optionally supplies the device
    tensors (Q, K, V, Kc, Vc), e.g. strided views into one cache."""
    dt = x.dtype
    Q, K = (P.to_dev(x.Q, dt), P.to_dev(x.K, dt)) if dev is None else (dev[0], dev[1])
    kv_idx, kv_count, q_idx, s_agg = q().quoka_select(Q, K, x.NQ, x.BSA, want_q_idx=True,
                                                      want_s_agg=True)
    ws = q().workspace_for(Q, K, x.NQ, x.BSA)
    q().quoka_select(Q, K, x.NQ, x.BSA, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    torch.cuda.synchronize()
    ref = orc.select(x.Q, x.K, x.NQ, x.BSA)
    gq = q_idx.cpu().numpy().astype(np.int64)
    if not P.check_q_idx(gq, ref["SQ"], ref["q_idx"]):
        ref = orc.select(x.Q, x.K, x.NQ, x.BSA, override_q_idx=gq)
    T = x.K.shape[2]
    if T > 0:
        sg = s_agg.cpu().numpy().astype(np.float64)
        dif = np.abs(sg - ref["S_agg"])
        err = dif.max()
        at = np.unravel_index(int(dif.argmax()), dif.shape)
        assert err <= P.S_TOL, (f"S_agg max-abs error {err:.3e} at {tuple(int(v) for v in at)}: got "
                                f"{sg[at]:.6f}, want {ref['S_agg'][at]:.6f}; {int((dif > P.S_TOL).sum())} "
                                f"entries out of tolerance")
    bsa_eff = min(x.BSA, T)
    gi = kv_idx.cpu().numpy().astype(np.int64)
    gc = kv_count.cpu().numpy()
    assert gi.shape == (x.K.shape[0], x.K.shape[1], bsa_eff)
    P.check_kv_sets(gi, gc, ref["S_agg"], bsa_eff, ref["sel"])
    return ref, gi, gc


def run_prefill_and_check(x: inputs.ChunkInputs, ref, gi, rows=None, dev=None):
    dt = x.dtype
    if dev is None:
        dev = [P.to_dev(a, dt) for a in (x.Q, x.K, x.V, x.Kc, x.Vc)]
    Q, K, V, Kc, Vc = dev
    O, lse, kv_idx = q().quoka_prefill_chunk(Q, K, V, Kc, Vc, x.NQ, x.BSA, want_lse=True,
                                             want_kv_idx=True)
    torch.cuda.synchronize()
    # the whole step selects the same set as quoka_select (deterministic)
    np.testing.assert_array_equal(kv_idx.cpu().numpy(), gi)
    Og = O.float().cpu().numpy().astype(np.float64)
    Lg = lse.cpu().numpy().astype(np.float64)
    tol = P.o_tol(dt)
    if rows is None:
        O_ref, L_ref = orc.sparse_attention(x.Q, x.K, x.V, gi, x.Kc, x.Vc)
        err = np.abs(Og - O_ref).max()
        lerr = np.abs(Lg - L_ref).max()
    else:
        O_ref, L_ref = orc.sparse_attention_rows(x.Q, x.K, x.V, gi, x.Kc, x.Vc, rows)
        Os = np.stack([Og[r] for r in rows])
        Ls = np.array([Lg[r] for r in rows])
        err = np.abs(Os - O_ref).max()
        lerr = np.abs(Ls - L_ref).max()
    assert err <= tol, f"O max-abs error {err:.3e} > {tol}"
    assert lerr <= max(P.LSE_TOL, tol), f"LSE max-abs error {lerr:.3e}"
    # quoka_prefill_chunk takes the decode attention for short chunks: the
    # prefill attention kernels must agree on the same selection too
    gi_t = torch.from_numpy(gi.astype(np.int32)).cuda()
    cnt = torch.full(gi.shape[:2], gi.shape[2], dtype=torch.int32, device="cuda")
    O2, _ = q().quoka_sparse_gqa_attn(Q, K, V, gi_t, cnt, Kc, Vc)
    torch.cuda.synchronize()
    O2g = O2.float().cpu().numpy().astype(np.float64)
    err2 = np.abs(O2g - O_ref).max() if rows is None else np.abs(np.stack([O2g[r] for r in rows]) - O_ref).max()
    assert err2 <= tol, f"quoka_sparse_gqa_attn O max-abs error {err2:.3e} > {tol}"
    return O


SMALL = [
    # b, nq, nkv, d, T, BCP, NQ, BSA, dtype, structure
    (2, 6, 2, 128, 1000, 100, 7, 300, "bf16", "llama"),
    (1, 8, 8, 64, 333, 37, 37, 50, "bf16", "iid"),
    (1, 3, 1, 128, 0, 64, 4, 16, "bf16", "iid"),
    (1, 4, 1, 128, 200, 64, 1, 500, "f32", "iid"),
    (2, 16, 2, 128, 4096, 256, 16, 1024, "bf16", "qwen"),
    (1, 4, 2, 128, 5000, 16, 16, 0, "bf16", "iid"),
    (1, 2, 2, 64, 40000, 48, 3, 4000, "bf16", "iid"),
    (1, 6, 3, 64, 777, 130, 9, 129, "f32", "llama"),
    (3, 4, 4, 128, 129, 1, 1, 128, "bf16", "iid"),
]


@pytest.mark.parametrize("k", range(len(SMALL)), ids=[f"b{c[0]}_nq{c[1]}_nkv{c[2]}_d{c[3]}_T{c[4]}_L{c[5]}_NQ{c[6]}_BSA{c[7]}_{c[8]}" for c in SMALL])
def test_small_shapes(k):
    b, nq, nkv, d, T, BCP, NQ, BSA, dt, st = SMALL[k]
    x = inputs.make_chunk(b, nq, nkv, d, T, BCP, NQ, BSA, dtype=dt, structure=st, seed=500 + k)
    ref, gi, _ = run_select_and_check(x)
    run_prefill_and_check(x, ref, gi)


def test_tiny_fp32_workload():
    x = inputs.make_workload(0)
    ref, gi, _ = run_select_and_check(x)
    run_prefill_and_check(x, ref, gi)


def test_llama_workload():
    x = inputs.make_workload(1)
    ref, gi, _ = run_select_and_check(x)
    run_prefill_and_check(x, ref, gi)


def test_qwen_workload_T32k():
    x = inputs.make_workload(2)
    ref, gi, _ = run_select_and_check(x)
    run_prefill_and_check(x, ref, gi)


def test_long_workload_T128k():
    x = inputs.make_workload(4)
    ref, gi, _ = run_select_and_check(x)
    r = np.random.default_rng(0)
    nq, L = x.Q.shape[1], x.Q.shape[2]
    rows = [(0, int(h), int(t)) for h, t in zip(r.integers(0, nq, 48), r.integers(0, L, 48))]
    rows += [(0, 0, 0), (0, nq - 1, L - 1), (0, 5, 127), (0, 63, 128)]
    O = run_prefill_and_check(x, ref, gi, rows=rows)
    # every row of one whole KV head (its G query heads x the chunk: every
    # query tile and every chunk-key tail), against the oracle in full
    j = 3
    G = nq // x.K.shape[1]
    hs = slice(j * G, (j + 1) * G)
    js = slice(j, j + 1)
    O_ref, _ = orc.sparse_attention(x.Q[:, hs], x.K[:, js], x.V[:, js], gi[:, js], x.Kc[:, js], x.Vc[:, js])
    err = np.abs(O[:, hs].float().cpu().numpy().astype(np.float64) - O_ref).max()
    assert err <= P.O_TOL_BF16, f"KV head {j}: O max-abs error {err:.3e}"


@pytest.fixture(scope="module")
def sweep():
    s = inputs.make_sweep()
    dev = [P.to_dev(a, s.dtype) for a in (s.Qs, s.Ks, s.Vs)]
    return s, dev


@pytest.mark.parametrize("c", [0, 1, 7, 40, 63])
def test_sweep_chunks(c, sweep):
    """Chunk c of the chunked-prefill sweep, called on strided views into one
    (b, nkv, 16384, d) cache as the benchmark does."""
    s, (Qs, Ks, Vs) = sweep
    x = s.chunk(c)
    L, T = s.BCP, c * s.BCP
    dev = [Qs[:, :, T:T + L], Ks[:, :, :T], Vs[:, :, :T], Ks[:, :, T:T + L], Vs[:, :, T:T + L]]
    ref, gi, _ = run_select_and_check(x, dev=dev)
    r = np.random.default_rng(c)
    b, nq = x.Q.shape[:2]
    rows = [(int(bi), int(h), int(t)) for bi, h, t in zip(r.integers(0, b, 24), r.integers(0, nq, 24),
                                                           r.integers(0, L, 24))]
    run_prefill_and_check(x, ref, gi, rows=rows, dev=dev)


@pytest.mark.parametrize("path", ["gathered", "fused", "split"])
def test_attention_on_given_selection_and_gather(path):
    """quoka_sparse_gqa_attn and quoka_gather_kv on an externally given
    sorted index set (the oracle's), independent of the selection kernels.
    `gathered`: a workspace with room for the gathered copy (step (f) as its
    own kernel, then dense tiles); `fused`: a 256-byte workspace (the
    attention gathers the rows while loading them); `split`: quoka_gather_kv
    then quoka_sparse_gqa_attn_gathered."""
    x = inputs.make_chunk(2, 8, 2, 128, 3000, 200, 8, 700, dtype="bf16", structure="qwen", seed=5)
    ref = orc.select(x.Q, x.K, x.NQ, x.BSA)
    sel = ref["sel"]
    dt = x.dtype
    Q, K, V, Kc, Vc = (P.to_dev(a, dt) for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    kv_idx = torch.from_numpy(sel.astype(np.int32)).cuda()
    kv_count = torch.full((2, 2), sel.shape[2], dtype=torch.int32, device="cuda")
    ws = None if path == "gathered" else torch.zeros(256, dtype=torch.uint8, device="cuda")
    Ks, Vs = q().quoka_gather_kv(K, V, kv_idx, kv_count)
    if path == "split":
        O, lse = q().quoka_sparse_gqa_attn_gathered(Q, Ks, Vs, kv_count, Kc, Vc, want_lse=True, ws=ws)
    else:
        O, lse = q().quoka_sparse_gqa_attn(Q, K, V, kv_idx, kv_count, Kc, Vc, want_lse=True, ws=ws)
    torch.cuda.synchronize()
    O_ref, L_ref = orc.sparse_attention(x.Q, x.K, x.V, sel, x.Kc, x.Vc)
    assert np.abs(O.float().cpu().numpy() - O_ref).max() <= P.O_TOL_BF16
    assert np.abs(lse.cpu().numpy() - L_ref).max() <= P.O_TOL_BF16
    Ks_ref, Vs_ref = orc.gather_kv(x.K, x.V, sel)
    np.testing.assert_array_equal(Ks.float().cpu().numpy(), Ks_ref)
    np.testing.assert_array_equal(Vs.float().cpu().numpy(), Vs_ref)


def test_partial_count_uses_prefix_of_index_rows():
    """kv_count below the row length: only the first kv_count indices of a
    row take part (the rest may hold anything)."""
    x = inputs.make_chunk(1, 4, 2, 64, 500, 40, 4, 100, dtype="f32", structure="iid", seed=6)
    sel = np.stack([[np.sort(np.random.default_rng(k).choice(500, 100, replace=False)) for k in range(2)]])
    counts = np.array([[60, 100]], dtype=np.int32)
    idx = sel.copy()
    idx[0, 0, 60:] = 10 ** 6  # never read
    Q, K, V, Kc, Vc = (P.to_dev(a, "f32") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    O, _ = q().quoka_sparse_gqa_attn(Q, K, V, torch.from_numpy(idx.astype(np.int32)).cuda(),
                                     torch.from_numpy(counts).cuda(), Kc, Vc, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    for j, n in enumerate([60, 100]):
        rows = [(0, h, t) for h in range(2 * j, 2 * j + 2) for t in range(40)]
        sub = np.zeros((1, 2, n), dtype=np.int64)
        sub[0, j] = sel[0, j, :n]
        O_ref, _ = orc.sparse_attention_rows(x.Q, x.K, x.V, sub, x.Kc, x.Vc, rows)
        Og = O.cpu().numpy()
        got = np.stack([Og[r] for r in rows])
        assert np.abs(got - O_ref).max() <= P.O_TOL_F32


@pytest.mark.parametrize("path", ["gathered", "fused"])
def test_partial_count_bf16_tensor_core_path(path):
    """bf16, d = 128: kv_count below the row length on the tensor-core path.
    The workspace starts as all-ones bytes (NaN as bf16), so rows of the
    gathered copy past the count that were not zero-filled would poison the
    output; the index tail holds out-of-range values that must not be read."""
    x = inputs.make_chunk(1, 8, 2, 128, 3000, 200, 8, 600, dtype="bf16", structure="llama", seed=16)
    rng = np.random.default_rng(16)
    sel = np.stack([[np.sort(rng.choice(3000, 600, replace=False)) for _ in range(2)]])
    counts = np.array([[1, 333]], dtype=np.int32)
    idx = sel.copy()
    idx[0, 0, 1:] = 10 ** 6
    idx[0, 1, 333:] = -5
    Q, K, V, Kc, Vc = (P.to_dev(a, "bf16") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    n = q().quoka_attn_workspace_size(1, 2, 128, 600, torch.bfloat16) if path == "gathered" else 256
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")
    O, lse = q().quoka_sparse_gqa_attn(Q, K, V, torch.from_numpy(idx.astype(np.int32)).cuda(),
                                       torch.from_numpy(counts).cuda(), Kc, Vc, want_lse=True, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    Og = O.float().cpu().numpy()
    for j, c in enumerate([1, 333]):
        rows = [(0, h, t) for h in range(4 * j, 4 * j + 4) for t in range(200)]
        sub = np.zeros((1, 2, c), dtype=np.int64)
        sub[0, j] = sel[0, j, :c]
        O_ref, _ = orc.sparse_attention_rows(x.Q, x.K, x.V, sub, x.Kc, x.Vc, rows)
        got = np.stack([Og[r] for r in rows])
        assert np.abs(got - O_ref).max() <= P.O_TOL_BF16


@pytest.mark.parametrize("ws_kind", ["split", "whole"])
def test_split_key_ranges(ws_kind):
    """bf16, d = 128 over gathered rows with few query tiles (8: most SMs
    idle), so that, given room in the workspace, every query tile's key
    tiles are cut into ranges whose partials a merge kernel combines; with a
    256-byte workspace the same call runs unsplit. Both against the oracle.
    The second KV head keeps 5 selected keys, so some of its ranges hold no
    key tile at all (lse = -inf partials). The workspace starts as all-ones
    bytes: partials must be written before they are read."""
    from tests.test_decode import oracle_attention
    x = inputs.make_chunk(1, 4, 2, 128, 3000, 200, 8, 600, dtype="bf16", structure="llama", seed=18)
    rng = np.random.default_rng(18)
    sel = np.stack([[np.sort(rng.choice(3000, 600, replace=False)) for _ in range(2)]])
    counts = np.array([[600, 5]], dtype=np.int32)
    Q, K, V, Kc, Vc = (P.to_dev(a, "bf16") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    idx = torch.from_numpy(sel.astype(np.int32)).cuda()
    cnt = torch.from_numpy(counts).cuda()
    Ks, Vs = q().quoka_gather_kv(K, V, idx, cnt)
    n = (16 << 20) if ws_kind == "split" else 256
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")
    O, lse = q().quoka_sparse_gqa_attn_gathered(Q, Ks, Vs, cnt, Kc, Vc, want_lse=True, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    O_ref, L_ref = oracle_attention(x, sel, counts)
    assert np.abs(O.float().cpu().numpy() - O_ref).max() <= P.O_TOL_BF16
    assert np.abs(lse.cpu().numpy() - L_ref).max() <= P.O_TOL_BF16


@pytest.mark.parametrize("pos,mag,ws_kind", [(300, 40.0, "whole"), (200, 40.0, "whole"), (300, 40.0, "split"),
                                             (300, 24.0, "whole")],
                         ids=["far_later_tile", "far_first_tile_of_warpgroup_1", "far_split", "near"])
def test_scores_far_above_the_first_tile(pos, mag, ws_kind):
    """A key whose score is far above the rows' max over their first key
    tile: selected key `pos` of KV head 0 and every third chunk row of its
    two query heads are mag * e_0, so those rows' score for that key lies
    ~190 (mag = 40) or ~65 (mag = 24) log2 units above the first tile's max.
    The running max of those rows jumps by far more than the lazy-rescale
    threshold, so the O accumulator of the warpgroup that owns the key's
    tile is rescaled in TMEM, and the two warpgroups' partials meet with
    maxima ~190 log2 units apart. Key 200 lies in warpgroup 1's first tile, key 300
    in warpgroup 0's second; "split" cuts the key tiles into ranges. O and
    lse against the oracle."""
    from tests.test_decode import oracle_attention
    x = inputs.make_chunk(1, 4, 2, 128, 3000, 200, 8, 600, dtype="bf16", structure="llama", seed=25)
    rng = np.random.default_rng(25)
    sel = np.stack([[np.sort(rng.choice(3000, 600, replace=False)) for _ in range(2)]])
    counts = np.array([[600, 600]], dtype=np.int32)
    e0 = np.zeros(128)
    e0[0] = mag
    x.K[0, 0, sel[0, 0, pos]] = e0
    x.Q[0, 0:2, 0::3] = e0
    Q, K, V, Kc, Vc = (P.to_dev(a, "bf16") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    idx = torch.from_numpy(sel.astype(np.int32)).cuda()
    cnt = torch.from_numpy(counts).cuda()
    Ks, Vs = q().quoka_gather_kv(K, V, idx, cnt)
    n = (16 << 20) if ws_kind == "split" else 256
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")
    O, lse = q().quoka_sparse_gqa_attn_gathered(Q, Ks, Vs, cnt, Kc, Vc, want_lse=True, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    O_ref, L_ref = oracle_attention(x, sel, counts)
    assert np.isfinite(O.float().cpu().numpy()).all()
    assert np.abs(O.float().cpu().numpy() - O_ref).max() <= P.O_TOL_BF16
    assert np.abs(lse.cpu().numpy() - L_ref).max() <= P.O_TOL_BF16


@pytest.mark.parametrize("no_chunk", [False, True], ids=["with_chunk_keys", "no_chunk_keys"])
def test_split_key_ranges_ragged_through_the_indexed_entry(no_chunk):
    """quoka_sparse_gqa_attn(_ex) with room past the gathered copy: 24 query
    tiles of a ragged chunk (BCP = 200: a full and a 72-row tile per head,
    G = 3, two batches) split their key ranges; with the chunk's own keys
    left out (one rank's partial attention) rows see only selected keys.
    O and lse against the oracle."""
    x = inputs.make_chunk(2, 6, 2, 128, 3000, 200, 8, 700, dtype="bf16", structure="llama", seed=21)
    rng = np.random.default_rng(21)
    sel = np.stack([[np.sort(rng.choice(3000, 700, replace=False)) for _ in range(2)] for _ in range(2)])
    Q, K, V, Kc, Vc = (P.to_dev(a, "bf16") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    idx = torch.from_numpy(sel.astype(np.int32)).cuda()
    cnt = torch.full((2, 2), 700, dtype=torch.int32, device="cuda")
    ws = torch.full((32 << 20,), 255, dtype=torch.uint8, device="cuda")
    O, lse = q().quoka_sparse_gqa_attn(Q, K, V, idx, cnt, Kc, Vc, want_lse=True, ws=ws, no_chunk=no_chunk)
    assert q().quoka_get_device_status(ws) == 0
    O_ref, L_ref = orc.sparse_attention(x.Q, x.K, x.V, sel, x.Kc, x.Vc, include_chunk=not no_chunk)
    assert np.abs(O.float().cpu().numpy() - O_ref).max() <= P.O_TOL_BF16
    assert np.abs(lse.cpu().numpy() - L_ref).max() <= P.O_TOL_BF16


def test_gathered_attention_fp32_and_partial_counts():
    """quoka_gather_kv + quoka_sparse_gqa_attn_gathered in fp32 (CUDA-core
    path), with counts below the row length: the gather writes zeros past the
    count and the attention masks those rows."""
    x = inputs.make_chunk(2, 6, 3, 64, 900, 70, 5, 200, dtype="f32", structure="llama", seed=17)
    rng = np.random.default_rng(17)
    sel = np.stack([[np.sort(rng.choice(900, 200, replace=False)) for _ in range(3)] for _ in range(2)])
    counts = np.array([[200, 0, 17], [5, 199, 200]], dtype=np.int32)
    Q, K, V, Kc, Vc = (P.to_dev(a, "f32") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    idx = torch.from_numpy(sel.astype(np.int32)).cuda()
    cnt = torch.from_numpy(counts).cuda()
    Ks = torch.full((2, 3, 200, 64), float("nan"), device="cuda")
    Vs = torch.full((2, 3, 200, 64), float("nan"), device="cuda")
    q().quoka_gather_kv(K, V, idx, cnt, Ksel=Ks, Vsel=Vs)
    O, lse = q().quoka_sparse_gqa_attn_gathered(Q, Ks, Vs, cnt, Kc, Vc, want_lse=True)
    torch.cuda.synchronize()
    for bi in range(2):
        for j in range(3):
            c = counts[bi, j]
            np.testing.assert_array_equal(Ks[bi, j, :c].cpu().numpy(), x.K[bi, j, sel[bi, j, :c]])
            assert (Ks[bi, j, c:] == 0).all() and (Vs[bi, j, c:] == 0).all()
    rows = [(bi, h, t) for bi in range(2) for h in range(6) for t in range(0, 70, 3)]
    Og = O.cpu().numpy()
    for (bi, h, t) in rows:
        j = h // 2
        sub = np.zeros((2, 3, counts[bi, j]), dtype=np.int64)
        sub[bi, j] = sel[bi, j, :counts[bi, j]]
        O_ref, _ = orc.sparse_attention_rows(x.Q, x.K, x.V, sub, x.Kc, x.Vc, [(bi, h, t)])
        assert np.abs(Og[bi, h, t] - O_ref[0]).max() <= P.O_TOL_F32


def test_planted_exact_ties_go_to_lower_index():
    """Identical key rows get bit-identical scores; at the budget boundary the
    lower key indices must win, deterministically."""
    x = inputs.make_chunk(1, 4, 2, 128, 2048, 64, 4, 300, dtype="bf16", structure="iid", seed=7)
    ref0 = orc.select(x.Q, x.K, x.NQ, x.BSA)
    for j in range(2):
        s = ref0["S_agg"][0, j]
        order = np.argsort(-s, kind="stable")
        boundary = order[x.BSA - 1]
        # make 40 other keys identical copies of the boundary key, straddling it
        others = order[x.BSA - 20:x.BSA + 21]
        for t in others:
            x.K[0, j, t] = x.K[0, j, boundary]
    ref, gi, _ = run_select_and_check(x)
    for j in range(2):
        np.testing.assert_array_equal(gi[0, j], ref["sel"][0, j])
    # deterministic across runs
    _, gi2, _ = run_select_and_check(x)
    np.testing.assert_array_equal(gi, gi2)


def test_dense_reduction_on_gpu():
    """NQ = BCP and BSA = T: the CUDA step equals dense causal attention."""
    x = inputs.make_chunk(1, 8, 2, 128, 700, 96, 96, 700, dtype="bf16", structure="llama", seed=8)
    ref, gi, _ = run_select_and_check(x)
    assert np.array_equal(gi[0, 0], np.arange(700))
    run_prefill_and_check(x, ref, gi)


def test_out_of_range_index_is_latched_not_read():
    x = inputs.make_chunk(1, 2, 1, 64, 100, 8, 2, 10, dtype="f32", structure="iid", seed=9)
    Q, K, V, Kc, Vc = (P.to_dev(a, "f32") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    idx = torch.tensor([[[1, 5, 99, 100, 2000]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[5]], dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    q().quoka_sparse_gqa_attn(Q, K, V, idx, cnt, Kc, Vc, ws=ws)
    assert q().quoka_get_device_status(ws) == 6
    Ks, Vs = q().quoka_gather_kv(K, V, idx, cnt, ws=ws)
    assert q().quoka_get_device_status(ws) == 6
    torch.cuda.synchronize()
    # the in-range rows were still gathered
    np.testing.assert_array_equal(Ks[0, 0, :3].cpu().numpy(), x.K[0, 0, [1, 5, 99]])
    # each call clears the status words first: valid calls on the same
    # workspace read 0 again (the gather's clear runs in a kernel of its own)
    good = torch.tensor([[[1, 5, 99, 7, 8]]], dtype=torch.int32, device="cuda")
    q().quoka_gather_kv(K, V, good, cnt, ws=ws)
    assert q().quoka_get_device_status(ws) == 0 and q().quoka_get_device_fault_site(ws) == 0
    q().quoka_gather_kv(K, V, idx, cnt, ws=ws)
    assert q().quoka_get_device_status(ws) == 6
    q().quoka_sparse_gqa_attn(Q, K, V, good, cnt, Kc, Vc, ws=ws)
    assert q().quoka_get_device_status(ws) == 0


@pytest.mark.parametrize("path", ["gathered", "fused"])
def test_out_of_range_index_latched_bf16_tensor_core_path(path):
    x = inputs.make_chunk(1, 4, 1, 128, 300, 64, 2, 10, dtype="bf16", structure="iid", seed=19)
    Q, K, V, Kc, Vc = (P.to_dev(a, "bf16") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    idx = torch.tensor([[[1, 5, 99, 300, 2000]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[5]], dtype=torch.int32, device="cuda")
    n = q().quoka_attn_workspace_size(1, 1, 128, 5, torch.bfloat16) if path == "gathered" else 256
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    O, _ = q().quoka_sparse_gqa_attn(Q, K, V, idx, cnt, Kc, Vc, ws=ws)
    assert q().quoka_get_device_status(ws) == 6
    assert torch.isfinite(O.float()).all()


def test_index_reuse_across_layers():
    """A later layer attends over the key set an earlier layer selected
    (steps (a)-(e) skipped on that layer): quoka_select on layer A, then
    quoka_sparse_gqa_attn on layer B's Q, K, V with layer A's kv_idx, for
    both attention paths (gathered copy, and gathered while loading)."""
    xa = inputs.make_chunk(1, 8, 2, 128, 3000, 200, 8, 600, dtype="bf16", structure="llama", seed=61)
    xb = inputs.make_chunk(1, 8, 2, 128, 3000, 200, 8, 600, dtype="bf16", structure="llama", seed=62)
    _, gi, gc = run_select_and_check(xa)
    Q, K, V, Kc, Vc = (P.to_dev(a, xb.dtype) for a in (xb.Q, xb.K, xb.V, xb.Kc, xb.Vc))
    idx = torch.from_numpy(gi.astype(np.int32)).cuda()
    cnt = torch.from_numpy(gc.astype(np.int32)).cuda()
    O_ref, L_ref = orc.sparse_attention(xb.Q, xb.K, xb.V, gi, xb.Kc, xb.Vc)
    for ws in (None, torch.zeros(256, dtype=torch.uint8, device="cuda")):
        O, lse = q().quoka_sparse_gqa_attn(Q, K, V, idx, cnt, Kc, Vc, want_lse=True, ws=ws)
        torch.cuda.synchronize()
        err = np.abs(O.float().cpu().numpy().astype(np.float64) - O_ref).max()
        lerr = np.abs(lse.cpu().numpy().astype(np.float64) - L_ref).max()
        assert err <= P.o_tol(xb.dtype), f"O max-abs error {err:.3e}"
        assert lerr <= max(P.LSE_TOL, P.o_tol(xb.dtype)), f"lse max-abs error {lerr:.3e}"


@pytest.mark.parametrize("shape", [
    # b, nq, nkv, d, T, BCP, NQ, BSA, dtype, structure: the fused tensor-core
    # path (bf16, d = 128), the general query select with the tensor-core
    # score, and the fp32 path on the CUDA cores
    (1, 8, 2, 128, 3000, 200, 8, 600, "bf16", "llama"),
    (2, 6, 3, 64, 900, 70, 5, 200, "bf16", "iid"),
    (1, 4, 2, 64, 700, 40, 4, 100, "f32", "llama"),
], ids=["bf16_d128", "bf16_d64", "f32_d64"])
def test_dot_product_score_variant(shape):
    """quoka_select_ex with QUOKA_SCORE_DOT_PRODUCT vs the oracle's
    dot_product=True. The scores are unbounded, so the S_agg tolerance and
    the top-BSA tie band scale with the largest score."""
    b, nq, nkv, d, T, BCP, NQ, BSA, dt, st = shape
    x = inputs.make_chunk(b, nq, nkv, d, T, BCP, NQ, BSA, dtype=dt, structure=st, seed=71)
    Q, K = P.to_dev(x.Q, dt), P.to_dev(x.K, dt)
    kv_idx, kv_count, q_idx, s_agg = q().quoka_select(Q, K, NQ, BSA, want_q_idx=True, want_s_agg=True,
                                                      dot_product=True)
    torch.cuda.synchronize()
    ref = orc.select(x.Q, x.K, NQ, BSA, dot_product=True)
    gq = q_idx.cpu().numpy().astype(np.int64)
    if not P.check_q_idx(gq, ref["SQ"], ref["q_idx"]):
        ref = orc.select(x.Q, x.K, NQ, BSA, override_q_idx=gq, dot_product=True)
    scale = max(1.0, float(np.abs(ref["S_agg"]).max()))
    err = np.abs(s_agg.cpu().numpy().astype(np.float64) - ref["S_agg"]).max()
    assert err <= P.S_TOL * scale, f"S_agg max-abs error {err:.3e} (scores up to {scale:.1f})"
    P.check_kv_sets(kv_idx.cpu().numpy().astype(np.int64), kv_count.cpu().numpy(), ref["S_agg"],
                    min(BSA, T), ref["sel"], band=P.KV_TIE_BAND * scale)
    # flags 0 through quoka_select_ex is quoka_select
    lib = q().load()
    from sparse_kv_selection_quoka_b200._lib import tensor_view, _ptr, _stream
    ws = q().workspace_for(Q, K, NQ, BSA)
    i0 = torch.empty_like(kv_idx)
    c0 = torch.empty_like(kv_count)
    qv, kv = tensor_view(Q), tensor_view(K)
    import ctypes
    st0 = lib.quoka_select_ex(ctypes.byref(qv), ctypes.byref(kv), NQ, BSA, _ptr(i0), _ptr(c0), None, None, 0,
                              _ptr(ws), ws.numel(), _stream(None))
    assert st0 == 0
    i1, _, _, _ = q().quoka_select(Q, K, NQ, BSA)
    torch.cuda.synchronize()
    assert torch.equal(i0, i1)
    assert lib.quoka_select_ex(ctypes.byref(qv), ctypes.byref(kv), NQ, BSA, _ptr(i0), _ptr(c0), None, None, 2,
                               _ptr(ws), ws.numel(), _stream(None)) != 0


def _crowded_bucket_inputs(n_crowd, n_levels, seed, gap=2e-5):
    """Keys whose threshold value bucket (width 1/2048 of the cosine range)
    holds n_crowd keys: n_levels distinct bf16 key vectors near the first
    group mean's direction, all scoring inside one bucket, at least `gap`
    apart (far above the fp32 scores' rounding), each repeated at random
    positions (exact ties). BSA cuts through the crowd. The levels are
    picked with the oracle's scores, so the expected selection is exact:
    order between levels and ties (lower index) alike."""
    T, BSA = 8192, n_crowd // 2 + 7
    x = inputs.make_chunk(1, 8, 2, 128, T, 128, 8, BSA, dtype="bf16", structure="iid", seed=seed)
    rng = np.random.default_rng(seed)
    Qg = orc.select(x.Q, x.K, x.NQ, BSA)["Q_group"]
    for j in range(2):
        u = Qg[0, j, 0] / np.linalg.norm(Qg[0, j, 0])
        cand = P.bf16_round(11.0 * u[None, :] + 0.05 * rng.standard_normal((800, 128)))
        sc = orc.key_scores(Qg[:, j:j + 1], cand[None, None])[0, 0]
        b = np.floor((sc + 1.0) * 2048.0)
        vals, cnts = np.unique(b, return_counts=True)
        idx = np.where(b == vals[np.argmax(cnts)])[0]
        order = idx[np.argsort(sc[idx])]
        pick = [order[0]]
        for i in order[1:]:
            if sc[i] - sc[pick[-1]] >= gap:
                pick.append(i)
        assert len(pick) >= n_levels, "not enough separated levels in one bucket"
        pick = rng.permutation(pick)[:n_levels]
        pos = rng.choice(T, n_crowd, replace=False)
        x.K[0, j, pos] = cand[np.asarray(pick)[np.arange(n_crowd) % n_levels]]
    return x


@pytest.mark.parametrize("n_crowd", [1000, 5000], ids=["list_radix", "row_radix"])
def test_crowded_threshold_bucket(n_crowd):
    """The BSA-th score's value bucket holds 1000 keys (the candidate list
    is resolved by radix passes) or 5000 (more than the list holds: radix
    passes over the row), with exact ties: the selection must equal the
    oracle's exactly, both from quoka_select and from quoka_topk on the
    scores quoka_select returned."""
    x = _crowded_bucket_inputs(n_crowd, 10, 90 + n_crowd)
    ref = orc.select(x.Q, x.K, x.NQ, x.BSA)
    for j in range(2):  # the case is what it claims to be
        s = ref["S_agg"][0, j]
        thr = np.sort(s)[::-1][x.BSA - 1]
        bins = np.floor((s + 1.0) * 2048.0)
        assert (bins == np.floor((thr + 1.0) * 2048.0)).sum() >= n_crowd
    Q, K = P.to_dev(x.Q, x.dtype), P.to_dev(x.K, x.dtype)
    kv_idx, kv_count, q_idx, s_agg = q().quoka_select(Q, K, x.NQ, x.BSA, want_q_idx=True, want_s_agg=True)
    torch.cuda.synchronize()
    gq = q_idx.cpu().numpy().astype(np.int64)
    if not P.check_q_idx(gq, ref["SQ"], ref["q_idx"]):
        ref = orc.select(x.Q, x.K, x.NQ, x.BSA, override_q_idx=gq)
    assert np.abs(s_agg.cpu().numpy().astype(np.float64) - ref["S_agg"]).max() <= P.S_TOL
    np.testing.assert_array_equal(kv_idx.cpu().numpy(), ref["sel"])
    assert np.all(kv_count.cpu().numpy() == x.BSA)
    i2, c2 = q().quoka_topk(s_agg, x.BSA)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(i2.cpu().numpy(), ref["sel"])
