"""Robustness of the CUDA path on the GPU, through the C ABI.

* Timeout path: the tensor-core scoring and attention kernels bound every
  wait. A test hook (quoka_debug_set_wait_hooks) makes one barrier of a
  kernel expect one arrival more than it ever receives and shortens the
  bound to a few milliseconds; the kernel must give up, latch
  QUOKA_ERR_TIMEOUT and a fault site of that kernel in the workspace, drain
  its copies and products and free its TMEM. A normal call on the same
  device right after must then match the oracle (a leaked TMEM allocation
  or a copy still landing would show there). No kernel traps or hangs.
* Repetition: the headline Qwen-shaped step is run many times back to back
  with the L2 flushed in between, as the benchmark runs it; the scores, the
  selected sets and the outputs must be bit-identical to the first call,
  which is checked against the oracle. A race between the kernels'
  producer / consumer hand-offs would show up as a run that differs.
"""
import numpy as np
import pytest
import torch

from oracle import quoka_oracle as orc
from sparse_kv_selection_quoka_b200 import inputs
from tests import parity as P
from tests.test_gpu_parity import run_prefill_and_check, run_select_and_check

pytestmark = pytest.mark.gpu

WAIT_NS = 5_000_000  # the shortened bound of the injected calls (5 ms)
SCORE_SITES = set(range(51, 58))
ATTN_SITES = set(range(11, 16)) | set(range(21, 28)) | set(range(31, 34))


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


def _injected(kind, call):
    """Runs call() with the wait bound shortened and the barrier of `kind`
    injected; returns (status, fault site) read from the workspace it
    returns. The hooks are reset whatever happens."""
    q().quoka_debug_set_wait_hooks(WAIT_NS, kind)
    try:
        ws = call()
        torch.cuda.synchronize()
    finally:
        q().quoka_debug_set_wait_hooks()
    return q().quoka_get_device_status(ws), q().quoka_get_device_fault_site(ws)


def test_scoring_timeout_unwinds_and_next_call_is_exact():
    # 8 KV heads over 16384 keys: every scoring CTA gets 8 tiles of 128 keys,
    # so each one reaches the injected wait (its fourth tile's accumulator)
    x = inputs.make_chunk(1, 32, 8, 128, 16384, 256, 16, 2048, dtype="bf16", structure="qwen", seed=81)
    Q, K = P.to_dev(x.Q, x.dtype), P.to_dev(x.K, x.dtype)
    ws = q().workspace_for(Q, K, x.NQ, x.BSA)

    def call():
        q().quoka_select(Q, K, x.NQ, x.BSA, ws=ws)
        return ws

    status, site = _injected(q()._lib.DEBUG_INJECT_SCORE, call)
    assert status == 5, f"status {status} (want QUOKA_ERR_TIMEOUT)"
    assert site in SCORE_SITES, f"fault site {site}"
    # the same device and workspace, hooks off: exact again
    q().quoka_select(Q, K, x.NQ, x.BSA, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    assert q().quoka_get_device_fault_site(ws) == 0
    ref, gi, _ = run_select_and_check(x)
    run_prefill_and_check(x, ref, gi, rows=[(0, h, t) for h in (0, 13, 31) for t in range(0, 256, 5)])


@pytest.mark.parametrize("ws_bytes", [256, 16 << 20], ids=["whole", "split_key_ranges"])
def test_attention_timeout_unwinds_and_next_call_is_exact(ws_bytes):
    """With a 256-byte workspace every query tile runs whole; with room for
    the partials its key tiles are split into ranges (16 query tiles), and
    the merge kernel runs after the kernel that gave up."""
    x = inputs.make_chunk(1, 8, 2, 128, 3000, 200, 8, 700, dtype="bf16", structure="qwen", seed=82)
    ref = orc.select(x.Q, x.K, x.NQ, x.BSA)
    sel = ref["sel"]
    Q, K, V, Kc, Vc = (P.to_dev(a, x.dtype) for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    kv_idx = torch.from_numpy(sel.astype(np.int32)).cuda()
    kv_count = torch.full((1, 2), sel.shape[2], dtype=torch.int32, device="cuda")
    Ks, Vs = q().quoka_gather_kv(K, V, kv_idx, kv_count)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")

    def call():
        q().quoka_sparse_gqa_attn_gathered(Q, Ks, Vs, kv_count, Kc, Vc, ws=ws)
        return ws

    status, site = _injected(q()._lib.DEBUG_INJECT_ATTN, call)
    assert status == 5, f"status {status} (want QUOKA_ERR_TIMEOUT)"
    assert site in ATTN_SITES, f"fault site {site}"
    O, lse = q().quoka_sparse_gqa_attn_gathered(Q, Ks, Vs, kv_count, Kc, Vc, want_lse=True, ws=ws)
    assert q().quoka_get_device_status(ws) == 0
    O_ref, L_ref = orc.sparse_attention(x.Q, x.K, x.V, sel, x.Kc, x.Vc)
    assert np.abs(O.float().cpu().numpy() - O_ref).max() <= P.O_TOL_BF16
    assert np.abs(lse.cpu().numpy() - L_ref).max() <= P.O_TOL_BF16


def test_hooks_reject_unknown_injection():
    with pytest.raises(q().QuokaError):
        q().quoka_debug_set_wait_hooks(0, 7)
    q().quoka_debug_set_wait_hooks()


def test_headline_step_repeats_bit_identical():
    """The Qwen-shaped layer at T = 32768: quoka_select (with S_agg) and
    quoka_prefill_chunk, 50 times each, alternating, with a 256 MiB L2-flush
    write before every call; every call equals the first bit for bit, and the
    first equals the oracle."""
    x = inputs.make_workload(2)
    dev = [P.to_dev(a, x.dtype) for a in (x.Q, x.K, x.V, x.Kc, x.Vc)]
    Q, K, V, Kc, Vc = dev
    ws = q().workspace_for(Q, K, x.NQ, x.BSA)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    bsa = min(x.BSA, x.K.shape[2])
    kv_idx = torch.empty((1, 8, bsa), dtype=torch.int32, device="cuda")
    kv_count = torch.empty((1, 8), dtype=torch.int32, device="cuda")
    q_idx = torch.empty((1, 32, x.NQ), dtype=torch.int32, device="cuda")
    s_agg = torch.empty((1, 8, x.K.shape[2]), dtype=torch.float32, device="cuda")
    O = torch.empty_like(Q)
    kv_step = torch.empty_like(kv_idx)
    first = None
    n_bad = 0
    for it in range(50):
        flush.fill_(it & 0xFF)
        q().quoka_select(Q, K, x.NQ, x.BSA, kv_idx=kv_idx, kv_count=kv_count, q_idx=q_idx, s_agg=s_agg, ws=ws)
        flush.fill_((it + 1) & 0xFF)
        q().quoka_prefill_chunk(Q, K, V, Kc, Vc, x.NQ, x.BSA, O=O, kv_idx=kv_step, ws=ws)
        if first is None:
            torch.cuda.synchronize()
            first = [t.clone() for t in (s_agg, kv_idx, kv_count, q_idx, O, kv_step)]
            continue
        same = [torch.equal(a, b) for a, b in zip((s_agg, kv_idx, kv_count, q_idx, O, kv_step), first)]
        if not all(same):
            n_bad += 1
    assert q().quoka_get_device_status(ws) == 0
    assert n_bad == 0, f"{n_bad} of 49 repetitions differ from the first call"
    # the first call against the oracle
    s0, k0, c0, qi0, O0, ks0 = (t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()
                                for t in first)
    ref = orc.select(x.Q, x.K, x.NQ, x.BSA)
    gq = qi0.astype(np.int64)
    if not P.check_q_idx(gq, ref["SQ"], ref["q_idx"]):
        ref = orc.select(x.Q, x.K, x.NQ, x.BSA, override_q_idx=gq)
    err = np.abs(s0.astype(np.float64) - ref["S_agg"]).max()
    assert err <= P.S_TOL, f"S_agg max-abs error {err:.3e}"
    gi = k0.astype(np.int64)
    P.check_kv_sets(gi, c0, ref["S_agg"], bsa, ref["sel"])
    np.testing.assert_array_equal(ks0, k0)
    r = np.random.default_rng(3)
    rows = [(0, int(h), int(t)) for h, t in zip(r.integers(0, 32, 96), r.integers(0, 512, 96))]
    O_ref, _ = orc.sparse_attention_rows(x.Q, x.K, x.V, gi, x.Kc, x.Vc, rows)
    got = np.stack([O0[rw] for rw in rows])
    assert np.abs(got - O_ref).max() <= P.O_TOL_BF16


@pytest.mark.parametrize("BCP", [512, 1])
def test_step_replays_from_a_cuda_graph(BCP):
    """quoka_prefill_chunk enqueues only kernels and a memset on its stream
    (no allocation, no synchronisation), so a CUDA graph can capture the
    whole step; replaying the graph gives the eager call's outputs bit for
    bit (Qwen-shaped layer at T = 8192, a full chunk and a decode token)."""
    x = inputs.make_chunk(1, 32, 8, 128, 8192, BCP, min(32, BCP), 2048, dtype="bf16", structure="qwen", seed=83)
    Q, K, V, Kc, Vc = (P.to_dev(a, x.dtype) for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    ws = q().workspace_for(Q, K, x.NQ, x.BSA)
    O = torch.empty_like(Q)
    kv_idx = torch.empty((1, 8, 2048), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q().quoka_prefill_chunk(Q, K, V, Kc, Vc, x.NQ, x.BSA, O=O, kv_idx=kv_idx, ws=ws, stream=s)
    s.synchronize()
    O_eager, idx_eager = O.clone(), kv_idx.clone()
    O.zero_()
    kv_idx.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        q().quoka_prefill_chunk(Q, K, V, Kc, Vc, x.NQ, x.BSA, O=O, kv_idx=kv_idx, ws=ws, stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert q().quoka_get_device_status(ws) == 0
    assert torch.equal(kv_idx, idx_eager)
    assert torch.equal(O, O_eager)


GUARD = 4096  # bytes of sentinel on each side of every output


class Guarded:
    """A tensor of the given shape and dtype between two sentinel bands of
    GUARD bytes inside one larger byte buffer (the band lengths keep the
    tensor's 256-byte alignment)."""

    def __init__(self, shape, dtype, fill=0x5A):
        esize = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * esize
        self.fill = fill
        self.buf = torch.full((2 * GUARD + self.n,), fill, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + self.n].view(dtype).view(*shape)

    def intact(self):
        return bool((self.buf[:GUARD] == self.fill).all()) and bool((self.buf[GUARD + self.n:] == self.fill).all())


@pytest.mark.parametrize("BCP", [1, 160], ids=["decode_token", "chunk"])
def test_calls_write_only_inside_their_outputs_and_workspace(BCP):
    """Every output of quoka_select, quoka_gather_kv, quoka_sparse_gqa_attn
    (gathered copy and split key ranges inside its workspace),
    quoka_decode_attn and quoka_prefill_chunk, and the workspace itself
    (exactly quoka_workspace_size bytes), sits between sentinel bands; after
    each call the bands are unchanged and the outputs equal those of the
    same call on plainly allocated buffers."""
    NQ, BSA, T = min(8, BCP), 400, 1500
    x = inputs.make_chunk(1, 8, 2, 128, T, BCP, NQ, BSA, dtype="bf16", structure="llama", seed=31)
    Q, K, V, Kc, Vc = (P.to_dev(a, "bf16") for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
    b, nq, _, d = Q.shape
    nkv = K.shape[1]
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    n = q().quoka_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, bf)
    ws = Guarded((n,), torch.uint8)

    idx, cnt = Guarded((b, nkv, BSA), i32), Guarded((b, nkv), i32)
    qi, sg = Guarded((b, nq, NQ), i32), Guarded((b, nkv, T), f32)
    q().quoka_select(Q, K, NQ, BSA, kv_idx=idx.t, kv_count=cnt.t, q_idx=qi.t, s_agg=sg.t, ws=ws.t)
    r_idx, r_cnt, r_qi, r_sg = q().quoka_select(Q, K, NQ, BSA, want_q_idx=True, want_s_agg=True)
    torch.cuda.synchronize()
    assert q().quoka_get_device_status(ws.t) == 0
    assert torch.equal(idx.t, r_idx) and torch.equal(cnt.t, r_cnt) and torch.equal(qi.t, r_qi)
    assert torch.equal(sg.t, r_sg)

    Ks, Vs = Guarded((b, nkv, BSA, d), bf), Guarded((b, nkv, BSA, d), bf)
    q().quoka_gather_kv(K, V, idx.t, cnt.t, Ksel=Ks.t, Vsel=Vs.t, ws=ws.t)
    r_Ks, r_Vs = q().quoka_gather_kv(K, V, r_idx, r_cnt)
    torch.cuda.synchronize()
    assert torch.equal(Ks.t, r_Ks) and torch.equal(Vs.t, r_Vs)

    O, L = Guarded((b, nq, BCP, d), bf), Guarded((b, nq, BCP), f32)
    q().quoka_sparse_gqa_attn(Q, K, V, idx.t, cnt.t, Kc, Vc, O=O.t, lse=L.t, ws=ws.t)
    r_O, r_L = q().quoka_sparse_gqa_attn(Q, K, V, r_idx, r_cnt, Kc, Vc, want_lse=True,
                                         ws=torch.empty(n, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert q().quoka_get_device_status(ws.t) == 0
    assert torch.equal(O.t, r_O) and torch.equal(L.t, r_L)

    O2, L2, kvi = Guarded((b, nq, BCP, d), bf), Guarded((b, nq, BCP), f32), Guarded((b, nkv, BSA), i32)
    q().quoka_prefill_chunk(Q, K, V, Kc, Vc, NQ, BSA, O=O2.t, lse=L2.t, kv_idx=kvi.t, ws=ws.t)
    r_O2, r_L2, r_kvi = q().quoka_prefill_chunk(Q, K, V, Kc, Vc, NQ, BSA, want_lse=True, want_kv_idx=True)
    torch.cuda.synchronize()
    assert q().quoka_get_device_status(ws.t) == 0
    assert torch.equal(O2.t, r_O2) and torch.equal(L2.t, r_L2) and torch.equal(kvi.t, r_kvi)

    bands = [ws, idx, cnt, qi, sg, Ks, Vs, O, L, O2, L2, kvi]
    if BCP == 1:
        nd = q().quoka_decode_workspace_size(b, nq, nkv, d, BCP, BSA, bf)
        wsd = Guarded((nd,), torch.uint8)
        O3, L3 = Guarded((b, nq, BCP, d), bf), Guarded((b, nq, BCP), f32)
        q().quoka_decode_attn(Q, K, V, idx.t, cnt.t, Kc, Vc, O=O3.t, lse=L3.t, ws=wsd.t)
        r_O3, r_L3 = q().quoka_decode_attn(Q, K, V, r_idx, r_cnt, Kc, Vc, want_lse=True)
        torch.cuda.synchronize()
        assert q().quoka_get_device_status(wsd.t) == 0
        assert torch.equal(O3.t, r_O3) and torch.equal(L3.t, r_L3)
        bands += [wsd, O3, L3]
    bad = [i for i, g in enumerate(bands) if not g.intact()]
    assert not bad, f"sentinel bands overwritten around outputs {bad}"
