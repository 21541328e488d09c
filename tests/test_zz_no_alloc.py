"""quoka_select_static: key selection for callers that cannot allocate.

Some callers cannot call cudaMalloc (a plugin inside a framework whose own
allocator owns the device memory, or a latency-critical path where an
allocation that may synchronise the device is not acceptable). For them the
library offers quoka_select_static, which takes no workspace and uses a fixed
per-device scratch array instead. These tests call it through the C ABI and
check, on two calls in a row with different inputs (so the second call runs
on scratch the first one left behind), that its outputs equal those of
quoka_select with a caller workspace, within the tolerances the parity tests
use. This file is collected last so that a failure here comes after every
other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_kv_selection_quoka_b200 import inputs
from tests import parity as P

pytestmark = pytest.mark.gpu


def _both(x):
    import sparse_kv_selection_quoka_b200 as q
    Q, K = P.to_dev(x.Q, x.dtype), P.to_dev(x.K, x.dtype)
    a = q.quoka_select(Q, K, x.NQ, x.BSA, want_q_idx=True, want_s_agg=True)
    b = q.quoka_select_static(Q, K, x.NQ, x.BSA, want_q_idx=True, want_s_agg=True)
    torch.cuda.synchronize()
    return a, b


def _compare(a, b):
    kv_a, cnt_a, qi_a, s_a = (t.cpu().numpy() for t in a)
    kv_b, cnt_b, qi_b, s_b = (t.cpu().numpy() for t in b)
    np.testing.assert_array_equal(cnt_b, cnt_a)
    np.testing.assert_array_equal(qi_b, qi_a)
    if s_a.size:
        assert np.abs(s_b.astype(np.float64) - s_a).max() <= P.S_TOL
    # same kernels, same inputs: the selected sets agree exactly
    np.testing.assert_array_equal(kv_b, kv_a)


def test_static_scratch_select_matches_workspace_select_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    first = inputs.make_chunk(1, 24, 8, 128, 8192, 256, 16, 2048, dtype="bf16", structure="llama", seed=41)
    second = inputs.make_chunk(2, 8, 2, 128, 3000, 100, 7, 500, dtype="bf16", structure="qwen", seed=42)
    import sparse_kv_selection_quoka_b200 as q
    for x in (first, second):
        _compare(*_both(x))
        # the fixed scratch's status words (ws = NULL): no device fault
        assert q.quoka_get_device_status(None) == 0
        assert q.quoka_get_device_fault_site(None) == 0


def test_static_scratch_rejects_oversized_shapes():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_kv_selection_quoka_b200 as q
    from sparse_kv_selection_quoka_b200 import _lib
    lib = q.load()
    # S_agg alone would need 4 * 2 * 8 * 200000 bytes > 8 MiB
    Q = torch.zeros((2, 8, 64, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((2, 8, 200000, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((2, 8, 10), dtype=torch.int32, device="cuda")
    cnt = torch.empty((2, 8), dtype=torch.int32, device="cuda")
    qv, kv = _lib.tensor_view(Q), _lib.tensor_view(K)
    st = lib.quoka_select_static(ctypes.byref(qv), ctypes.byref(kv), 4, 10,
                                 ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()),
                                 None, None, None)
    assert st == 3  # QUOKA_ERR_WORKSPACE
