"""ctypes binding of libquoka.so.

Argument marshalling only: torch tensors are turned into the C ABI's strided
views (device pointer, dtype, shape, element strides) and the call is
enqueued on the current CUDA stream. Every step of the computation runs in
the library's CUDA kernels. Output and workspace buffers the caller does not
pass are allocated with torch (the library itself never allocates).

The library must have been built (python -m sparse_kv_selection_quoka_b200.build);
there is no fallback: a missing library raises at load time.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libquoka.so")

QUOKA_F32 = 0
QUOKA_BF16 = 1

STATUS_NAMES = {
    0: "QUOKA_OK",
    1: "QUOKA_ERR_INVALID_ARG",
    2: "QUOKA_ERR_UNSUPPORTED",
    3: "QUOKA_ERR_WORKSPACE",
    4: "QUOKA_ERR_CUDA",
    5: "QUOKA_ERR_TIMEOUT",
    6: "QUOKA_ERR_BOUNDS",
}

# names of every entry point include/quoka.h declares
EXPORTS = (
    "quoka_workspace_size",
    "quoka_select_workspace_size",
    "quoka_attn_workspace_size",
    "quoka_select",
    "quoka_select_ex",
    "quoka_gather_kv",
    "quoka_sparse_gqa_attn",
    "quoka_sparse_gqa_attn_gathered",
    "quoka_prefill_chunk",
    "quoka_get_device_status",
    "quoka_status_string",
    "quoka_select_static",
    "quoka_sparse_gqa_attn_ex",
    "quoka_shard_candidate_scores",
    "quoka_shard_interleave",
    "quoka_topk",
    "quoka_shard_take",
    "quoka_combine_partials",
    "quoka_decode_workspace_size",
    "quoka_decode_attn",
    "quoka_get_device_fault_site",
    "quoka_debug_set_wait_hooks",
)


class QuokaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class quoka_tensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int),
        ("shape", ctypes.c_int64 * 4),
        ("stride", ctypes.c_int64 * 4),
    ]


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_T = ctypes.POINTER(quoka_tensor)
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float


def load() -> ctypes.CDLL:
    """Load libquoka.so once and declare the signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m sparse_kv_selection_quoka_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(LIB_PATH)
        lib.quoka_workspace_size.restype = _SZ
        lib.quoka_workspace_size.argtypes = [_I, _I, _I, _I, _I64, _I, _I, _I, _I]
        lib.quoka_select_workspace_size.restype = _SZ
        lib.quoka_select_workspace_size.argtypes = [_I, _I, _I, _I, _I64, _I, _I, _I, _I]
        lib.quoka_attn_workspace_size.restype = _SZ
        lib.quoka_attn_workspace_size.argtypes = [_I, _I, _I, _I, _I]
        lib.quoka_select.restype = _I
        lib.quoka_select.argtypes = [_T, _T, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]
        lib.quoka_select_ex.restype = _I
        lib.quoka_select_ex.argtypes = [_T, _T, _I, _I, _P, _P, _P, _P, ctypes.c_uint32, _P, _SZ, _P]
        lib.quoka_gather_kv.restype = _I
        lib.quoka_gather_kv.argtypes = [_T, _T, _P, _P, _I, _P, _P, _P, _SZ, _P]
        lib.quoka_sparse_gqa_attn.restype = _I
        lib.quoka_sparse_gqa_attn.argtypes = [_T, _T, _T, _P, _P, _I, _T, _T, _F, _P, _P, _P, _SZ, _P]
        lib.quoka_sparse_gqa_attn_gathered.restype = _I
        lib.quoka_sparse_gqa_attn_gathered.argtypes = [_T, _T, _T, _P, _T, _T, _F, _P, _P, _P, _SZ, _P]
        lib.quoka_prefill_chunk.restype = _I
        lib.quoka_prefill_chunk.argtypes = [_T, _T, _T, _T, _T, _I, _I, _F, _P, _P, _P, _P, _SZ, _P]
        lib.quoka_get_device_status.restype = _I
        lib.quoka_get_device_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_int32)]
        lib.quoka_status_string.restype = ctypes.c_char_p
        lib.quoka_status_string.argtypes = [_I]
        lib.quoka_select_static.restype = _I
        lib.quoka_select_static.argtypes = [_T, _T, _I, _I, _P, _P, _P, _P, _P]
        lib.quoka_sparse_gqa_attn_ex.restype = _I
        lib.quoka_sparse_gqa_attn_ex.argtypes = [_T, _T, _T, _P, _P, _I, _T, _T, _F, _P, _P, ctypes.c_uint32,
                                                 _P, _SZ, _P]
        lib.quoka_shard_candidate_scores.restype = _I
        lib.quoka_shard_candidate_scores.argtypes = [_P, _I, _I, _I64, _P, _P, _I, _I, _P, _P, _P, _SZ, _P]
        lib.quoka_shard_interleave.restype = _I
        lib.quoka_shard_interleave.argtypes = [_P, _I, _I64, _I64, _P, _P]
        lib.quoka_topk.restype = _I
        lib.quoka_topk.argtypes = [_P, _I, _I, _I64, _I, _P, _P, _P, _SZ, _P]
        lib.quoka_shard_take.restype = _I
        lib.quoka_shard_take.argtypes = [_P, _P, _I, _I, _I, _P, _I, _I, _P, _P, _P, _SZ, _P]
        lib.quoka_decode_workspace_size.restype = _SZ
        lib.quoka_decode_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, _I]
        lib.quoka_decode_attn.restype = _I
        lib.quoka_decode_attn.argtypes = [_T, _T, _T, _P, _P, _I, _T, _T, _F, _P, _P, _P, _SZ, _P]
        lib.quoka_get_device_fault_site.restype = _I
        lib.quoka_get_device_fault_site.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_int32)]
        lib.quoka_debug_set_wait_hooks.restype = _I
        lib.quoka_debug_set_wait_hooks.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
        lib.quoka_combine_partials.restype = _I
        lib.quoka_combine_partials.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P]
        _lib = lib
        return lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return QUOKA_F32
    if t.dtype == torch.bfloat16:
        return QUOKA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def tensor_view(t: torch.Tensor) -> quoka_tensor:
    """The C ABI view of a 4-D tensor (no copy)."""
    if t.dim() != 4:
        raise ValueError("expected a 4-D tensor")
    v = quoka_tensor()
    v.data = t.data_ptr() if t.numel() > 0 else 0
    v.dtype = _dtype_code(t)
    for i in range(4):
        v.shape[i] = t.shape[i]
        v.stride[i] = t.stride(i)
    return v


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise QuokaError(status, where)


def _code(dtype) -> int:
    return dtype if isinstance(dtype, int) else (QUOKA_BF16 if dtype == torch.bfloat16 else QUOKA_F32)


def quoka_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, dtype) -> int:
    return int(load().quoka_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, _code(dtype)))


def quoka_select_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, dtype) -> int:
    return int(load().quoka_select_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, _code(dtype)))


def quoka_attn_workspace_size(b, nkv, d, BSA_eff, dtype) -> int:
    return int(load().quoka_attn_workspace_size(b, nkv, d, BSA_eff, _code(dtype)))


def quoka_decode_workspace_size(b, nq, nkv, d, BCP, BSA_eff, dtype) -> int:
    return int(load().quoka_decode_workspace_size(b, nq, nkv, d, BCP, BSA_eff, _code(dtype)))


def quoka_decode_attn(Q, K, V, kv_idx, kv_count, Kc, Vc, scale=None, *, O=None, lse=None, want_lse=False,
                      ws=None, stream=None):
    """Steps (f)+(g) for a short chunk (G * BCP <= 64 query rows per KV head):
    the attention of quoka_sparse_gqa_attn, by key slices read straight from
    the cache. Returns (O (b,nq,BCP,d), lse or None); `ws` defaults to a new
    workspace of quoka_decode_workspace_size bytes."""
    lib = load()
    b, nq, BCP, d = Q.shape
    if scale is None:
        scale = d ** -0.5
    if O is None:
        O = torch.empty((b, nq, BCP, d), dtype=Q.dtype, device=Q.device)
    if lse is None and want_lse:
        lse = torch.empty((b, nq, BCP), dtype=torch.float32, device=Q.device)
    if ws is None:
        n = quoka_decode_workspace_size(b, nq, K.shape[1], d, BCP, kv_idx.shape[2], Q.dtype)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=Q.device)
    views = [tensor_view(x) for x in (Q, K, V, Kc, Vc)]
    st = lib.quoka_decode_attn(ctypes.byref(views[0]), ctypes.byref(views[1]), ctypes.byref(views[2]),
                               _ptr(kv_idx) if kv_idx.numel() else None, _ptr(kv_count), kv_idx.shape[2],
                               ctypes.byref(views[3]), ctypes.byref(views[4]), float(scale), _ptr(O), _ptr(lse),
                               _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "quoka_decode_attn")
    return O, lse


def workspace_for(Q: torch.Tensor, K: torch.Tensor, NQ: int, BSA: int) -> torch.Tensor:
    """A torch-allocated workspace large enough for every call on these shapes."""
    b, nq, BCP, d = Q.shape
    nkv, T = K.shape[1], K.shape[2]
    n = quoka_workspace_size(b, nq, nkv, d, T, BCP, max(1, min(NQ, BCP)), BSA, Q.dtype)
    if n == 0:
        raise QuokaError(1, "quoka_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=Q.device)


SCORE_DOT_PRODUCT = 1  # quoka_select_ex flag: plain dot-product score


def quoka_select(Q, K, NQ: int, BSA: int, *, kv_idx=None, kv_count=None, q_idx=None,
                 s_agg=None, want_q_idx=False, want_s_agg=False, ws=None, stream=None,
                 dot_product=False):
    """Steps (a)-(e). Returns (kv_idx (b,nkv,BSA_eff) int32 ascending,
    kv_count (b,nkv) int32, q_idx or None, s_agg or None). dot_product=True
    calls quoka_select_ex with the dot-product score variant."""
    lib = load()
    b, nq, BCP, d = Q.shape
    nkv, T = K.shape[1], K.shape[2]
    bsa_eff = min(BSA, T)
    dev = Q.device
    if kv_idx is None:
        kv_idx = torch.empty((b, nkv, bsa_eff), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((b, nkv), dtype=torch.int32, device=dev)
    if q_idx is None and want_q_idx:
        q_idx = torch.empty((b, nq, NQ), dtype=torch.int32, device=dev)
    if s_agg is None and want_s_agg:
        s_agg = torch.empty((b, nkv, T), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace_for(Q, K, NQ, BSA)
    qv, kv = tensor_view(Q), tensor_view(K)
    outs = (_ptr(kv_idx) if kv_idx.numel() else None, _ptr(kv_count), _ptr(q_idx),
            _ptr(s_agg) if s_agg is not None and s_agg.numel() else None)
    if dot_product:
        st = lib.quoka_select_ex(ctypes.byref(qv), ctypes.byref(kv), NQ, BSA, *outs, SCORE_DOT_PRODUCT,
                                 _ptr(ws), ws.numel(), _stream(stream))
        _check(st, "quoka_select_ex")
    else:
        st = lib.quoka_select(ctypes.byref(qv), ctypes.byref(kv), NQ, BSA, *outs, _ptr(ws), ws.numel(),
                              _stream(stream))
        _check(st, "quoka_select")
    return kv_idx, kv_count, q_idx, s_agg


def quoka_gather_kv(K, V, kv_idx, kv_count, *, Ksel=None, Vsel=None, ws=None, stream=None):
    """Step (f). Returns (Ksel, Vsel) of shape (b, nkv, BSA_eff, d)."""
    lib = load()
    b, nkv, T, d = K.shape
    bsa_eff = kv_idx.shape[2]
    if Ksel is None:
        Ksel = torch.empty((b, nkv, bsa_eff, d), dtype=K.dtype, device=K.device)
    if Vsel is None:
        Vsel = torch.empty((b, nkv, bsa_eff, d), dtype=V.dtype, device=V.device)
    kv, vv = tensor_view(K), tensor_view(V)
    st = lib.quoka_gather_kv(ctypes.byref(kv), ctypes.byref(vv),
                             _ptr(kv_idx) if kv_idx.numel() else None, _ptr(kv_count), bsa_eff,
                             _ptr(Ksel) if Ksel.numel() else None, _ptr(Vsel) if Vsel.numel() else None,
                             _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "quoka_gather_kv")
    return Ksel, Vsel


ATTN_NO_CHUNK_KEYS = 1  # quoka_sparse_gqa_attn_ex flag: the chunk's own keys left out


def quoka_sparse_gqa_attn(Q, K, V, kv_idx, kv_count, Kc, Vc, scale=None, *, O=None, lse=None,
                          want_lse=False, ws=None, stream=None, no_chunk=False):
    """Steps (f)+(g). Returns (O (b,nq,BCP,d), lse or None). Without `ws`
    a workspace of quoka_attn_workspace_size bytes is allocated (the path
    that gathers the selected rows first); a 256-byte `ws` selects the path
    that gathers them while loading."""
    lib = load()
    b, nq, BCP, d = Q.shape
    if scale is None:
        scale = d ** -0.5
    if O is None:
        O = torch.empty((b, nq, BCP, d), dtype=Q.dtype, device=Q.device)
    if lse is None and want_lse:
        lse = torch.empty((b, nq, BCP), dtype=torch.float32, device=Q.device)
    if ws is None:
        n = quoka_attn_workspace_size(b, K.shape[1], d, kv_idx.shape[2], Q.dtype)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=Q.device)
    views = [tensor_view(x) for x in (Q, K, V, Kc, Vc)]
    args = ([ctypes.byref(views[0]), ctypes.byref(views[1]), ctypes.byref(views[2]),
             _ptr(kv_idx) if kv_idx.numel() else None, _ptr(kv_count), kv_idx.shape[2],
             ctypes.byref(views[3]), ctypes.byref(views[4]), float(scale), _ptr(O), _ptr(lse)])
    if no_chunk:
        st = lib.quoka_sparse_gqa_attn_ex(*args, ATTN_NO_CHUNK_KEYS, _ptr(ws), ws.numel(), _stream(stream))
        _check(st, "quoka_sparse_gqa_attn_ex")
    else:
        st = lib.quoka_sparse_gqa_attn(*args, _ptr(ws), ws.numel(), _stream(stream))
        _check(st, "quoka_sparse_gqa_attn")
    return O, lse


def quoka_sparse_gqa_attn_gathered(Q, Ksel, Vsel, kv_count, Kc, Vc, scale=None, *, O=None, lse=None,
                                   want_lse=False, ws=None, stream=None):
    """Step (g) on an already gathered selected KV (rows of Ksel / Vsel,
    e.g. from quoka_gather_kv). Returns (O, lse or None)."""
    lib = load()
    b, nq, BCP, d = Q.shape
    if scale is None:
        scale = d ** -0.5
    if O is None:
        O = torch.empty((b, nq, BCP, d), dtype=Q.dtype, device=Q.device)
    if lse is None and want_lse:
        lse = torch.empty((b, nq, BCP), dtype=torch.float32, device=Q.device)
    if ws is None:
        ws = torch.empty(256, dtype=torch.uint8, device=Q.device)
    views = [tensor_view(x) for x in (Q, Ksel, Vsel, Kc, Vc)]
    st = lib.quoka_sparse_gqa_attn_gathered(ctypes.byref(views[0]), ctypes.byref(views[1]),
                                            ctypes.byref(views[2]), _ptr(kv_count), ctypes.byref(views[3]),
                                            ctypes.byref(views[4]), float(scale), _ptr(O), _ptr(lse),
                                            _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "quoka_sparse_gqa_attn_gathered")
    return O, lse


def quoka_prefill_chunk(Q, K, V, Kc, Vc, NQ: int, BSA: int, scale=None, *, O=None, lse=None,
                        want_lse=False, kv_idx=None, want_kv_idx=False, ws=None, stream=None):
    """Steps (a)-(g). Returns (O, lse or None, kv_idx or None)."""
    lib = load()
    b, nq, BCP, d = Q.shape
    nkv, T = K.shape[1], K.shape[2]
    if scale is None:
        scale = d ** -0.5
    if O is None:
        O = torch.empty((b, nq, BCP, d), dtype=Q.dtype, device=Q.device)
    if lse is None and want_lse:
        lse = torch.empty((b, nq, BCP), dtype=torch.float32, device=Q.device)
    if kv_idx is None and want_kv_idx:
        kv_idx = torch.empty((b, nkv, min(BSA, T)), dtype=torch.int32, device=Q.device)
    if ws is None:
        ws = workspace_for(Q, K, NQ, BSA)
    views = [tensor_view(x) for x in (Q, K, V, Kc, Vc)]
    st = lib.quoka_prefill_chunk(*[ctypes.byref(v) for v in views], NQ, BSA, float(scale), _ptr(O),
                                 _ptr(lse), _ptr(kv_idx) if kv_idx is not None and kv_idx.numel() else None,
                                 _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "quoka_prefill_chunk")
    return O, lse, kv_idx


def quoka_get_device_status(ws, stream=None) -> int:
    """Synchronise the stream and return the device status word of ws
    (ws = None: that of quoka_select_static's fixed scratch)."""
    lib = load()
    out = ctypes.c_int32(0)
    st = lib.quoka_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(out))
    _check(st, "quoka_get_device_status")
    return int(out.value)


def quoka_get_device_fault_site(ws, stream=None) -> int:
    """Synchronise the stream and return the fault-site word of ws (0: no
    device fault in the latest call that used ws; ws = None: quoka_select_static's
    fixed scratch)."""
    lib = load()
    out = ctypes.c_int32(0)
    st = lib.quoka_get_device_fault_site(_ptr(ws), _stream(stream), ctypes.byref(out))
    _check(st, "quoka_get_device_fault_site")
    return int(out.value)


DEBUG_INJECT_NONE = 0
DEBUG_INJECT_SCORE = 1
DEBUG_INJECT_ATTN = 2


def quoka_debug_set_wait_hooks(wait_limit_ns: int = 0, inject: int = DEBUG_INJECT_NONE) -> None:
    """Test hooks of the tensor-core kernels: the bound of every wait (0 =
    the default 2 s) and an injected barrier that never completes (see
    include/quoka.h). Process-wide; reset with no arguments."""
    _check(load().quoka_debug_set_wait_hooks(int(wait_limit_ns), int(inject)), "quoka_debug_set_wait_hooks")


def quoka_status_string(status: int) -> str:
    return load().quoka_status_string(status).decode()


STATIC_SCRATCH_BYTES = 8 << 20


def quoka_select_static(Q, K, NQ: int, BSA: int, *, kv_idx=None, kv_count=None, q_idx=None,
                        s_agg=None, want_q_idx=False, want_s_agg=False, stream=None):
    """quoka_select for callers that cannot allocate device scratch: the
    library uses its own fixed per-device scratch array (8 MiB) instead of a
    workspace. Outputs the caller does not pass are allocated here with torch
    (the C entry point itself allocates nothing). Calls sharing a device must
    not overlap on the GPU."""
    lib = load()
    b, nq, BCP, d = Q.shape
    nkv, T = K.shape[1], K.shape[2]
    bsa_eff = min(BSA, T)
    dev = Q.device
    if kv_idx is None:
        kv_idx = torch.empty((b, nkv, bsa_eff), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((b, nkv), dtype=torch.int32, device=dev)
    if q_idx is None and want_q_idx:
        q_idx = torch.empty((b, nq, NQ), dtype=torch.int32, device=dev)
    if s_agg is None and want_s_agg:
        s_agg = torch.empty((b, nkv, T), dtype=torch.float32, device=dev)
    qv, kv = tensor_view(Q), tensor_view(K)
    st = lib.quoka_select_static(ctypes.byref(qv), ctypes.byref(kv), NQ, BSA,
                                 _ptr(kv_idx) if kv_idx.numel() else None, _ptr(kv_count),
                                 _ptr(q_idx), _ptr(s_agg) if s_agg is not None and s_agg.numel() else None,
                                 _stream(stream))
    _check(st, "quoka_select_static")
    return kv_idx, kv_count, q_idx, s_agg


# ---------------------------------------------------------------- prior keys split over ranks

def quoka_shard_candidate_scores(s_agg, kv_idx, kv_count, C, *, scores=None, cand_idx=None, ws=None,
                                 stream=None):
    """This rank's candidates padded to length C: returns (scores (b,nkv,C)
    float, cand_idx (b,nkv,C) int32), padding -inf / -1."""
    lib = load()
    b, nkv, T = s_agg.shape
    Cl = kv_idx.shape[2]
    if scores is None:
        scores = torch.empty((b, nkv, C), dtype=torch.float32, device=s_agg.device)
    if cand_idx is None:
        cand_idx = torch.empty((b, nkv, C), dtype=torch.int32, device=s_agg.device)
    st = lib.quoka_shard_candidate_scores(_ptr(s_agg), b, nkv, T, _ptr(kv_idx) if kv_idx.numel() else None,
                                          _ptr(kv_count), Cl, C, _ptr(scores), _ptr(cand_idx), _ptr(ws),
                                          0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "quoka_shard_candidate_scores")
    return scores, cand_idx


def quoka_shard_interleave(gathered, *, out=None, stream=None):
    """(N, b, nkv, C) 32-bit -> (b, nkv, N * C), rank-major within a row."""
    lib = load()
    N, b, nkv, C = gathered.shape
    if out is None:
        out = torch.empty((b, nkv, N * C), dtype=gathered.dtype, device=gathered.device)
    st = lib.quoka_shard_interleave(_ptr(gathered), N, b * nkv, C, _ptr(out), _stream(stream))
    _check(st, "quoka_shard_interleave")
    return out


def quoka_topk(scores, BSA, *, kv_idx=None, kv_count=None, ws=None, stream=None):
    """Step (e) alone on scores (b, nkv, T): (kv_idx (b,nkv,min(BSA,T)) int32
    ascending, kv_count (b,nkv))."""
    lib = load()
    b, nkv, T = scores.shape
    n = min(BSA, T)
    if kv_idx is None:
        kv_idx = torch.empty((b, nkv, n), dtype=torch.int32, device=scores.device)
    if kv_count is None:
        kv_count = torch.empty((b, nkv), dtype=torch.int32, device=scores.device)
    st = lib.quoka_topk(_ptr(scores), b, nkv, T, BSA, _ptr(kv_idx) if kv_idx.numel() else None,
                        _ptr(kv_count), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "quoka_topk")
    return kv_idx, kv_count


def quoka_shard_take(sel_pos, sel_count, cand_idx, rank, *, kv_idx=None, kv_count=None, ws=None, stream=None):
    """This rank's share of a selection over the concatenated candidate
    lists: (kv_idx (b,nkv,C) int32 ascending, kv_count (b,nkv))."""
    lib = load()
    b, nkv, S = sel_pos.shape
    C = cand_idx.shape[2]
    if kv_idx is None:
        kv_idx = torch.zeros((b, nkv, C), dtype=torch.int32, device=cand_idx.device)
    if kv_count is None:
        kv_count = torch.empty((b, nkv), dtype=torch.int32, device=cand_idx.device)
    st = lib.quoka_shard_take(_ptr(sel_pos) if sel_pos.numel() else None, _ptr(sel_count), b, nkv, S,
                              _ptr(cand_idx) if cand_idx.numel() else None, C, rank,
                              _ptr(kv_idx) if kv_idx.numel() else None, _ptr(kv_count), _ptr(ws),
                              0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "quoka_shard_take")
    return kv_idx, kv_count


def quoka_combine_partials(O_parts, lse_parts, *, O=None, lse=None, stream=None):
    """Merge (N, b, nq, BCP, d) partial outputs by their (N, b, nq, BCP)
    log-sum-exps: returns (O (b,nq,BCP,d), lse (b,nq,BCP))."""
    lib = load()
    N, b, nq, BCP, d = O_parts.shape
    if O is None:
        O = torch.empty((b, nq, BCP, d), dtype=O_parts.dtype, device=O_parts.device)
    if lse is None:
        lse = torch.empty((b, nq, BCP), dtype=torch.float32, device=O_parts.device)
    st = lib.quoka_combine_partials(_ptr(O_parts), _ptr(lse_parts), N, b, nq, BCP, d, _dtype_code(O_parts),
                                    _ptr(O), _ptr(lse), _stream(stream))
    _check(st, "quoka_combine_partials")
    return O, lse
