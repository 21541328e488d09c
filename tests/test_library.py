"""Host-side checks of libquoka.so that need no GPU: the library builds and
loads, exports every entry point include/quoka.h declares, and rejects bad
arguments on the host before anything is enqueued."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "quoka.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_kv_selection_quoka_b200 import build, _lib
    build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(quoka_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("quoka_select", "quoka_gather_kv", "quoka_sparse_gqa_attn", "quoka_prefill_chunk",
              "quoka_workspace_size", "quoka_get_device_status", "quoka_status_string"):
        assert n in names


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++11")])
def test_header_compiles_on_its_own(lang, std, tmp_path):
    """include/quoka.h is a plain C header (fixed-width integers, opaque
    stream pointers, no CUDA or torch types): it compiles alone as C99 and
    as C++, and a C translation unit can take the address of every
    declared function."""
    import shutil
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / ("use." + ("c" if lang == "c" else "cpp"))
    refs = "\n".join(f"  (void)&{n};" for n in declared_functions())
    src.write_text(f'#include "quoka.h"\nvoid use(void) {{\n{refs}\n}}\n')
    subprocess.run([cc, "-std=" + std, "-Wall", "-Werror", "-fsyntax-only", "-I", os.path.dirname(HEADER), str(src)],
                   check=True, capture_output=True, text=True)


def test_plain_c_program_links_and_calls_the_host_entry_points(lib, tmp_path):
    """A C program linked against libquoka.so (no Python, no torch) sizes a
    workspace, names a status, and gets a bad call turned away on the host,
    through the header alone."""
    import shutil
    from sparse_kv_selection_quoka_b200 import _lib
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / "main.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "quoka.h"
int main(void) {
  size_t n = quoka_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, QUOKA_BF16);
  size_t bad = quoka_workspace_size(1, 32, 7, 128, 32768, 512, 32, 4096, QUOKA_BF16);
  quoka_tensor q;
  memset(&q, 0, sizeof q);
  quoka_status st = quoka_select(&q, NULL, 4, 10, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("%zu %zu %d %s\n", n, bad, (int)st, quoka_status_string(st));
  return 0;
}
""")
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "main"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-L", libdir,
                    "-lquoka", "-o", str(exe)], check=True, capture_output=True, text=True)
    env = dict(os.environ, LD_LIBRARY_PATH=libdir + os.pathsep + os.environ.get("LD_LIBRARY_PATH", ""))
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, env=env).stdout.split(" ", 3)
    assert int(out[0]) == lib.quoka_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, 1) > 0
    assert int(out[1]) == 0  # nq not a multiple of nkv
    assert int(out[2]) == 1  # QUOKA_ERR_INVALID_ARG
    assert out[3].strip() == lib.quoka_status_string(1).decode()


def test_every_declared_symbol_is_exported(lib):
    from sparse_kv_selection_quoka_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (quoka_\w+)", out))
    for n in declared_functions():
        assert n in exported, f"{n} declared in quoka.h but not exported"
        assert getattr(lib, n) is not None
    assert set(_lib.EXPORTS) <= exported


def test_status_strings(lib):
    from sparse_kv_selection_quoka_b200 import _lib
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.quoka_status_string(code).decode() == name


def test_workspace_size_host_only(lib):
    n = lib.quoka_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, 1)
    # at least S_agg (b*nkv*T fp32) and the selected indices
    assert n >= 8 * 32768 * 4 + 8 * 4096 * 4
    assert lib.quoka_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, 1) % 256 == 0
    assert lib.quoka_workspace_size(1, 30, 8, 128, 100, 64, 4, 10, 1) == 0    # nq % nkv
    assert lib.quoka_workspace_size(1, 32, 8, 128, -1, 64, 4, 10, 1) == 0     # T < 0
    assert lib.quoka_workspace_size(1, 32, 8, 128, 100, 64, 4, 10, 7) == 0    # dtype


def test_workspace_parts_host_only(lib):
    # quoka_select needs only its own part; the full size adds the gathered
    # selected K and V (bf16, d = 128) of the attention
    full = lib.quoka_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, 1)
    sel = lib.quoka_select_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, 1)
    att = lib.quoka_attn_workspace_size(1, 8, 128, 4096, 1)
    gathered = 2 * 8 * 4096 * 128 * 2
    assert att == 256 + gathered
    assert full == sel + gathered
    # fp32, d = 64 and BSA_eff = 0 need no gathered copy
    assert lib.quoka_attn_workspace_size(1, 8, 128, 4096, 0) == 256
    assert lib.quoka_attn_workspace_size(1, 8, 64, 4096, 1) == 256
    assert lib.quoka_attn_workspace_size(1, 8, 128, 0, 1) == 256
    assert (lib.quoka_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, 0)
            == lib.quoka_select_workspace_size(1, 32, 8, 128, 32768, 512, 32, 4096, 0))
    # BSA beyond T is clipped to BSA_eff = T
    assert (lib.quoka_workspace_size(1, 4, 2, 128, 100, 64, 4, 1000, 1)
            == lib.quoka_select_workspace_size(1, 4, 2, 128, 100, 64, 4, 1000, 1)
            + 2 * ((2 * 100 * 128 * 2 + 255) // 256 * 256))
    assert lib.quoka_select_workspace_size(1, 30, 8, 128, 100, 64, 4, 10, 1) == 0
    assert lib.quoka_attn_workspace_size(0, 8, 128, 10, 1) == 0
    assert lib.quoka_attn_workspace_size(1, 8, 128, -1, 1) == 0
    assert lib.quoka_attn_workspace_size(1, 8, 128, 10, 7) == 0


def _view(shape, dtype=1, data=0x10000, stride=None):
    from sparse_kv_selection_quoka_b200._lib import quoka_tensor
    v = quoka_tensor()
    v.data = data
    v.dtype = dtype
    if stride is None:
        stride = [shape[1] * shape[2] * shape[3], shape[2] * shape[3], shape[3], 1]
    for i in range(4):
        v.shape[i] = shape[i]
        v.stride[i] = stride[i]
    return v


def test_workspace_size_covers_every_call_host_only(lib):
    """quoka_workspace_size is the select part, plus the gathered copy (bf16,
    d = 128), plus the partials of the attention's split key ranges when the
    query tiles fill less than half of the GPU, plus, for a short chunk
    (G * BCP <= 64), the decode attention's partials: so one workspace serves
    quoka_select, quoka_sparse_gqa_attn at its fastest, quoka_decode_attn and
    quoka_prefill_chunk."""
    al = lambda n: (n + 255) // 256 * 256

    def splits(b, nq, BCP, bsa):
        # key-range splits of the tensor-core attention: one wave of 148 CTAs
        tiles = b * nq * ((BCP + 127) // 128)
        if 2 * tiles > 148:
            return 1
        s = min(4, 148 // tiles, ((bsa + 127) // 128 + 1) // 2)
        return s if s >= 2 else 1

    cases = [  # b, nq, nkv, d, T, BCP, NQ, BSA, dtype (1 = bf16)
        (1, 32, 8, 128, 32768, 512, 32, 4096, 1),
        (1, 32, 8, 128, 32768, 1, 1, 4096, 1),
        (2, 16, 2, 128, 3000, 8, 8, 700, 1),
        (1, 6, 3, 64, 900, 3, 3, 200, 0),
        (1, 8, 2, 128, 0, 1, 1, 0, 1),
        (1, 24, 8, 128, 8192, 256, 16, 2048, 1),  # 48 query tiles: split key ranges
    ]
    for b, nq, nkv, d, T, BCP, NQ, BSA, dt in cases:
        full = lib.quoka_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, dt)
        sel = lib.quoka_select_workspace_size(b, nq, nkv, d, T, BCP, NQ, BSA, dt)
        bsa = min(BSA, T)
        att = lib.quoka_attn_workspace_size(b, nkv, d, bsa, dt)
        dec = lib.quoka_decode_workspace_size(b, nq, nkv, d, BCP, bsa, dt)
        gathered = 2 * al(b * nkv * bsa * d * 2) if (dt == 1 and d == 128 and bsa > 0) else 0
        ns = splits(b, nq, BCP, bsa) if gathered else 1
        rows = ns * b * nq * BCP
        parts = al(rows * d * 2) + al(rows * 4) if ns > 1 else 0
        short = (nq // nkv) * BCP <= 64
        assert (dec > 0) == short
        assert att == 256 + gathered
        assert full == sel + gathered + parts + (dec - 256 if short else 0)
        assert full >= max(sel, att, dec)


def test_select_rejects_bad_arguments_on_host(lib):
    Q = _view((1, 8, 64, 128))
    K = _view((1, 2, 500, 128))
    ws = ctypes.c_void_p(0x100000)
    buf = ctypes.c_void_p(0x200000)
    call = lambda q, k, NQ, BSA, wsb=1 << 30: lib.quoka_select(ctypes.byref(q), ctypes.byref(k), NQ, BSA,
                                                               buf, buf, None, None, ws, wsb, None)
    assert call(Q, K, 0, 10) == 1                      # NQ < 1
    assert call(Q, K, 65, 10) == 1                     # NQ > BCP
    assert call(Q, K, 4, -1) == 1                      # BSA < 0
    assert call(Q, _view((1, 3, 500, 128)), 4, 10) == 1           # nq % nkv
    assert call(Q, _view((1, 2, 500, 128), dtype=0), 4, 10) == 1  # dtype mismatch
    assert call(_view((1, 8, 64, 96)), _view((1, 2, 500, 96)), 4, 10) == 2  # d unsupported
    assert call(_view((1, 8, 64, 128), data=0x10004), K, 4, 10) == 1        # misaligned data
    assert call(_view((1, 8, 64, 128), stride=[8 * 64 * 128, 64 * 128, 129, 1]), K, 4, 10) == 1
    assert call(_view((1, 8, 64, 128), stride=[8 * 64 * 128, 64 * 128, 128, 2]), K, 4, 10) == 1
    assert call(Q, K, 4, 10, wsb=64) == 3              # workspace too small
    assert lib.quoka_select(ctypes.byref(Q), ctypes.byref(K), 4, 10, buf, buf, None, None,
                            ctypes.c_void_p(0x100010), 1 << 30, None) == 3  # misaligned ws
    assert lib.quoka_select(None, ctypes.byref(K), 4, 10, buf, buf, None, None, ws, 1 << 30, None) == 1


def test_attention_rejects_bad_arguments_on_host(lib):
    Q = _view((1, 8, 64, 128))
    K = _view((1, 2, 500, 128))
    Kc = _view((1, 2, 64, 128))
    buf = ctypes.c_void_p(0x200000)
    ws = ctypes.c_void_p(0x100000)
    f = lib.quoka_sparse_gqa_attn
    B = ctypes.byref
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(_view((1, 2, 63, 128))), B(Kc), 0.1, buf, None, ws, 256, None) == 1
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), -1.0, buf, None, ws, 256, None) == 1
    assert f(B(Q), B(K), B(K), buf, buf, -1, B(Kc), B(Kc), 0.1, buf, None, ws, 256, None) == 1
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), 0.1, None, None, ws, 256, None) == 1
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), 0.1, buf, None, None, 256, None) == 3
    g = lib.quoka_prefill_chunk
    assert g(B(Q), B(K), B(K), B(Kc), B(Kc), 4, 10, 0.1, buf, None, None, ws, 16, None) == 3
    assert g(B(Q), B(K), B(K), B(Kc), B(Kc), 0, 10, 0.1, buf, None, None, ws, 1 << 30, None) == 1


def test_decode_attention_rejects_bad_arguments_on_host(lib):
    f = lib.quoka_decode_attn
    B = ctypes.byref
    buf = ctypes.c_void_p(0x200000)
    ws = ctypes.c_void_p(0x100000)
    K = _view((1, 2, 500, 128))
    # G * BCP = 4 * 17 = 68 query rows per KV head: not a short chunk
    Q, Kc = _view((1, 8, 17, 128)), _view((1, 2, 17, 128))
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), 0.1, buf, None, ws, 1 << 30, None) == 2
    # G * BCP = 64: accepted shapes, but a workspace one byte short, or misaligned
    Q, Kc = _view((1, 8, 16, 128)), _view((1, 2, 16, 128))
    need = lib.quoka_decode_workspace_size(1, 8, 2, 128, 16, 10, 0)
    assert need > 256
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), 0.1, buf, None, ws, need - 1, None) == 3
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), 0.1, buf, None, ctypes.c_void_p(0x100010), need,
             None) == 3
    assert f(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), -1.0, buf, None, ws, need, None) == 1
    assert f(B(Q), B(K), B(K), None, buf, 10, B(Kc), B(Kc), 0.1, buf, None, ws, need, None) == 1
    assert lib.quoka_decode_workspace_size(1, 8, 2, 96, 1, 10, 0) == 0  # d = 96


def test_select_variants_reject_bad_arguments_on_host(lib):
    """quoka_select_ex's unknown flag bits, and quoka_select_static's shapes
    with no valid workspace or one past its fixed scratch array, are turned
    away before any device call."""
    Q = _view((1, 8, 64, 128))
    K = _view((1, 2, 500, 128))
    buf = ctypes.c_void_p(0x200000)
    ws = ctypes.c_void_p(0x100000)
    B = ctypes.byref
    for flags in (2, 4, 0x80000000):
        assert lib.quoka_select_ex(B(Q), B(K), 4, 10, buf, buf, None, None, flags, ws, 1 << 30, None) == 1
    st = lib.quoka_select_static
    assert st(None, B(K), 4, 10, buf, buf, None, None, None) == 1
    assert st(B(Q), B(K), 0, 10, buf, buf, None, None, None) == 1                    # NQ < 1
    assert st(B(Q), B(_view((1, 3, 500, 128))), 4, 10, buf, buf, None, None, None) == 1  # nq % nkv
    # S_agg alone of (1, 8, 2^20) keys is 32 MiB: past the 8 MiB array
    Kbig = _view((1, 8, 1 << 20, 128))
    need = lib.quoka_select_workspace_size(1, 32, 8, 128, 1 << 20, 512, 32, 4096, 1)
    assert need > (8 << 20)
    assert st(B(_view((1, 32, 512, 128))), B(Kbig), 32, 4096, buf, buf, None, None, None) == 3


def test_gather_and_gathered_attention_reject_bad_arguments_on_host(lib):
    K = _view((1, 2, 500, 128))
    buf = ctypes.c_void_p(0x200000)
    ws = ctypes.c_void_p(0x100000)
    B = ctypes.byref
    g = lib.quoka_gather_kv
    assert g(None, B(K), buf, buf, 10, buf, buf, None, 0, None) == 1
    assert g(B(K), B(K), None, None, 10, buf, buf, None, 0, None) == 1              # no kv_count
    assert g(B(K), B(K), buf, buf, -1, buf, buf, None, 0, None) == 1                # BSA_eff < 0
    assert g(B(K), B(_view((1, 2, 500, 128), dtype=0)), buf, buf, 10, buf, buf, None, 0, None) == 1  # V dtype
    assert g(B(K), B(K), buf, buf, 10, None, buf, None, 0, None) == 1               # no Ksel
    assert g(B(K), B(K), buf, buf, 10, ctypes.c_void_p(0x200008), buf, None, 0, None) == 1  # Ksel misaligned
    assert g(B(_view((1, 2, 500, 96))), B(_view((1, 2, 500, 96))), buf, buf, 10, buf, buf, None, 0, None) == 2
    assert g(B(K), B(K), buf, buf, 10, buf, buf, ctypes.c_void_p(0x100010), 256, None) == 3  # ws misaligned
    assert g(B(K), B(K), buf, buf, 10, buf, buf, ws, 4, None) == 3                  # ws under the status words
    Q = _view((1, 8, 64, 128))
    Ks = _view((1, 2, 10, 128))
    Kc = _view((1, 2, 64, 128))
    a = lib.quoka_sparse_gqa_attn_gathered
    assert a(B(Q), B(Ks), B(Ks), None, B(Kc), B(Kc), 0.1, buf, None, ws, 256, None) == 1     # no kv_count
    assert a(B(Q), B(Ks), B(Ks), buf, B(Kc), B(Kc), 0.1, None, None, ws, 256, None) == 1     # no O
    assert a(B(Q), B(Ks), B(Ks), buf, B(Kc), B(Kc), 0.1, ctypes.c_void_p(0x200004), None, ws, 256,
             None) == 1                                                                      # O misaligned
    assert a(B(Q), B(Ks), B(Ks), buf, B(Kc), B(Kc), 0.0, buf, None, ws, 256, None) == 1      # scale <= 0
    assert a(B(Q), B(Ks), B(Ks), buf, B(Kc), B(Kc), float("nan"), buf, None, ws, 256, None) == 1
    assert a(B(Q), B(Ks), B(Ks), buf, B(_view((1, 2, 63, 128))), B(Kc), 0.1, buf, None, ws, 256, None) == 1
    assert a(B(Q), B(Ks), B(Ks), buf, B(Kc), B(Kc), 0.1, buf, None, None, 256, None) == 3
    assert a(B(Q), B(Ks), B(Ks), buf, B(Kc), B(Kc), 0.1, buf, None, ctypes.c_void_p(0x100010), 256, None) == 3
    assert a(B(Q), B(Ks), B(Ks), buf, B(Kc), B(Kc), 0.1, buf, None, ws, 255, None) == 3
    e = lib.quoka_sparse_gqa_attn_ex
    for flags in (2, 0x100):
        assert e(B(Q), B(K), B(K), buf, buf, 10, B(Kc), B(Kc), 0.1, buf, None, flags, ws, 1 << 30, None) == 1


def test_context_parallel_calls_reject_bad_arguments_on_host(lib):
    buf = ctypes.c_void_p(0x200000)
    odd = ctypes.c_void_p(0x200002)
    cs = lib.quoka_shard_candidate_scores
    assert cs(buf, 0, 2, 500, buf, buf, 10, 20, buf, buf, None, 0, None) == 1       # b < 1
    assert cs(buf, 1, 2, 500, buf, buf, 10, 5, buf, buf, None, 0, None) == 1        # C < Cl
    assert cs(buf, 1, 2, 500, buf, None, 10, 20, buf, buf, None, 0, None) == 1      # no kv_count
    assert cs(buf, 1, 2, 500, buf, buf, 10, 20, None, buf, None, 0, None) == 1      # no scores out
    assert cs(buf, 1, 2, 500, buf, buf, 10, 0, buf, buf, None, 0, None) == 1        # C = 0 < Cl
    assert cs(None, 1, 2, 500, None, buf, 0, 0, None, None, None, 0, None) == 0     # empty: nothing to do
    il = lib.quoka_shard_interleave
    assert il(buf, 0, 4, 4, buf, None) == 1                                          # N < 1
    assert il(buf, 2, -1, 4, buf, None) == 1
    assert il(odd, 2, 4, 4, buf, None) == 1                                          # not 4-byte aligned
    assert il(None, 2, 0, 4, None, None) == 0                                        # empty
    tk = lib.quoka_topk
    assert tk(buf, 1, 2, 500, -1, buf, buf, None, 0, None) == 1                      # BSA < 0
    assert tk(buf, 1, 2, 500, 10, buf, None, None, 0, None) == 1                     # no kv_count
    assert tk(None, 1, 2, 500, 10, buf, buf, None, 0, None) == 1                     # no scores
    assert tk(buf, 1, 70000, 500, 10, buf, buf, None, 0, None) == 1                  # nkv past the grid
    tkn = lib.quoka_shard_take
    assert tkn(buf, buf, 1, 2, 8, buf, 10, -1, buf, buf, None, 0, None) == 1         # rank < 0
    assert tkn(buf, None, 1, 2, 8, buf, 10, 0, buf, buf, None, 0, None) == 1         # no sel_count
    assert tkn(None, buf, 1, 2, 8, buf, 10, 0, buf, buf, None, 0, None) == 1         # S > 0 without sel_pos
    cp = lib.quoka_combine_partials
    assert cp(buf, buf, 2, 1, 8, 64, 96, 1, buf, None, None) == 1                    # d not 64 / 128
    assert cp(buf, buf, 2, 1, 8, 64, 128, 7, buf, None, None) == 1                   # dtype
    assert cp(buf, buf, 0, 1, 8, 64, 128, 1, buf, None, None) == 1                   # N < 1
    assert cp(ctypes.c_void_p(0x200008), buf, 2, 1, 8, 64, 128, 1, buf, None, None) == 1  # misaligned
    assert cp(buf, None, 2, 1, 8, 64, 128, 1, buf, None, None) == 1                  # no lse_parts


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from sparse_kv_selection_quoka_b200 import _lib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load()
