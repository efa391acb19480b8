"""C-ABI checks that need no GPU: the library builds for sm_100a, loads, exports
every entry point include/bi.h declares, and rejects bad arguments on the host
(returning the right status and launching nothing)."""
import ctypes
import os
import re

import pytest

import invariant_deterministic_04_b200 as bi
from invariant_deterministic_04_b200._build import build_library

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bi.h")

OK, NULL, SHAPE, ALIGN, WS, UNSUP = 0, 1, 2, 3, 4, 5
P = 0x10000  # 16-byte aligned stand-in address; host validation never dereferences it


@pytest.fixture(scope="module")
def L():
    build_library()
    return bi.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bi_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("bi_rmsnorm", "bi_matmul", "bi_attention_decode", "bi_attention_prefill", "bi_lmhead_argmax",
              "bi_attention_workspace_size", "bi_lmhead_workspace_size", "bi_get_device_error", "bi_kv_append"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert L.bi_status_string(0) == b"BI_OK"
    assert L.bi_status_string(4) == b"BI_ERR_WORKSPACE"
    assert L.bi_status_string(99) == b"BI_ERR_UNKNOWN"
    assert L.bi_version() == 4


def test_rmsnorm_validation(L):
    f = L.bi_rmsnorm
    assert f(None, 512, P, P, 512, 4, 512, 1e-6, None) == NULL
    assert f(P, 512, P, P, 512, -1, 512, 1e-6, None) == SHAPE
    assert f(P, 512, P, P, 512, 4, 500, 1e-6, None) == SHAPE        # K % 8
    assert f(P, 256, P, P, 512, 4, 512, 1e-6, None) == SHAPE        # ldx < K
    assert f(P, 512, P, P, 512, 4, 512, float("nan"), None) == SHAPE
    assert f(P, 32768, P, P, 32768, 4, 32768, 1e-6, None) == UNSUP
    assert f(P + 2, 512, P, P, 512, 4, 512, 1e-6, None) == ALIGN
    assert f(P, 516, P, P, 512, 4, 512, 1e-6, None) == ALIGN        # ld % 8
    assert f(P, 512, P, P, 512, 0, 512, 1e-6, None) == OK           # empty: no-op
    # partially overlapping input and output rows are rejected (exact aliasing is allowed)
    assert f(P, 512, P + 0x100000, P + 16, 512, 4, 512, 1e-6, None) == SHAPE
    # in place needs the same row stride on both sides
    assert f(P, 512, P + 0x100000, P, 1024, 4, 512, 1e-6, None) == SHAPE


def test_matmul_validation(L):
    f = L.bi_matmul
    assert f(P, 512, None, 512, P, 64, 4, 64, 512, None) == NULL
    assert f(P, 500, P, 500, P, 64, 4, 64, 500, None) == SHAPE      # K % 64
    assert f(P, 512, P, 512, P, 64, 4, 60, 512, None) == SHAPE      # N % 8
    assert f(P, 512, P, 512, P, 64, 4, 64, 0, None) == SHAPE        # K == 0
    assert f(P, 256, P, 512, P, 64, 4, 64, 512, None) == SHAPE      # lda < K
    assert f(P, 512, P + 8, 512, P, 64, 4, 64, 512, None) == ALIGN
    assert f(P, 512, P, 516, P, 64, 4, 64, 512, None) == ALIGN      # ldw % 8
    assert f(P, 512, P, 512, P, 64, 0, 64, 512, None) == OK         # M == 0
    assert f(P, 512, P, 512, P, 64, 4, 0, 512, None) == OK          # N == 0
    # output overlapping an operand
    assert f(P, 512, P + 0x1000000, 512, P + 64, 64, 4, 64, 512, None) == SHAPE


def test_matmul_multi_validation(L):
    f = L.bi_matmul_multi
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int, P, P, P, P, P, ctypes.c_int64, ctypes.c_int64, P]

    def arrays(ws, ldws, cs, ldcs, ns):
        n = len(ws)
        return ((P * n)(*ws), (ctypes.c_int64 * n)(*ldws), (P * n)(*cs), (ctypes.c_int64 * n)(*ldcs),
                (ctypes.c_int64 * n)(*ns))

    a, w0, w1, c0, c1 = 0x10000, 0x200000, 0x400000, 0x600000, 0x800000
    ok = arrays([w0, w1], [64, 64], [c0, c1], [128, 256], [128, 256])
    assert f(None, 64, 2, *ok, 4, 64, None) == 1                      # null A
    assert f(a, 64, 2, None, ok[1], ok[2], ok[3], ok[4], 4, 64, None) == 1  # null array
    assert f(a, 64, 2, *arrays([w0, 0], [64, 64], [c0, c1], [128, 256], [128, 256]), 4, 64, None) == 1
    assert f(a, 64, 0, *ok, 4, 64, None) == 2                         # count 0
    assert f(a, 64, 4, *arrays([w0] * 4, [64] * 4, [c0] * 4, [128] * 4, [128] * 4), 4, 64, None) == 2
    assert f(a, 96, 2, *ok, 4, 96, None) == 2                         # K % 64
    assert f(a, 64, 2, *arrays([w0, w1], [64, 64], [c0, c1], [128, 256], [128, 12]), 4, 64, None) == 2  # N % 8
    assert f(a, 64, 2, *arrays([w0, w1], [64, 64], [c0, c1], [128, 100], [128, 256]), 4, 64, None) == 2  # ldc < N
    assert f(a + 8, 64, 2, *ok, 4, 64, None) == 3                     # A not 16-byte aligned
    assert f(a, 64, 2, *arrays([w0, w1 + 2], [64, 64], [c0, c1], [128, 256], [128, 256]), 4, 64, None) == 3
    # outputs overlapping A, a weight, or each other
    assert f(a, 64, 2, *arrays([w0, w1], [64, 64], [a, c1], [128, 256], [128, 256]), 4, 64, None) == 2
    assert f(a, 64, 2, *arrays([w0, w1], [64, 64], [c0, w1], [128, 256], [128, 256]), 4, 64, None) == 2
    assert f(a, 64, 2, *arrays([w0, w1], [64, 64], [c0, c0 + 64], [128, 256], [128, 256]), 4, 64, None) == 2
    # column ranges of one wider output (row stride 256) that share columns 120..127
    assert f(a, 64, 2, *arrays([w0, w1], [64, 64], [c0, c0 + 2 * 120], [256, 256], [128, 128]), 4, 64, None) == 2
    # M == 0, or every N == 0: nothing to launch (no device needed)
    assert f(a, 64, 2, *ok, 0, 64, None) == 0
    assert f(a, 64, 2, *arrays([w0, w1], [64, 64], [c0, c1], [128, 256], [0, 0]), 4, 64, None) == 0


def test_attention_workspace_size(L):
    s = L.bi_attention_workspace_size
    assert s(0, 32, 128, 2048) > 0
    a, b = s(4, 32, 128, 2048), s(8, 32, 128, 2048)
    assert b > a
    # 128 splits of 256 tokens for 32768 tokens; fp32 o[D] + (m, l) per split and head
    assert s(1, 32, 128, 2048) >= 128 * 32 * (128 * 4 + 8)
    assert s(-1, 32, 128, 16) == 0 and s(4, 0, 128, 16) == 0


def test_attention_validation(L):
    d = L.bi_attention_decode
    ws = L.bi_attention_workspace_size(4, 32, 128, 64)
    args = lambda **k: [k.get("q", P), P, P, k.get("np", 100), P, k.get("maxp", 64), P, P, k.get("B", 4),
                        k.get("Hq", 32), k.get("Hkv", 8), k.get("D", 128), k.get("scale", 0.088),
                        k.get("ws", P), k.get("wsb", ws), None]
    assert d(*args(q=None)) == NULL
    assert d(*args(B=-1)) == SHAPE
    assert d(*args(Hq=30)) == SHAPE                  # Hq % Hkv
    assert d(*args(D=96)) == UNSUP
    assert d(*args(Hq=48, Hkv=3)) == UNSUP           # group 16
    assert d(*args(wsb=ws - 1)) == WS
    assert d(*args(ws=None)) == WS
    assert d(*args(q=P + 4)) == ALIGN
    assert d(*args(np=0)) == SHAPE
    assert d(*args(scale=float("inf"))) == SHAPE
    assert d(*args(B=0, ws=None, wsb=0)) == OK
    p = L.bi_attention_prefill
    wsp = L.bi_attention_workspace_size(10, 32, 64, 8)
    assert p(P, 2048, None, P, P, P, 100, P, 2, 8, P, 10, 32, 8, 64, 0.125, P, wsp, None) == NULL
    assert p(P, 2048, P, P, P, P, 100, P, 0, 8, P, 10, 32, 8, 64, 0.125, P, wsp, None) == SHAPE
    assert p(P, 2048, P, P, P, P, 100, P, 2, 8, P, 10, 32, 8, 64, 0.125, P, wsp - 256, None) == WS
    assert p(P, 1024, P, P, P, P, 100, P, 2, 8, P, 10, 32, 8, 64, 0.125, P, wsp, None) == SHAPE   # ldq < Hq*D
    assert p(P, 3076, P, P, P, P, 100, P, 2, 8, P, 10, 32, 8, 64, 0.125, P, wsp, None) == ALIGN   # ldq % 8
    assert p(P, 2048, P, P, P, P, 100, P, 2, 8, P, 0, 32, 8, 64, 0.125, None, 0, None) == OK


def test_kv_append_validation(L):
    f = L.bi_kv_append
    assert f(None, P, 1024, P, P, P, P, 10, P, 1, 4, 3, 8, 128, None) == NULL
    assert f(P, P, 1024, P, P, P, P, 10, P, 1, 4, -3, 8, 128, None) == SHAPE
    assert f(P, P, 1024, P, P, P, P, 10, P, 1, 4, 3, 8, 100, None) == UNSUP
    assert f(P + 8, P, 1024, P, P, P, P, 10, P, 1, 4, 3, 8, 128, None) == ALIGN
    assert f(P, P, 512, P, P, P, P, 10, P, 1, 4, 3, 8, 128, None) == SHAPE     # ld_new < Hkv*D
    assert f(P, P, 1028, P, P, P, P, 10, P, 1, 4, 3, 8, 128, None) == ALIGN    # ld_new % 8
    assert f(P, P, 1024, P, P, P, P, 10, P, 1, 4, 0, 8, 128, None) == OK


def test_glue_validation(L):
    assert L.bi_gather_rows(None, 2048, 10, P, 4, 2048, P, 2048, None) == NULL
    assert L.bi_gather_rows(P, 2048, 10, P, 4, 2044, P, 2048, None) == SHAPE    # width % 8
    assert L.bi_gather_rows(P, 2048, 0, P, 4, 2048, P, 2048, None) == SHAPE
    assert L.bi_gather_rows(P + 2, 2048, 10, P, 4, 2048, P, 2048, None) == ALIGN
    assert L.bi_gather_rows(P, 2048, 10, P, 0, 2048, P, 2048, None) == OK
    assert L.bi_rope(None, 2048, 4, 32, 64, P, P, 384, None) == NULL
    assert L.bi_rope(P, 2048, 4, 32, 63, P, P, 384, None) == SHAPE              # odd D
    assert L.bi_rope(P, 1024, 4, 32, 64, P, P, 384, None) == SHAPE              # ldx < H*D
    assert L.bi_rope(P, 2048, 0, 32, 64, P, P, 384, None) == OK
    assert L.bi_rope(P, 2, 2**31, 1, 2, P, P, 384, None) == SHAPE             # T beyond int32
    assert L.bi_swiglu(P, 16384, None, 8192, 4, 8192, None) == NULL
    assert L.bi_swiglu(P, 16000, P, 8192, 4, 8192, None) == SHAPE               # ld_gu < 2F
    assert L.bi_swiglu(P, 16384, P, 8192, 4, 8190, None) == SHAPE               # F % 8
    assert L.bi_swiglu(P + 4, 16384, P, 8192, 4, 8192, None) == ALIGN
    assert L.bi_swiglu(P, 16384, P, 8192, 0, 8192, None) == OK
    assert L.bi_add(P, None, P, 64, None) == NULL
    assert L.bi_add(P, P, P, 63, None) == SHAPE
    assert L.bi_add(P, P + 8, P, 64, None) == ALIGN
    assert L.bi_add(P, P, P, 0, None) == OK


def test_lmhead_validation(L):
    f = L.bi_lmhead_argmax
    ws = L.bi_lmhead_workspace_size(4, 32000)
    assert ws >= 4 * 32000 * 6
    assert f(None, 2048, P, 4, 32000, 2048, 0.5, P, P, None, P, ws, None) == NULL
    assert f(P, 2048, P, 4, 32004, 2048, 0.5, P, P, None, P, ws, None) == SHAPE   # V % 8
    assert f(P, 2048, P, 4, 32000, 2000, 0.5, P, P, None, P, ws, None) == SHAPE   # K % 64
    assert f(P, 2048, P, 4, 32000, 2048, float("nan"), P, P, None, P, ws, None) == SHAPE
    assert f(P, 2048, P, 4, 32000, 2048, 0.5, P, P, None, P, ws - 1, None) == WS
    assert f(P, 2048, P, 4, 32000, 2048, 0.5, P, P, None, None, ws, None) == WS
    assert f(P, 2048, P, 4, 32000, 2048, 0.5, P, P, P + 4, P, ws, None) == ALIGN
    assert f(P, 2048, P, 0, 32000, 2048, 0.5, P, P, None, None, 0, None) == OK


def test_reduction_and_sampling_validation(L):
    Y = P + (1 << 30)  # a second, non-overlapping stand-in address
    ls, tl, mean, uni, smp = (L.bi_log_softmax, L.bi_token_logprob, L.bi_row_mean, L.bi_sampling_uniforms,
                              L.bi_sample)
    assert ls(None, 32000, Y, 32000, 4, 32000, None) == NULL
    assert ls(P, 32000, Y, 32000, 4, 31999, None) == SHAPE          # N % 8
    assert ls(P, 32000, Y, 32000, 4, 0, None) == SHAPE
    assert ls(P, 32000, Y, 32000, 4, (1 << 24) + 8, None) == SHAPE  # N > 2^24
    assert ls(P, 16000, Y, 32000, 4, 32000, None) == SHAPE          # ldx < N
    assert ls(P, 32000, Y, 16000, 4, 32000, None) == SHAPE          # ldy < N
    assert ls(P, 32000, P + 8, 32000, 4, 32000, None) == ALIGN      # y not 16-byte aligned
    assert ls(P, 32000, Y, 32002, 4, 32000, None) == ALIGN          # ldy % 4
    assert ls(P, 32004, Y, 32000, 4, 32000, None) == ALIGN          # ldx % 8
    assert ls(P, 32000, P + 64, 32000, 4, 32000, None) == SHAPE     # y overlaps x
    assert ls(P, 32000, Y, 32000, 0, 32000, None) == OK
    assert tl(P, 32000, None, Y, 4, 32000, None) == NULL
    assert tl(P, 32000, P, Y, -1, 32000, None) == SHAPE
    assert tl(P, 32000, P, Y, 0, 32000, None) == OK
    assert mean(P, 4096, None, 4, 4096, None) == NULL
    assert mean(P + 2, 4096, Y, 4, 4096, None) == ALIGN
    assert mean(P, 4096, Y, 4, 4100, None) == SHAPE                 # ldx < K
    assert mean(P, 4096, Y, 0, 4096, None) == OK
    assert uni(None, P, Y, 32000, 4, 32000, None) == NULL
    assert uni(P, P, Y, 32000, 4, 31996, None) == SHAPE             # V % 8
    assert uni(P, P, Y + 4, 32000, 4, 32000, None) == ALIGN
    assert uni(P, P, Y, 32000, 0, 32000, None) == OK
    assert smp(P, 32000, P, P, 0.8, None, 4, 32000, None) == NULL
    for t in (0.0, -1.0, float("inf"), float("nan"), 1e-45):        # T <= 0, not finite, 1/T overflows
        assert smp(P, 32000, P, P, t, Y, 4, 32000, None) == SHAPE, t
    assert smp(P, 32000, P, P, 0.8, Y, 4, 32004, None) == SHAPE     # ld < V
    assert smp(P, 32000, P, P, 0.8, Y, 0, 32000, None) == OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib

    mod = importlib.import_module("invariant_deterministic_04_b200")
    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "_load_error", None)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mod.lib()


def test_selftest_validation(L):
    assert L.bi_selftest_wait_timeout(0, None) == SHAPE
    assert L.bi_selftest_wait_timeout(2001, None) == SHAPE


def test_prefill_tc_validation(L):
    f = L.bi_attention_prefill_tc
    assert f(None, 4096, 0, 0, 100, P, P, 100, P, 1, 256, P, 32, 8, 128, 0.088, None) == NULL
    assert f(P, 4096, 1, 0, 100, P, P, 100, P, 1, 256, P, 32, 8, 128, 0.088, None) == SHAPE    # seq out of range
    assert f(P, 4096, 0, 4000, 100, P, P, 100, P, 1, 256, P, 32, 8, 128, 0.088, None) == SHAPE  # past the table
    assert f(P, 4096, 0, 0, 100, P, P, 100, P, 1, 256, P, 32, 8, 96, 0.088, None) == UNSUP
    assert f(P, 1536, 0, 0, 100, P, P, 100, P, 1, 256, P, 12, 4, 128, 0.088, None) == UNSUP  # odd group (3)
    assert f(P, 4096, 0, 0, 100, P, P, 100, P, 1, 256, P, 32, 8, 128, 0.0, None) == SHAPE     # scale <= 0
    assert f(P, 4100, 0, 0, 100, P, P, 100, P, 1, 256, P, 32, 8, 128, 0.088, None) == ALIGN
    assert f(P, 4096, 0, 0, 0, P, P, 100, P, 1, 256, P, 32, 8, 128, 0.088, None) == OK
    # 2^23 row blocks x 256 head pairs: the 32-bit work list would overflow
    assert f(P, 32768, 0, 0, 2**30, P, P, 100, P, 1, 2**26, P, 512, 256, 64, 0.125, None) == SHAPE
