"""Host-side checks of the C ABI that need no GPU: the library builds and loads,
it exports every function include/olmo3.h declares, the host-only entry points
agree with the oracle bit for bit, and invalid arguments are rejected before
anything is launched."""
import ctypes
import os
import re

import pytest

import oracle.olmo3_oracle as O
from conftest import ROOT, read_golden
from hybrid_sliding_window_olmo3_b200 import build as B
from hybrid_sliding_window_olmo3_b200 import olmo3 as L

HEADER = os.path.join(ROOT, "include", "olmo3.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(olmo3_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_hot_path_entry_points():
    names = declared_functions()
    for n in ["olmo3_layer_types", "olmo3_qknorm_rope", "olmo3_kv_append", "olmo3_attn_prefill",
              "olmo3_attn_decode", "olmo3_attn_decode_workspace_size", "olmo3_attn_mask",
              "olmo3_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in olmo3.h but not exported by libolmo3.so"


def test_layer_types_bit_exact_vs_oracle(lib):
    for n in list(range(0, 70)):
        want = [1 if x == O.FULL else 0 for x in O.layer_types(n)]
        assert L.layer_types(n) == want
    for r in read_golden("layer_types.txt"):
        n = int(r[0])
        assert L.layer_types(n) == [1 if x == "full" else 0 for x in r[1:]]


def test_status_strings(lib):
    assert L.status_string(0) == "ok"
    for s in (-1, -2, -3, -4):
        assert L.status_string(s) != "unknown status"


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
NULL = None


def test_qknorm_rope_rejects_bad_arguments(lib):
    f = lib.olmo3_qknorm_rope
    args = [FAKE, FAKE, NULL, L.BF16, FAKE, FAKE, FAKE, FAKE, NULL, FAKE, 1, 4, 2, 1, 128, 1e-6, 5e5, NULL]
    bad_d = list(args)
    bad_d[14] = 96
    assert f(*bad_d) == L.ERR_UNSUPPORTED
    bad_dtype = list(args)
    bad_dtype[3] = 7
    assert f(*bad_dtype) == L.ERR_INVALID_ARG
    null_q = list(args)
    null_q[0] = NULL
    assert f(*null_q) == L.ERR_INVALID_ARG
    wide = list(args)
    wide[12] = 65  # H*d = 8320 > 8192
    assert f(*wide) == L.ERR_UNSUPPORTED
    neg = list(args)
    neg[11] = -1
    assert f(*neg) == L.ERR_INVALID_ARG
    empty = list(args)
    empty[11] = 0
    assert f(*empty) == L.OK  # nothing to do, nothing launched
    misaligned = list(args)
    misaligned[0] = ctypes.c_void_p(0x1002)
    assert f(*misaligned) == L.ERR_INVALID_ARG


def test_prefill_rejects_bad_arguments(lib):
    f = lib.olmo3_attn_prefill
    args = [FAKE, FAKE, FAKE, FAKE, 1, 256, 4, 2, 128, L.SLIDING, 64, 0.1, NULL, NULL, NULL]
    a = list(args); a[6] = 3                       # H % G != 0
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[8] = 256                     # d
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[9] = 2                       # layer type
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[10] = 0                      # window
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[11] = float("nan")
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[0] = NULL
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[5] = 0                       # T == 0: nothing to do
    assert f(*a) == L.OK


def _cache(**kw):
    c = dict(k=0x1000, v=0x2000, seq_base=0x3000, total_slots=64, capacity=16, layer_type=L.SLIDING,
             window=16, B=4, G=2, d=128)
    c.update(kw)
    return L.CacheStruct(c["k"], c["v"], c["seq_base"], c["total_slots"], c["capacity"], c["layer_type"],
                         c["window"], c["B"], c["G"], c["d"])


def test_cache_validation(lib):
    app = lib.olmo3_kv_append
    ok_args = lambda c: (ctypes.byref(c), FAKE, FAKE, FAKE, 1, NULL, NULL, NULL)  # noqa: E731
    assert app(*ok_args(_cache(capacity=8))) == L.ERR_INVALID_ARG      # ring must hold exactly `window`
    assert app(*ok_args(_cache(d=80))) == L.ERR_UNSUPPORTED
    assert app(*ok_args(_cache(layer_type=5))) == L.ERR_INVALID_ARG
    assert app(*ok_args(_cache(k=0))) == L.ERR_INVALID_ARG
    assert app(*ok_args(_cache(total_slots=1 << 31))) == L.ERR_UNSUPPORTED
    assert app(*ok_args(_cache(k=0x1008))) == L.ERR_INVALID_ARG         # misaligned
    c = _cache()
    assert app(ctypes.byref(c), FAKE, FAKE, FAKE, 0, NULL, NULL, NULL) == L.OK  # T == 0


def test_decode_workspace_and_validation(lib):
    ws = L.attn_decode_workspace_size
    assert ws(32, 32, 32, 128, 32769, L.FULL, 4096) > 0
    # sliding layers never need more than `window` keys, whatever the context
    assert ws(32, 32, 32, 128, 10 ** 6, L.SLIDING, 4096) == ws(32, 32, 32, 128, 4096, L.SLIDING, 4096)
    assert ws(2, 3, 2, 128, 100, L.FULL, 4096) == 0      # H % G
    assert ws(2, 4, 2, 100, 100, L.FULL, 4096) == 0      # d
    for B_, G_, n in [(1, 1, 1), (32, 32, 32769), (8, 8, 65537), (64, 32, 65536), (3, 2, 100)]:
        need = ws(B_, G_, G_, 128, n, L.FULL, 4096)
        assert need % (130 * 4) == 0 and need >= B_ * G_ * 130 * 4
    dec = lib.olmo3_attn_decode
    c = _cache(layer_type=L.FULL, capacity=16)
    # workspace too small
    assert dec(FAKE, 4, ctypes.byref(c), FAKE, 16, FAKE, NULL, 0.1, 0, FAKE, 4, NULL, NULL) == L.ERR_WORKSPACE
    # more than 16 query heads per key/value head unsupported
    assert dec(FAKE, 34, ctypes.byref(c), FAKE, 16, FAKE, NULL, 0.1, 0, FAKE, 1 << 20, NULL, NULL) == \
        L.ERR_UNSUPPORTED
    assert dec(FAKE, 4, ctypes.byref(c), FAKE, 0, FAKE, NULL, 0.1, 0, FAKE, 1 << 20, NULL, NULL) == \
        L.ERR_INVALID_ARG


def test_prefill_chunk_workspace_and_validation(lib):
    ws = L.attn_prefill_chunk_workspace_size
    assert ws(2, 100, 8, 128, L.FULL, 4096) == 0                      # full layers read the cache in place
    assert ws(2, 100, 8, 128, L.SLIDING, 4096) == 2 * 2 * 128 * 8 * 128 * 2       # ring read in place + bridge tile
    assert ws(2, 100, 8, 128, L.SLIDING, 4000) == 2 * 2 * (3999 + 100) * 8 * 128 * 2  # other windows: gathered
    assert ws(2, 100, 8, 96, L.SLIDING, 4096) == 0                    # unsupported d
    f = lib.olmo3_attn_prefill_chunk
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(L.CacheStruct), ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    c = _cache()  # sliding, window 16
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), FAKE, 8, 4, FAKE, 0.1, NULL, NULL, 0, NULL, NULL) == L.ERR_WORKSPACE
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), FAKE, 8, 3, FAKE, 0.1, NULL, FAKE, 1 << 20, NULL, NULL) == \
        L.ERR_UNSUPPORTED                                               # H % G
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), NULL, 8, 4, FAKE, 0.1, NULL, FAKE, 1 << 20, NULL, NULL) == \
        L.ERR_INVALID_ARG                                               # no pos_offset
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), FAKE, 0, 4, FAKE, 0.1, NULL, NULL, 0, NULL, NULL) == L.OK


def test_out_proj_validation(lib):
    # per-row sums of squares, one counter per 128-row block and an abort flag, in 256-byte units
    assert L.out_proj_workspace_size(8192, 4096) == (8192 * 4 + (64 + 1) * 4 + 255) // 256 * 256
    f = lib.olmo3_out_proj_postnorm_residual
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 3 + [ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t,
                                                              ctypes.c_void_p, ctypes.c_void_p]
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 16, 256, 128, 1e-6, FAKE, 1 << 20, NULL, NULL]
    a = list(args); a[7] = 100                   # K not a multiple of 64
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[6] = 250                   # D not a multiple of 8
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[10] = 16                   # workspace too small
    assert f(*a) == L.ERR_WORKSPACE
    a = list(args); a[0] = NULL
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[5] = 0                     # nothing to do
    assert f(*a) == L.OK


def test_qkv_proj_validation(lib):
    # q and k sums of squares per row, two counters per 128-row block and an abort flag
    assert L.qkv_proj_workspace_size(8192) == (8192 * 8 + (2 * 64 + 1) * 4 + 255) // 256 * 256
    assert L.qkv_proj_workspace_size(0) == 256
    f = lib.olmo3_qkv_proj_qknorm_rope
    d_ = ctypes.c_double
    f.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int] * 6 + [ctypes.c_float, d_, d_, ctypes.c_int, d_, d_,
                                                               ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                                               ctypes.c_void_p]
    #       x     w     gq    gk    q     k     v     pos   B  T   H  G  d    D    eps   theta factor oc   bf  bs
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 50, 4, 2, 128, 256, 1e-6, 5e5, 1.0, 8192, 32., 1.,
            FAKE, 1 << 20, NULL, NULL]
    a = list(args); a[12] = 96                   # head dim
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[13] = 200                  # model width not a multiple of 64
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[10], a[11] = 3, 1          # H*d not a multiple of 256
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[11], a[10] = 1, 4          # G*d = 128
    assert f(*a) == L.ERR_UNSUPPORTED
    a = list(args); a[16] = 0.5                  # YaRN factor below 1
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[15] = 0.0                  # theta
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[21] = 64                   # workspace too small
    assert f(*a) == L.ERR_WORKSPACE
    a = list(args); a[7] = NULL                  # no positions
    assert f(*a) == L.ERR_INVALID_ARG
    a = list(args); a[9] = 0                     # nothing to do
    assert f(*a) == L.OK


def test_mask_and_layer_types_reject_bad_arguments(lib):
    assert lib.olmo3_layer_types(-1, None) == L.ERR_INVALID_ARG
    assert lib.olmo3_layer_types(3, None) == L.ERR_INVALID_ARG
    assert lib.olmo3_attn_mask(4, 0, L.SLIDING, FAKE, NULL) == L.ERR_INVALID_ARG
    assert lib.olmo3_attn_mask(4, 2, 9, FAKE, NULL) == L.ERR_INVALID_ARG
    assert lib.olmo3_attn_mask(0, 2, L.SLIDING, NULL, NULL) == L.OK
