"""CPU checks of the C ABI: the library loads, exports every function include/sepattn.h declares,
and rejects bad arguments on the host before any launch (no GPU needed for these paths)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sepattn.h")
LIB = os.path.join(ROOT, "kv_cache_compression_sep_b200", "libsepattn.so")

SEP_OK, SEP_ERR_INVALID_ARG, SEP_ERR_UNSUPPORTED, SEP_ERR_MISALIGNED = 0, 1, 2, 3
SEP_ERR_WORKSPACE = 6


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from kv_cache_compression_sep_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:int|size_t|const char\*)\s+(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_five_calls():
    names = declared_functions()
    for n in ("sep_mask_build", "sep_attn_fwd", "sep_attn_bwd", "sepcache_update",
              "sepcache_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    f = lib.sep_status_string
    f.restype = ctypes.c_char_p
    f.argtypes = [ctypes.c_int]
    assert f(0) == b"ok"
    assert b"timed out" in f(5)
    assert f(99) == b"unknown status"


def test_mask_build_rejects_bad_arguments(lib):
    f = lib.sep_mask_build
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    good = P(16)
    # null output pointer
    assert f(good, 1, 8, 0, 1, 128, 128, good, good, None, good, good, None, None) == SEP_ERR_INVALID_ARG
    # non-positive sizes, negative a, n < 1
    for B, L, a, n in ((0, 8, 0, 1), (1, 0, 0, 1), (1, 8, -1, 1), (1, 8, 0, 0)):
        assert f(good, B, L, a, n, 128, 128, good, good, good, good, good, None, None) == SEP_ERR_INVALID_ARG


class _SepMask(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("L", ctypes.c_int), ("a", ctypes.c_int), ("n", ctypes.c_int),
                ("sep", ctypes.c_void_p), ("anchor_idx", ctypes.c_void_p),
                ("anchor_cnt", ctypes.c_void_p), ("anchor_bits", ctypes.c_void_p),
                ("gather_end", ctypes.c_void_p), ("tile_map", ctypes.c_void_p)]


def _fwd(lib, q=256, B=1, L=128, Hq=4, Hkv=2, d=64, a=4, n=64, mask=None, o=256, ws=4096,
         ws_bytes=1 << 30):
    f = lib.sep_attn_fwd
    f.restype = ctypes.c_int
    m = mask if mask is not None else _SepMask(B, L, a, n, 16, 16, 16, 16, 16, 16)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    return f(P(q), P(256), P(256), I(B), I(L), I(Hq), I(Hkv), I(d), F(0.125), I(a), I(n),
             ctypes.byref(m), P(o), P(256), P(ws), ctypes.c_size_t(ws_bytes), None)


def test_attention_rejects_bad_arguments(lib):
    assert _fwd(lib, Hq=3, Hkv=2) == SEP_ERR_INVALID_ARG          # Hq % Hkv != 0
    assert _fwd(lib, d=96) == SEP_ERR_UNSUPPORTED                 # head dim
    assert _fwd(lib, q=258) == SEP_ERR_MISALIGNED                 # 16-byte alignment
    assert _fwd(lib, o=264) == SEP_ERR_MISALIGNED
    bad = _SepMask(1, 64, 4, 64, 16, 16, 16, 16, 16, 16)          # mask built for another L
    assert _fwd(lib, mask=bad) == SEP_ERR_INVALID_ARG
    assert _fwd(lib, ws_bytes=16) == SEP_ERR_WORKSPACE
    assert _fwd(lib, ws=4100) == SEP_ERR_MISALIGNED               # workspace 256-byte aligned


def test_workspace_sizes_grow_with_shape(lib):
    fw = lib.sep_attn_fwd_workspace_size
    bw = lib.sep_attn_bwd_workspace_size
    fw.restype = bw.restype = ctypes.c_size_t
    assert fw(1, 128, 1, 64) > 0
    assert fw(2, 256, 2, 128) > fw(1, 128, 1, 64)
    assert bw(1, 2048, 12, 12, 64) > fw(1, 2048, 12, 64)
    assert fw(0, 128, 1, 64) == 0


class _CacheState(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("a", ctypes.c_int32), ("s", ctypes.c_int32),
                ("w", ctypes.c_int32), ("c", ctypes.c_int32),
                ("original_positions", ctypes.c_int32), ("rope_theta", ctypes.c_float),
                ("k_slots", ctypes.c_void_p), ("v_slots", ctypes.c_void_p),
                ("slot_pos", ctypes.c_void_p), ("slot_sep", ctypes.c_void_p),
                ("meta", ctypes.c_void_p), ("rope_freq", ctypes.c_void_p)]


def test_cache_rejects_bad_state(lib):
    f = lib.sepcache_update
    f.restype = ctypes.c_int
    P = ctypes.c_void_p

    def st(**kw):
        base = dict(S=2, Hq=8, Hkv=2, d=128, a=4, s=8, w=16, rope_theta=1e4, k_slots=256,
                    v_slots=256, slot_pos=256, slot_sep=256, meta=256, rope_freq=256)
        base.update(kw)
        return _CacheState(**base)

    assert f(None, P(256), P(256), P(256), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st(w=0)), P(256), P(256), P(256), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st(Hq=6, Hkv=4)), P(256), P(256), P(256), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st(Hq=24, Hkv=2)), P(256), P(256), P(256), None) == SEP_ERR_UNSUPPORTED
    assert f(ctypes.byref(st(d=96)), P(256), P(256), P(256), None) == SEP_ERR_UNSUPPORTED
    assert f(ctypes.byref(st(k_slots=258)), P(256), P(256), P(256), None) == SEP_ERR_MISALIGNED
    assert f(ctypes.byref(st(rope_theta=0.0)), P(256), P(256), P(256), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st()), P(258), P(256), P(256), None) == SEP_ERR_MISALIGNED
    # Past Window threshold: 0 or above a + s + w
    assert f(ctypes.byref(st(c=28)), P(256), P(256), P(256), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st(c=-1)), P(256), P(256), P(256), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st(c=20000, s=5000)), P(256), P(256), P(256), None) == SEP_ERR_UNSUPPORTED


def test_prefill_rejects_bad_arguments(lib):
    f = lib.sepcache_prefill
    f.restype = ctypes.c_int
    P, I = ctypes.c_void_p, ctypes.c_int
    st = _CacheState(S=2, Hq=8, Hkv=2, d=128, a=4, s=8, w=16, rope_theta=1e4, k_slots=256,
                     v_slots=256, slot_pos=256, slot_sep=256, meta=256, rope_freq=256)
    assert f(ctypes.byref(st), P(256), P(256), P(256), I(0), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st), None, P(256), P(256), I(8), None) == SEP_ERR_INVALID_ARG
    assert f(ctypes.byref(st), P(264), P(256), P(256), I(8), None) == SEP_ERR_MISALIGNED
    big = _CacheState(S=2, Hq=8, Hkv=2, d=128, a=4, s=20000, w=16, rope_theta=1e4, k_slots=256,
                      v_slots=256, slot_pos=256, slot_sep=256, meta=256, rope_freq=256)
    assert f(ctypes.byref(big), P(256), P(256), P(256), I(8), None) == SEP_ERR_UNSUPPORTED
