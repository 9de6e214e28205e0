"""sep_attn_fwd_noalloc: the forward through the library's fixed device scratch.

Collected last (file name) so that it also runs after every other test in one process. The GPU
tests compare two calls in a row against the workspace entry point sep_attn_fwd on the same
inputs: the kernels are the same and deterministic, so the outputs must be bit-identical (the
forward tolerances are checked as well, for a readable message); the CPU test checks that an
oversized problem is refused on the host before any device work.
"""

import ctypes
import os
import re

import numpy as np
import pytest

from gpu_common import LSE_ABS, O_MAX_ABS, O_MEAN_ABS, f64

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sepattn.h")
LIB = os.path.join(ROOT, "kv_cache_compression_sep_b200", "libsepattn.so")
SEP_ERR_SCRATCH_LIMIT = 7


def _scratch_bytes():
    m = re.search(r"#define\s+SEP_NOALLOC_SCRATCH_BYTES\s+\((\d+)u \* (\d+)u \* (\d+)u\)",
                  open(HEADER).read())
    return int(m.group(1)) * int(m.group(2)) * int(m.group(3))


class _SepMask(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("L", ctypes.c_int), ("a", ctypes.c_int), ("n", ctypes.c_int),
                ("sep", ctypes.c_void_p), ("anchor_idx", ctypes.c_void_p),
                ("anchor_cnt", ctypes.c_void_p), ("anchor_bits", ctypes.c_void_p),
                ("gather_end", ctypes.c_void_p), ("tile_map", ctypes.c_void_p)]


def test_oversized_problem_is_refused_on_the_host():
    if not os.path.exists(LIB):
        from kv_cache_compression_sep_b200 import build
        build.build()
    lib = ctypes.CDLL(LIB)
    f = lib.sep_attn_fwd_noalloc
    f.restype = ctypes.c_int
    st = lib.sep_status_string
    st.restype = ctypes.c_char_p
    st.argtypes = [ctypes.c_int]
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float

    def call(B, L, Hkv, d):
        m = _SepMask(B, L, 4, 64, 16, 16, 16, 16, 16, 16)
        return f(P(256), P(256), P(256), I(B), I(L), I(Hkv), I(Hkv), I(d), F(0.125), I(4), I(64),
                 ctypes.byref(m), P(256), P(256), None)

    cap = _scratch_bytes()
    assert cap == 64 << 20
    # 131072 tokens x 8 KV heads x d=128: 512 MiB of compacted K / V
    assert call(1, 131072, 8, 128) == SEP_ERR_SCRATCH_LIMIT
    # one token over the limit: 2 * B * L * Hkv * d * 2 bytes
    L_fit = cap // (2 * 2 * 8 * 128)
    assert call(1, L_fit + 1, 8, 128) == SEP_ERR_SCRATCH_LIMIT
    assert b"scratch" in st(SEP_ERR_SCRATCH_LIMIT)


@pytest.fixture(scope="module")
def S():
    import torch
    assert torch.cuda.is_available()
    from kv_cache_compression_sep_b200 import sepattn
    return sepattn


def _check(o, lse, o_ref, lse_ref, what):
    import torch
    err = np.abs(f64(o) - f64(o_ref))
    assert np.isfinite(f64(o)).all(), what
    assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, f"{what}: {err.max():.3e}"
    lerr = np.abs(f64(lse) - f64(lse_ref))
    assert lerr.max() <= LSE_ABS, f"{what}: lse {lerr.max():.3e}"
    assert torch.equal(o, o_ref), f"{what}: O not bit-identical to sep_attn_fwd"
    assert torch.equal(lse, lse_ref), f"{what}: LSE not bit-identical to sep_attn_fwd"


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny-gqa-L512-d64", "pythia160m-train-B8-H12-L2048-d64",
                                  "llama3-8b-prefill-H32-8-L8192-d128"])
def test_two_calls_match_workspace_entry_point(S, name):
    import torch
    import workloads
    cfg = workloads.ATTN_CONFIGS[name]
    dev = {k: (v.cuda() if v is not None else None)
           for k, v in workloads.attn_inputs(cfg, with_do=False).items()}
    mask = S.sep_mask_build(dev["sep"], cfg.a, cfg.n)
    o_ref, lse_ref = S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask)
    o1, lse1 = S.sep_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], mask)
    o2, lse2 = S.sep_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    _check(o1, lse1, o_ref, lse_ref, f"{name} first call")
    _check(o2, lse2, o_ref, lse_ref, f"{name} second call")


@pytest.mark.gpu
def test_two_calls_on_different_shapes(S):
    """Consecutive calls with different shapes reuse the one scratch array."""
    import torch
    import workloads
    for seed, (B, L, Hq, Hkv, d, a, n, p) in enumerate([(2, 300, 4, 2, 128, 1, 127, 0.1),
                                                        (1, 1030, 2, 1, 64, 4, 64, 0.3)]):
        inp = workloads.small_attn_inputs(seed, B, L, Hq, Hkv, d, p=p, with_do=False)
        dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
        mask = S.sep_mask_build(dev["sep"], a, n)
        o_ref, lse_ref = S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask)
        o, lse = S.sep_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], mask)
        torch.cuda.synchronize()
        assert S.sep_last_device_error() == 0
        _check(o, lse, o_ref, lse_ref, f"shape {B}x{L}x{Hq}x{Hkv}x{d}")
