"""The Python binding's argument checks (CPU only): every malformed call raises SepError before
anything reaches the library, and CPU tensors are refused (there is no CPU path)."""

import pytest
import torch

from kv_cache_compression_sep_b200 import sepattn as S


def _mask(B, L, a=2, n=4):
    sep = torch.zeros(B, L, dtype=torch.uint8)
    z = torch.zeros(1)
    return S.SepMask(sep=sep, anchor_idx=z, anchor_cnt=z, anchor_bits=z, gather_end=z,
                     tile_map=z, kept=z, a=a, n=n)


def test_library_loads_and_reports_a_missing_device():
    # on a machine without a GPU the error-word query reports the CUDA failure as a status
    # instead of crashing; with a GPU and nothing launched the word is clear
    code = S.sep_last_device_error()
    if torch.cuda.is_available():
        assert code == 0
    else:
        assert code == 4 and "CUDA" in S._lib.sep_status_string(code).decode().upper()


def test_mask_build_refuses_cpu_and_bad_rank():
    with pytest.raises(S.SepError, match="CUDA"):
        S.sep_mask_build(torch.zeros(2, 10, dtype=torch.uint8), 2, 4)
    with pytest.raises(S.SepError, match="2-D"):
        S.sep_mask_build(torch.zeros(2, 3, 10, dtype=torch.uint8), 2, 4)
    with pytest.raises(S.SepError, match="dtype"):
        S.sep_mask_build(torch.zeros(2, 10, dtype=torch.int32), 2, 4)


def test_mask_build_checks_reused_buffers():
    out = S.SepMask(sep=torch.zeros(2, 10, dtype=torch.uint8),
                    anchor_idx=torch.zeros(2, 9, dtype=torch.int32),  # one column short
                    anchor_cnt=torch.zeros(2, dtype=torch.int32),
                    anchor_bits=torch.zeros(2, 1, dtype=torch.int32),
                    gather_end=torch.zeros(2, 1, dtype=torch.int32),
                    tile_map=torch.zeros(2, 1, 1, dtype=torch.int8),
                    kept=torch.zeros(2, dtype=torch.int64), a=2, n=4)
    with pytest.raises(S.SepError, match="CUDA|shape"):
        S.sep_mask_build(torch.zeros(2, 10, dtype=torch.uint8), 2, 4, out=out)


def _qkv(B=1, L=16, Hq=4, Hkv=2, d=64):
    q = torch.zeros(B, L, Hq, d, dtype=torch.bfloat16)
    k = torch.zeros(B, L, Hkv, d, dtype=torch.bfloat16)
    return q, k, k.clone()


def test_attention_checks_shapes_before_the_device():
    q, k, v = _qkv()
    with pytest.raises(S.SepError, match="mask was built"):
        S.sep_attn_fwd(q, k, v, _mask(1, 17))
    with pytest.raises(S.SepError, match="shape"):
        S.sep_attn_fwd(q, k[:, :8].contiguous(), v, _mask(1, 16))
    with pytest.raises(S.SepError, match="multiple"):
        S.sep_attn_fwd(q, torch.zeros(1, 16, 3, 64, dtype=torch.bfloat16), v, _mask(1, 16))
    with pytest.raises(S.SepError, match="4-D"):
        S.sep_attn_fwd(q[0], k, v, _mask(1, 16))


def test_attention_refuses_cpu_tensors():
    q, k, v = _qkv()
    m = _mask(1, 16)
    with pytest.raises(S.SepError, match="CUDA"):
        S.sep_attn_fwd(q, k, v, m)
    with pytest.raises(S.SepError, match="CUDA"):
        S.sep_attn_fwd_noalloc(q, k, v, m)
    with pytest.raises(S.SepError, match="CUDA"):
        S.sep_attn_bwd(q, k, v, q, torch.zeros(1, 4, 16), q, m)


def test_cache_refuses_a_cpu_device():
    with pytest.raises(S.SepError, match="CUDA"):
        S.SepCache(2, 8, 2, 128, 2, 3, 5, 10000.0, device="cpu")


def test_device_checks(monkeypatch):
    """Every tensor of a call must be on one device, and that device must be the current one
    (the library launches there); checked before anything reaches the library."""
    import types
    d0, d1 = torch.device("cuda", 0), torch.device("cuda", 1)
    t0, t1 = types.SimpleNamespace(device=d0), types.SimpleNamespace(device=d1)
    monkeypatch.setattr(S, "_current_device_index", lambda: 0)
    S._same_device(d0, ("k", t0), ("v", t0), ("lse", None))
    with pytest.raises(S.SepError, match="v is on cuda:1"):
        S._same_device(d0, ("k", t0), ("v", t1))
    with pytest.raises(S.SepError, match="current CUDA device is cuda:0"):
        S._same_device(d1, ("k", t1))
    monkeypatch.setattr(S, "_current_device_index", lambda: 1)
    S._same_device(d1, ("k", t1))
