"""GPU parity of sep_mask_build against the oracle: bit-exact on every output."""

import numpy as np
import pytest

from conftest import load_golden
from oracle import sepattn_ref as R

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import torch
    assert torch.cuda.is_available()
    from kv_cache_compression_sep_b200 import sepattn
    return sepattn


def _run(S, sep_np, a, n, bm, bn):
    import torch
    sep = torch.from_numpy(np.ascontiguousarray(sep_np.astype(np.uint8))).cuda()
    m = S.sep_mask_build(sep, a, n, bm, bn)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    out = {k: getattr(m, k).cpu().numpy() for k in
           ("anchor_idx", "anchor_cnt", "gather_end", "tile_map", "kept")}
    out["anchor_bits"] = m.anchor_bits.cpu().numpy().view(np.uint32)
    return out


def _compare(got, ref):
    for k in ("anchor_idx", "anchor_cnt", "gather_end", "tile_map", "kept", "anchor_bits"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def test_golden_example(S):
    g = load_golden("mask_L10_a2_n3.txt")
    sep = np.zeros((1, g["L"][0]), np.uint8)
    sep[0, g["sep"]] = 1
    got = _run(S, sep, g["a"][0], g["n"][0], g["bm"][0], g["bn"][0])
    assert got["anchor_idx"][0, :4].tolist() == g["anchor_idx"]
    for t, row in g["tile"].items():
        assert got["tile_map"][0, t].tolist() == row
    assert got["gather_end"][0].tolist() == g["gather_end"]
    assert int(got["kept"][0]) == g["kept_total"][0]
    assert got["anchor_bits"][0].tolist() == g["anchor_bits"]


@pytest.mark.parametrize("B,L,a,n,bm,bn,p", [
    (1, 1, 0, 1, 128, 128, 0.5), (2, 129, 4, 64, 128, 128, 0.1), (3, 300, 0, 1, 128, 128, 0.3),
    (2, 513, 1, 127, 128, 128, 0.0), (1, 777, 4, 256, 128, 128, 1.0), (2, 1000, 2, 2000, 128, 128, 0.05),
    (1, 20000, 4, 256, 128, 128, 0.1), (2, 555, 3, 17, 64, 32, 0.2), (1, 70, 5, 9, 7, 5, 0.25)])
def test_random_shapes(S, B, L, a, n, bm, bn, p):
    rng = np.random.default_rng(L * 31 + n)
    sep = (rng.random((B, L)) < p).astype(np.uint8)
    _compare(_run(S, sep, a, n, bm, bn), R.mask_build(sep, a, n, bm, bn))


def test_fixed_interval_flags(S):
    """FixLLM-style anchors at a fixed interval: a pure flag pattern."""
    L = 2048
    sep = np.zeros((2, L), np.uint8)
    sep[0, 15::16] = 1
    sep[1, 63::64] = 1
    _compare(_run(S, sep, 4, 64, 128, 128), R.mask_build(sep, 4, 64, 128, 128))


@pytest.mark.parametrize("name", ["tiny-gqa-L512-d64", "pythia160m-train-B8-H12-L2048-d64",
                                  "llama3-8b-prefill-H32-8-L8192-d128"])
def test_configs_full(S, name):
    import workloads
    cfg = workloads.ATTN_CONFIGS[name]
    g = __import__("torch").Generator().manual_seed(cfg.seed)
    sep = workloads.separator_flags(g, cfg.B, cfg.L, cfg.flags, cfg.p, cfg.force0).numpy()
    _compare(_run(S, sep, cfg.a, cfg.n, 128, 128), R.mask_build(sep, cfg.a, cfg.n, 128, 128))


@pytest.mark.parametrize("n", [256, 131072])
def test_long_context_sampled(S, n):
    """L = 131072: every anchor, gather_end and kept count; tile classes on sampled tiles."""
    import workloads
    cfg = workloads.LONG_CONTEXT
    g = __import__("torch").Generator().manual_seed(cfg.seed)
    sep = workloads.separator_flags(g, cfg.B, cfg.L, cfg.flags, cfg.p).numpy()
    got = _run(S, sep, cfg.a, n, 128, 128)
    f = R.anchor_flags(sep[0], cfg.a)
    pos = np.nonzero(f)[0]
    assert int(got["anchor_cnt"][0]) == len(pos)
    np.testing.assert_array_equal(got["anchor_idx"][0, : len(pos)], pos)
    assert (got["anchor_idx"][0, len(pos):] == -1).all()
    T = cfg.L // 128
    lo = np.maximum(0, np.arange(T) * 128 - n + 1) // 128 * 128
    np.testing.assert_array_equal(got["gather_end"][0], np.searchsorted(pos, lo, side="left"))
    assert int(got["kept"][0]) == int(R.kept_pairs_closed_form(sep, cfg.a, n)[0])
    fb = np.zeros(cfg.L // 32, dtype=np.uint64)
    for k in range(32):
        fb |= f.reshape(-1, 32)[:, k].astype(np.uint64) << np.uint64(k)
    np.testing.assert_array_equal(got["anchor_bits"][0], fb.astype(np.uint32))
    rng = np.random.default_rng(0)
    tiles = [(0, 0), (T - 1, T - 1), (T - 1, 0), (T - 1, T - 3), (500, 498)]
    tiles += [(int(t), int(u)) for t, u in zip(rng.integers(0, T, 60), rng.integers(0, T, 60))]
    for t, u in tiles:
        assert got["tile_map"][0, t, u] == R.tile_class(sep[0], cfg.a, n, 128, 128, t, u), (t, u)


def test_tile_map_both_count_paths():
    """Tile classes from the staged flag words (L <= 192000) and from the binary search over the
    anchor list (longer sequences): the same gather ends and classes as the oracle, sampled."""
    import torch
    from kv_cache_compression_sep_b200 import sepattn as S
    for L in (192000, 196608 + 77):  # 6000 flag words (staged), 6147 (binary search)
        rng = np.random.default_rng(L)
        sep = (rng.random((1, L)) < 0.08).astype(np.uint8)
        n, a = 200, 3
        got = _run(S, sep, a, n, 128, 128)
        f = R.anchor_flags(sep[0], a)
        pos = np.nonzero(f)[0]
        T = -(-L // 128)
        lo = np.maximum(0, np.arange(T) * 128 - n + 1) // 128 * 128
        np.testing.assert_array_equal(got["gather_end"][0], np.searchsorted(pos, lo, side="left"))
        tiles = [(0, 0), (T - 1, T - 1), (T - 1, 0), (T - 1, T - 2), (T - 1, T - 3), (700, 698)]
        tiles += [(int(t), int(u)) for t, u in zip(rng.integers(0, T, 40), rng.integers(0, T, 40))]
        for t, u in tiles:
            assert got["tile_map"][0, t, u] == R.tile_class(sep[0], a, n, 128, 128, t, u), (L, t, u)
    torch.cuda.synchronize()
