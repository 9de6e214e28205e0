"""Pins for the oracle's mask and mask artefacts (CPU only).

Each test checks the oracle against something other than itself: a hand-derived worked
example of the keep rule, a pure-Python union of the three kept categories, library
triangles for the special cases, and the closed form of the kept-pair count.
"""

import itertools

import numpy as np
import pytest

from conftest import load_golden
from oracle import sepattn_ref as R


def _golden_mask():
    g = load_golden("mask_L10_a2_n3.txt")
    L, a, n = g["L"][0], g["a"][0], g["n"][0]
    sep = np.zeros(L, dtype=np.uint8)
    sep[g["sep"]] = 1
    return g, sep, a, n


def test_golden_kept_sets():
    g, sep, a, n = _golden_mask()
    M = R.keep_mask(sep, a, n)
    for i, kept in g["kept"].items():
        assert sorted(np.nonzero(M[i])[0].tolist()) == kept, i
    assert int(M.sum()) == g["kept_total"][0]
    assert int(R.kept_pairs(sep[None], a, n)[0]) == g["kept_total"][0]
    assert int(R.kept_pairs_closed_form(sep[None], a, n)[0]) == g["kept_total"][0]


def test_golden_artefacts():
    g, sep, a, n = _golden_mask()
    art = R.mask_build(sep[None], a, n, g["bm"][0], g["bn"][0])
    cnt = int(art["anchor_cnt"][0])
    assert art["anchor_idx"][0, :cnt].tolist() == g["anchor_idx"]
    assert (art["anchor_idx"][0, cnt:] == -1).all()
    tm = art["tile_map"][0]
    for t, row in g["tile"].items():
        assert tm[t].tolist() == row, t
    assert art["gather_end"][0].tolist() == g["gather_end"]
    assert int(art["kept"][0]) == g["kept_total"][0]
    assert art["anchor_bits"][0].tolist() == g["anchor_bits"]


def _brute_kept(sep, a, n, i):
    """The three kept categories of the pages, written separately, then united."""
    initial = {j for j in range(min(a, i + 1))}
    separators = {j for j in range(i + 1) if sep[j]}
    neighbours = {j for j in range(max(0, i - n + 1), i + 1)}
    return initial | separators | neighbours


@pytest.mark.parametrize("L,a,n,p", [(1, 0, 1, 0.5), (7, 0, 1, 0.3), (24, 3, 5, 0.2),
                                     (33, 1, 40, 0.1), (40, 0, 7, 0.0), (40, 5, 2, 1.0),
                                     (64, 4, 16, 0.1)])
def test_brute_force_union(L, a, n, p):
    rng = np.random.default_rng(L * 7 + a)
    sep = (rng.random(L) < p).astype(np.uint8)
    M = R.keep_mask(sep, a, n)
    for i in range(L):
        assert set(np.nonzero(M[i])[0].tolist()) == _brute_kept(sep, a, n, i)


def test_closed_form_count_many():
    rng = np.random.default_rng(0)
    for L, a, n in itertools.product([1, 5, 31, 64, 97], [0, 1, 4], [1, 3, 64, 200]):
        sep = (rng.random((2, L)) < 0.15).astype(np.uint8)
        assert (R.kept_pairs(sep, a, n) == R.kept_pairs_closed_form(sep, a, n)).all()


def test_special_cases_reduce_to_triangles():
    L = 37
    rng = np.random.default_rng(1)
    sep = (rng.random(L) < 0.2).astype(np.uint8)
    tril = np.tril(np.ones((L, L), dtype=bool))
    # n >= L keeps every causal pair: dense causal attention
    assert (R.keep_mask(sep, 2, L) == tril).all()
    # every token a separator: dense causal again
    assert (R.keep_mask(np.ones(L, np.uint8), 0, 1) == tril).all()
    # no separators, a = 0: a band of width n (sliding window)
    n = 5
    band = tril & ~np.tril(np.ones((L, L), dtype=bool), k=-n)
    assert (R.keep_mask(np.zeros(L, np.uint8), 0, n) == band).all()
    # no separators, a > 0: sinks plus the band (StreamingLLM pattern)
    sinks = tril & (np.arange(L)[None, :] < 3)
    assert (R.keep_mask(np.zeros(L, np.uint8), 3, n) == (band | sinks)).all()


@pytest.mark.parametrize("L,bm", [(8, 2), (13, 4), (17, 16)])
def test_tile_map_dense_causal(L, bm):
    """All-keep mask: tiles below the diagonal FULL, diagonal PARTIAL, above SKIP."""
    sep = np.zeros((1, L), np.uint8)
    tm = R.mask_build(sep, 0, L, bm, bm)["tile_map"][0]
    T = tm.shape[0]
    for t in range(T):
        for u in range(T):
            rows = min(L, (t + 1) * bm) - t * bm
            if u < t:
                assert tm[t, u] == R.FULL
            elif u > t:
                assert tm[t, u] == R.SKIP
            else:
                assert tm[t, u] == (R.FULL if rows == 1 else R.PARTIAL)


@pytest.mark.parametrize("L,a,n,bm,bn,p", [(50, 2, 5, 4, 4, 0.2), (70, 0, 9, 8, 8, 0.1),
                                            (33, 4, 40, 8, 8, 0.3), (65, 1, 1, 16, 16, 0.5)])
def test_gather_split_covers_mask_once(L, a, n, bm, bn, p):
    """Gathered anchors + whole key tiles lo(t)..t reproduce every row's kept set exactly once."""
    rng = np.random.default_rng(L + n)
    sep = (rng.random((1, L)) < p).astype(np.uint8)
    art = R.mask_build(sep, a, n, bm, bn)
    M = R.keep_mask(sep[0], a, n)
    T = art["gather_end"].shape[1]
    for t in range(T):
        lo_tile = max(0, t * bm - n + 1) // bn
        gathered = art["anchor_idx"][0, : art["gather_end"][0, t]].tolist()
        assert all(j < lo_tile * bn for j in gathered)
        for i in range(t * bm, min(L, (t + 1) * bm)):
            window_part = [j for j in range(lo_tile * bn, i + 1) if M[i, j]]
            assert sorted(gathered + window_part) == np.nonzero(M[i])[0].tolist()


def test_block_form_matches_full_mask():
    rng = np.random.default_rng(21)
    L, a, n = 90, 3, 11
    sep = (rng.random(L) < 0.15).astype(np.uint8)
    M = R.keep_mask(sep, a, n)
    np.testing.assert_array_equal(R.keep_block(sep, a, n, 17, 63, 5, 80), M[17:63, 5:80])
    tm = R.mask_build(sep[None], a, n, 16, 16)["tile_map"][0]
    for t in range(tm.shape[0]):
        for u in range(tm.shape[1]):
            assert R.tile_class(sep, a, n, 16, 16, t, u) == tm[t, u]
