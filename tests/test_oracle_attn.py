"""Pins for the oracle's attention forward and backward (CPU only).

Pins: pure-Python per-query loops, a closed form (zero queries + one-hot values read out
the kept set of the hand-derived example), torch's fp64 causal SDPA for the cases that
reduce to dense causal attention, slicing for the sliding-window case, the gathered form,
central finite differences for the gradients and exact gradient identities.
"""

import math

import numpy as np
import pytest
import torch

from conftest import load_golden
from oracle import sepattn_ref as R


def _rand(shape, rng):
    return rng.standard_normal(shape)


def _brute_fwd(q, k, v, sep, a, n, scale):
    """Per-query Python loops: build the kept list, softmax with math.exp, weighted sum."""
    B, L, Hq, d = q.shape
    G = Hq // k.shape[2]
    O = np.zeros((B, L, Hq, d))
    LSE = np.zeros((B, Hq, L))
    for b in range(B):
        for i in range(L):
            kept = [j for j in range(i + 1) if j < a or sep[b, j] or i - j < n]
            for h in range(Hq):
                s = [scale * sum(q[b, i, h, c] * k[b, j, h // G, c] for c in range(d)) for j in kept]
                m = max(s)
                e = [math.exp(x - m) for x in s]
                tot = sum(e)
                for c in range(d):
                    O[b, i, h, c] = sum(e[t] * v[b, j, h // G, c] for t, j in enumerate(kept)) / tot
                LSE[b, h, i] = m + math.log(tot)
    return O, LSE


@pytest.mark.parametrize("L,a,n,Hq,Hkv", [(9, 2, 3, 2, 1), (14, 0, 4, 2, 2), (12, 3, 20, 3, 1)])
def test_fwd_vs_brute_force(L, a, n, Hq, Hkv):
    rng = np.random.default_rng(L)
    B, d = 2, 3
    q, k, v = _rand((B, L, Hq, d), rng), _rand((B, L, Hkv, d), rng), _rand((B, L, Hkv, d), rng)
    sep = (rng.random((B, L)) < 0.3).astype(np.uint8)
    O, LSE = R.attn_fwd(q, k, v, sep, a, n, 0.7)
    Ob, LSEb = _brute_fwd(q, k, v, sep, a, n, 0.7)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(LSE, LSEb, rtol=1e-12, atol=1e-12)


def test_zero_query_reads_out_golden_kept_sets():
    """q = 0 makes attention uniform over the kept set: O_i = mean of one-hot v_j over K(i)."""
    g = load_golden("mask_L10_a2_n3.txt")
    L, a, n = g["L"][0], g["a"][0], g["n"][0]
    sep = np.zeros((1, L), np.uint8)
    sep[0, g["sep"]] = 1
    q = np.zeros((1, L, 1, L))
    k = np.random.default_rng(0).standard_normal((1, L, 1, L))
    v = np.eye(L)[None, :, None, :]
    O, LSE = R.attn_fwd(q, k, v, sep, a, n, 1.0)
    for i, kept in g["kept"].items():
        want = np.zeros(L)
        want[kept] = 1.0 / len(kept)
        np.testing.assert_allclose(O[0, i, 0], want, atol=1e-15)
        assert abs(LSE[0, 0, i] - math.log(len(kept))) < 1e-13


def _sdpa_causal(q, k, v, scale):
    G = q.shape[2] // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, G, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, G, axis=2)).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("mode", ["n_ge_L", "all_sep"])
def test_reduces_to_dense_causal(mode):
    rng = np.random.default_rng(3)
    B, L, Hq, Hkv, d = 2, 40, 4, 2, 8
    q, k, v = _rand((B, L, Hq, d), rng), _rand((B, L, Hkv, d), rng), _rand((B, L, Hkv, d), rng)
    if mode == "n_ge_L":
        sep, a, n = (rng.random((B, L)) < 0.1).astype(np.uint8), 3, L
    else:
        sep, a, n = np.ones((B, L), np.uint8), 0, 1
    O, _ = R.attn_fwd(q, k, v, sep, a, n, 0.35)
    np.testing.assert_allclose(O, _sdpa_causal(q, k, v, 0.35), rtol=1e-10, atol=1e-12)


def test_sliding_window_by_slicing():
    rng = np.random.default_rng(4)
    B, L, H, d, n = 1, 30, 2, 5, 6
    q, k, v = _rand((B, L, H, d), rng), _rand((B, L, H, d), rng), _rand((B, L, H, d), rng)
    O, LSE = R.attn_fwd(q, k, v, np.zeros((B, L), np.uint8), 0, n, 0.5)
    for i in range(L):
        lo = max(0, i - n + 1)
        for h in range(H):
            s = 0.5 * k[0, lo:i + 1, h] @ q[0, i, h]
            p = np.exp(s - s.max())
            np.testing.assert_allclose(O[0, i, h], (p / p.sum()) @ v[0, lo:i + 1, h], atol=1e-13)
            assert abs(LSE[0, h, i] - (s.max() + np.log(p.sum()))) < 1e-12


def test_masked_equals_gathered():
    rng = np.random.default_rng(5)
    B, L, Hq, Hkv, d = 2, 70, 4, 2, 6
    q, k, v = _rand((B, L, Hq, d), rng), _rand((B, L, Hkv, d), rng), _rand((B, L, Hkv, d), rng)
    sep = (rng.random((B, L)) < 0.15).astype(np.uint8)
    O, LSE = R.attn_fwd(q, k, v, sep, 2, 9, 0.4)
    for b in range(B):
        Og, Lg = R.attn_fwd_rows(q, k, v, sep, 2, 9, 0.4, b, list(range(L)))
        np.testing.assert_allclose(Og, O[b], atol=1e-13)
        np.testing.assert_allclose(Lg.T, LSE[b], atol=1e-12)


def test_gqa_is_mha_with_repeated_kv():
    rng = np.random.default_rng(6)
    B, L, Hq, Hkv, d = 1, 20, 6, 2, 4
    q, k, v = _rand((B, L, Hq, d), rng), _rand((B, L, Hkv, d), rng), _rand((B, L, Hkv, d), rng)
    do = _rand((B, L, Hq, d), rng)
    sep = (rng.random((B, L)) < 0.2).astype(np.uint8)
    G = Hq // Hkv
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    O1, L1 = R.attn_fwd(q, k, v, sep, 1, 4, 0.5)
    O2, L2 = R.attn_fwd(q, kr, vr, sep, 1, 4, 0.5)
    np.testing.assert_allclose(O1, O2, atol=1e-14)
    dq1, dk1, dv1 = R.attn_bwd(q, k, v, do, sep, 1, 4, 0.5)
    dq2, dk2, dv2 = R.attn_bwd(q, kr, vr, do, sep, 1, 4, 0.5)
    np.testing.assert_allclose(dq1, dq2, atol=1e-13)
    np.testing.assert_allclose(dk1, dk2.reshape(B, L, Hkv, G, d).sum(3), atol=1e-13)
    np.testing.assert_allclose(dv1, dv2.reshape(B, L, Hkv, G, d).sum(3), atol=1e-13)


def test_gradients_vs_finite_differences():
    rng = np.random.default_rng(7)
    B, L, Hq, Hkv, d = 1, 11, 2, 1, 3
    a, n, scale = 1, 3, 0.8
    q, k, v = _rand((B, L, Hq, d), rng), _rand((B, L, Hkv, d), rng), _rand((B, L, Hkv, d), rng)
    do = _rand((B, L, Hq, d), rng)
    sep = np.zeros((B, L), np.uint8)
    sep[0, [3, 6]] = 1

    def loss(q_, k_, v_):
        return float((R.attn_fwd(q_, k_, v_, sep, a, n, scale)[0] * do).sum())

    dq, dk, dv = R.attn_bwd(q, k, v, do, sep, a, n, scale)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            ap = [xp if nm == name else t for nm, t in zip("qkv", args)]
            am = [xm if nm == name else t for nm, t in zip("qkv", args)]
            num[idx] = (loss(*ap) - loss(*am)) / (2 * eps)
        err = np.abs(num - g).max() / max(1e-12, np.abs(g).max())
        assert err < 1e-6, (name, err)


def test_gradient_identities():
    """sum_j dS_ij = 0 gives sum over keys of dK = 0; sum_j P_ij = 1 gives sum dV = sum dO."""
    rng = np.random.default_rng(8)
    B, L, Hq, Hkv, d = 2, 45, 4, 2, 5
    q, k, v = _rand((B, L, Hq, d), rng), _rand((B, L, Hkv, d), rng), _rand((B, L, Hkv, d), rng)
    do = _rand((B, L, Hq, d), rng)
    sep = (rng.random((B, L)) < 0.1).astype(np.uint8)
    dq, dk, dv = R.attn_bwd(q, k, v, do, sep, 2, 6, 0.6)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    G = Hq // Hkv
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1).reshape(B, Hkv, G, d).sum(2),
                               atol=1e-12)


def test_sampled_backward_matches_full():
    rng = np.random.default_rng(9)
    B, L, Hq, Hkv, d = 1, 40, 4, 2, 4
    q, k, v = _rand((B, L, Hq, d), rng), _rand((B, L, Hkv, d), rng), _rand((B, L, Hkv, d), rng)
    do = _rand((B, L, Hq, d), rng)
    sep = (rng.random((B, L)) < 0.2).astype(np.uint8)
    dq, dk, dv = R.attn_bwd(q, k, v, do, sep, 3, 7, 0.5)
    rows = [0, 1, 7, 20, 39]
    keys = [0, 2, 5, 13, 30, 39]
    sq, sk, sv = R.attn_bwd_sampled(q, k, v, do, sep, 3, 7, 0.5, 0, rows, keys)
    np.testing.assert_allclose(sq, dq[0, rows], atol=1e-12)
    np.testing.assert_allclose(sk, dk[0, keys], atol=1e-12)
    np.testing.assert_allclose(sv, dv[0, keys], atol=1e-12)
