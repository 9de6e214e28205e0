"""Pins for the SepCache oracle (CPU only): hand-derived trajectory, invariants, RoPE forms."""

import numpy as np
import pytest
import torch

from conftest import load_golden
from oracle import sepattn_ref as R
from oracle import sepcache_ref as C


def test_golden_trajectory():
    g = load_golden("sepcache_a1_s2_w3.txt")
    sim = C.SepCacheSim(g["a"][0], g["s"][0], g["w"][0])
    seps = set(g["sep"])
    for t in sorted(g["step"]):
        sim.append(t in seps)
        assert sim.order() == g["step"][t], t


@pytest.mark.parametrize("a,s,w,p", [(4, 64, 732, 0.1), (0, 3, 5, 0.3), (2, 0, 4, 0.5),
                                     (1, 2, 1, 0.9), (3, 1, 2, 0.0)])
def test_invariants(a, s, w, p):
    rng = np.random.default_rng(a * 100 + s)
    steps = 3000
    flags = rng.random(steps) < p
    sim = C.SepCacheSim(a, s, w)
    for t in range(steps):
        sim.append(flags[t])
        order = sim.order()
        assert len(order) <= a + s + w
        assert order == sorted(order) and len(set(order)) == len(order)
        assert order[-1] == t                     # the new token is retained
        n_init = min(t + 1, a)
        assert order[:n_init] == list(range(n_init))
        n_win = min(t + 1 - n_init, w)
        assert order[len(order) - n_win:] == list(range(t + 1 - n_win, t + 1))
        middle = order[n_init:len(order) - n_win]
        assert len(middle) <= s
        assert all(flags[j] for j in middle)
        # every separator that left the window is retained unless s newer ones displaced it
        left = [j for j in range(n_init, t + 1 - n_win) if flags[j]]
        assert middle == left[max(0, len(left) - s):]


def test_unbounded_separator_cache_equals_prefill_mask():
    """With s >= #separators and w = n the retained set is the kept set K(t) of the mask."""
    rng = np.random.default_rng(11)
    a, n, steps = 3, 7, 400
    sep = (rng.random(steps) < 0.2).astype(np.uint8)
    sim = C.SepCacheSim(a, steps, n)
    f = R.anchor_flags(sep, a)
    for t in range(steps):
        sim.append(bool(sep[t]))
        assert sim.order() == R.kept_index_set(f, t, n).tolist()


def test_no_separator_cache_is_streaming_llm():
    sim = C.SepCacheSim(4, 0, 10)
    for t in range(100):
        sim.append(True)
        order = sim.order()
        assert order == list(range(min(t + 1, 4))) + list(range(max(4, t - 9), t + 1))


def test_rope_matches_complex_multiplication():
    rng = np.random.default_rng(12)
    d, theta = 16, 500000.0
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 7, 799, 12345])
    y = C.rope_rotate(x, pos, theta)
    w = theta ** (-np.arange(d // 2) * 2.0 / d)
    z = (x[:, : d // 2] + 1j * x[:, d // 2:]) * np.exp(1j * pos[:, None] * w)
    np.testing.assert_allclose(y, np.concatenate([z.real, z.imag], axis=1), atol=1e-12)
    np.testing.assert_allclose(C.rope_rotate(x, np.zeros(5), theta), x, atol=0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_small_worked_example():
    # d = 4, theta = 100: frequencies 1 and 0.1; e_0 at position 1 -> (cos 1, 0, sin 1, 0)
    y = C.rope_rotate(np.array([1.0, 0, 0, 0]), np.array(1), 100.0)
    np.testing.assert_allclose(y, [np.cos(1.0), 0.0, np.sin(1.0), 0.0], atol=1e-15)


def test_rope_relative_invariance():
    rng = np.random.default_rng(13)
    d = 32
    q, k = rng.standard_normal(d), rng.standard_normal((6, d))
    pk = np.array([0, 3, 4, 9, 10, 11])
    s1 = C.rope_rotate(k, pk, 1e4) @ C.rope_rotate(q, np.array(11), 1e4)
    s2 = C.rope_rotate(k, pk + 500, 1e4) @ C.rope_rotate(q, np.array(511), 1e4)
    np.testing.assert_allclose(s1, s2, atol=1e-10)


def test_decode_without_eviction_is_causal_rope_attention():
    """Before any eviction the in-cache rank is the original position: ordinary RoPE decode."""
    rng = np.random.default_rng(14)
    Hq, Hkv, d, theta, t = 4, 2, 8, 1e4, 9
    k = rng.standard_normal((t + 1, Hkv, d))
    v = rng.standard_normal((t + 1, Hkv, d))
    q = rng.standard_normal((Hq, d))
    o, lse = C.decode_attention(q, k, v, theta, 0.3)
    # library reference: rotate at original positions, SDPA over all keys (last query sees all)
    kr = C.rope_rotate(k, np.arange(t + 1)[:, None], theta)
    qr = C.rope_rotate(q, np.full(Hq, t), theta)
    G = Hq // Hkv
    qt = torch.from_numpy(qr)[:, None, :]
    kt = torch.from_numpy(np.repeat(kr, G, axis=1)).permute(1, 0, 2)
    vt = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=0.3)[:, 0].numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)
    s = 0.3 * np.einsum("khd,hd->hk", np.repeat(kr, G, axis=1), qr)
    np.testing.assert_allclose(lse, np.log(np.exp(s).sum(1)), atol=1e-12)


# ---------------------------------------------------------------- Past Window Cache (usage c)
def test_golden_trajectory_past_window():
    g = load_golden("sepcache_past_a1_s2_w2_c7.txt")
    sim = C.SepCacheSim(g["a"][0], g["s"][0], g["w"][0], g["c"][0])
    seps = set(g["sep"])
    for t in sorted(g["step"]):
        sim.append(t in seps)
        assert sim.order() == g["step"][t], t
        assert sim.usage() < g["c"][0]


@pytest.mark.parametrize("a,s,w,c,p", [(4, 64, 256, 800, 0.1), (0, 3, 5, 20, 0.3),
                                       (2, 0, 4, 12, 0.5), (1, 2, 1, 5, 0.9), (3, 1, 2, 7, 0.0)])
def test_past_window_invariants(a, s, w, c, p):
    rng = np.random.default_rng(a * 100 + s + c)
    steps = 3000
    flags = rng.random(steps) < p
    sim = C.SepCacheSim(a, s, w, c)
    ref = C.SepCacheSim(a, s, w)  # the one-token-at-a-time rule
    for t in range(steps):
        sim.append(flags[t])
        ref.append(flags[t])
        order = sim.order()
        assert len(order) < c
        assert order == sorted(order) and len(set(order)) == len(order)
        assert order[-1] == t
        n_init = min(t + 1, a)
        assert order[:n_init] == list(range(n_init))
        n_win = min(t + 1 - n_init, w)
        assert order[len(order) - n_win:] == list(range(t + 1 - n_win, t + 1))
        # middle = separators (all flagged, at most s) then the past window, a contiguous run
        # of the tokens that left the window since the last compression
        n_past = len(sim.past)
        past = order[len(order) - n_win - n_past:len(order) - n_win]
        assert past == list(range(t + 1 - n_win - n_past, t + 1 - n_win))
        mid = order[n_init:len(order) - n_win - n_past]
        assert len(mid) <= s and all(flags[j] for j in mid)
        # right after a compression the retained set is the one-token-at-a-time rule's
        if n_past == 0:
            assert order == ref.order(), t


# ---------------------------------------------------------------- decode without shifting
def test_original_positions_decode_is_the_mask_row():
    """With every separator retained (s large) and w = n, decode at step t without shifting is
    row t of the separator-sparse attention over RoPE'd queries and stored (rotated, bf16) keys."""
    rng = np.random.default_rng(5)
    a, n, L, Hq, Hkv, d, theta = 3, 6, 60, 4, 2, 8, 500000.0
    sep = (rng.random(L) < 0.25).astype(np.uint8)
    q = rng.standard_normal((L, Hq, d))
    k = rng.standard_normal((L, Hkv, d))
    v = rng.standard_normal((L, Hkv, d))
    pos = np.arange(L)
    k_st = C.stored_rotated_key(k, pos[:, None], theta)
    q_rot = C.rope_rotate(q, pos[:, None], theta)
    sim = C.SepCacheSim(a, L, n)
    for t in range(L):
        sim.append(bool(sep[t]))
        order = sim.order()
        o, lse = C.decode_attention_original_positions(q[t], k_st[order], v[order], t, theta,
                                                       d ** -0.5)
        ro, rl = R.attn_fwd_rows(q_rot[None], k_st[None], v[None], sep[None], a, n, d ** -0.5,
                                 0, [t])
        np.testing.assert_allclose(o, ro[0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, rl[0], rtol=1e-12, atol=1e-12)


def test_original_positions_before_eviction_is_causal_rope_attention():
    rng = np.random.default_rng(6)
    L, Hq, Hkv, d, theta = 20, 4, 4, 16, 10000.0
    q = rng.standard_normal((Hq, d))
    k = rng.standard_normal((L, Hkv, d))
    v = rng.standard_normal((L, Hkv, d))
    k_st = C.stored_rotated_key(k, np.arange(L)[:, None], theta)
    o, lse = C.decode_attention_original_positions(q, k_st, v, L - 1, theta, d ** -0.5)
    qr = C.rope_rotate(q, np.full((Hq,), L - 1), theta)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qr)[:, None, :], torch.from_numpy(k_st).permute(1, 0, 2),
        torch.from_numpy(v).permute(1, 0, 2), scale=d ** -0.5)
    np.testing.assert_allclose(o, ref[:, 0].numpy(), rtol=1e-10, atol=1e-12)


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7: ties go to the even one (1)
    assert C.bf16_round(1.0 + 2 ** -8) == 1.0
    assert C.bf16_round(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6
    assert C.bf16_round(1.0 + 2 ** -8 + 2 ** -20) == 1.0 + 2 ** -7
