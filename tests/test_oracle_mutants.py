"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case rewrites one expression of one oracle function: a dropped term, a wrong sign, an
off-by-one index, a transposed operand or a wrong convention. The rewritten function is
installed in place of the oracle's, and pins that the unmodified oracle passes are run
against it. At least one of them must fail. This checks the pins themselves: a plausible
slip anywhere in the oracle does not go unnoticed. The mistakes are planted in the oracle,
on the CPU only, and never touch the CUDA path.
"""

import inspect
import textwrap

import pytest

import test_oracle_attn as TA
import test_oracle_mask as TM
import test_oracle_sepcache as TS
from oracle import sepattn_ref as R
from oracle import sepcache_ref as C


def _mutant(owner, name, old, new):
    """Source of owner.name with the single occurrence of `old` replaced by `new`, compiled in
    the namespace of the function's own module."""
    fn = getattr(owner, name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, (name, old)
    ns = dict(vars(inspect.getmodule(fn)))
    exec(compile(src.replace(old, new), f"<planted mistake in {name}>", "exec"), ns)
    return ns[name]


# pins, as calls with fixed arguments
P_GOLDEN_MASK = TM.test_golden_kept_sets
P_GOLDEN_ART = TM.test_golden_artefacts
P_UNION = lambda: TM.test_brute_force_union(24, 3, 5, 0.2)  # noqa: E731
P_CLOSED = TM.test_closed_form_count_many
P_TRIANGLES = TM.test_special_cases_reduce_to_triangles
P_SPLIT = lambda: TM.test_gather_split_covers_mask_once(50, 2, 5, 4, 4, 0.2)  # noqa: E731
P_BRUTE = lambda: TA.test_fwd_vs_brute_force(9, 2, 3, 2, 1)  # noqa: E731
P_ZERO_Q = TA.test_zero_query_reads_out_golden_kept_sets
P_DENSE = lambda: TA.test_reduces_to_dense_causal("n_ge_L")  # noqa: E731
P_WINDOW = TA.test_sliding_window_by_slicing
P_GATHERED = TA.test_masked_equals_gathered
P_GQA = TA.test_gqa_is_mha_with_repeated_kv
P_FD = TA.test_gradients_vs_finite_differences
P_IDENT = TA.test_gradient_identities
P_SAMPLED = TA.test_sampled_backward_matches_full
P_TRAJ = TS.test_golden_trajectory
P_INV = lambda: TS.test_invariants(0, 3, 5, 0.3)  # noqa: E731
P_PREFILL = TS.test_unbounded_separator_cache_equals_prefill_mask
P_STREAM = TS.test_no_separator_cache_is_streaming_llm
P_TRAJ_PAST = TS.test_golden_trajectory_past_window
P_INV_PAST = lambda: TS.test_past_window_invariants(0, 3, 5, 20, 0.3)  # noqa: E731
P_COMPLEX = TS.test_rope_matches_complex_multiplication
P_ROPE_EX = TS.test_rope_small_worked_example
P_DEC = TS.test_decode_without_eviction_is_causal_rope_attention
P_ORIG_ROW = TS.test_original_positions_decode_is_the_mask_row
P_ORIG_CAUSAL = TS.test_original_positions_before_eviction_is_causal_rope_attention
P_BF16 = TS.test_bf16_round_ties_to_even

CASES = [
    # ---- keep rule and mask artefacts
    ("window one wider", R, "keep_mask", "((i - j) < n)", "((i - j) <= n)",
     [P_GOLDEN_MASK, P_UNION, P_TRIANGLES]),
    ("causality dropped", R, "keep_mask", "(j <= i) & ", "", [P_GOLDEN_MASK, P_UNION]),
    ("separators ignored", R, "keep_mask", "| f[None, :]", "| False", [P_GOLDEN_MASK, P_UNION]),
    ("initial tokens dropped", R, "anchor_flags", "f[..., : max(0, a)] = True", "pass",
     [P_GOLDEN_MASK, P_UNION, P_TRIANGLES]),
    ("initial tokens one short", R, "anchor_flags", "max(0, a)", "max(0, a - 1)",
     [P_GOLDEN_MASK, P_UNION]),
    ("closed form: anchor count one late", R, "kept_pairs_closed_form", "int(C[i - n])",
     "int(C[min(i - n + 1, L - 1)])", [P_CLOSED, P_GOLDEN_MASK]),
    ("closed form: window one short", R, "kept_pairs_closed_form", "tot += min(i + 1, n)",
     "tot += min(i, n)", [P_CLOSED, P_GOLDEN_MASK]),
    ("gather end counts the tile's first key", R, "mask_build", "if j < lo_tile * bn)",
     "if j <= lo_tile * bn)", [P_GOLDEN_ART, P_SPLIT]),
    ("tile map: FULL and PARTIAL swapped", R, "mask_build", "tile_map[b, t, u] = FULL",
     "tile_map[b, t, u] = PARTIAL", [P_GOLDEN_ART]),
    ("anchor bits off by one", R, "mask_build", "1 << (j % 32)", "1 << ((j + 1) % 32)",
     [P_GOLDEN_ART]),
    # ---- forward
    ("LSE in log2", R, "attn_fwd", "mx[:, 0] + np.log(l[:, 0])", "mx[:, 0] + np.log2(l[:, 0])",
     [P_BRUTE, P_ZERO_Q]),
    ("QK^T transposed", R, "attn_fwd", "scale * (q[b, :, h, :] @ k[b, :, kh, :].T)",
     "scale * (k[b, :, kh, :] @ q[b, :, h, :].T)", [P_BRUTE, P_DENSE]),
    ("scale dropped", R, "attn_fwd", "S = scale * (", "S = (", [P_BRUTE, P_DENSE]),
    ("GQA map interleaved", R, "attn_fwd", "kh = h // G", "kh = h % Hkv", [P_BRUTE, P_DENSE, P_GQA]),
    ("no max subtraction in LSE", R, "attn_fwd", "LSE[b, h, :] = mx[:, 0] + ", "LSE[b, h, :] = ",
     [P_BRUTE, P_ZERO_Q]),
    ("gathered window one short", R, "kept_index_set", "lo = max(0, i - n + 1)",
     "lo = max(0, i - n + 2)", [P_GATHERED, P_PREFILL]),
    ("gathered form: anchors up to the query", R, "kept_index_set", "np.nonzero(f[:lo])",
     "np.nonzero(f[:lo + 1])", [P_GATHERED, P_PREFILL]),
    # ---- backward
    ("dS sign of Delta", R, "attn_bwd", "dS = P * (dP - Delta)\n", "dS = P * (dP + Delta)\n",
     [P_FD, P_IDENT]),
    ("dK scale dropped", R, "attn_bwd", "dk[b, :, kh, :] += scale * (dS.T @ Q)",
     "dk[b, :, kh, :] += (dS.T @ Q)", [P_FD]),
    ("dV not summed over the group", R, "attn_bwd", "dv[b, :, kh, :] += P.T @ dO",
     "dv[b, :, kh, :] = P.T @ dO", [P_FD, P_IDENT, P_GQA]),
    ("dQ with dS transposed", R, "attn_bwd", "dq[b, :, h, :] = scale * (dS @ K)",
     "dq[b, :, h, :] = scale * (dS.T @ K)", [P_FD]),
    ("Delta from dO alone", R, "attn_bwd", "Delta = (dO * O)", "Delta = (dO * dO)", [P_FD]),
    ("dP from K instead of V", R, "attn_bwd", "dP = dO @ V.T", "dP = dO @ K.T", [P_FD]),
    # ---- SepCache state machine
    ("window evicts its newest", C.SepCacheSim, "append", "self.window.popleft()",
     "self.window.pop()", [P_TRAJ, P_INV]),
    ("non-separators kept", C.SepCacheSim, "append", "if old_sep:", "if True:",
     [P_TRAJ, P_INV]),
    ("separator cache evicts its newest", C.SepCacheSim, "_to_separators",
     "self.seps.popleft()", "self.seps.pop()", [P_TRAJ, P_INV]),
    ("initial cache one larger", C.SepCacheSim, "append", "if tok < self.a:",
     "if tok <= self.a:", [P_TRAJ, P_INV, P_STREAM]),
    ("compression one token late", C.SepCacheSim, "append", "self.usage() >= self.c",
     "self.usage() > self.c", [P_TRAJ_PAST, P_INV_PAST]),
    ("past window separators dropped", C.SepCacheSim, "append", "if p_sep:", "if False:",
     [P_TRAJ_PAST, P_INV_PAST]),
    ("logical order: separators before initial", C.SepCacheSim, "order",
     "list(self.initial) + list(self.seps)", "list(self.seps) + list(self.initial)",
     [P_TRAJ, P_INV]),
    # ---- RoPE and decode
    ("RoPE adjacent pairs", C, "rope_rotate", "x1, x2 = x[..., :h], x[..., h:]",
     "x1, x2 = x[..., 0::2], x[..., 1::2]", [P_COMPLEX, P_ROPE_EX]),
    ("RoPE rotation sign", C, "rope_rotate", "x1 * c - x2 * s", "x1 * c + x2 * s",
     [P_COMPLEX, P_ROPE_EX]),
    ("RoPE frequency exponent halved", C, "rope_rotate", "theta ** (-2.0 * np.arange(h) / d)",
     "theta ** (-1.0 * np.arange(h) / d)", [P_COMPLEX]),
    ("decode query one position late", C, "decode_attention", "np.full((Hq,), n_ret - 1)",
     "np.full((Hq,), n_ret)", [P_DEC]),
    ("decode GQA map interleaved", C, "decode_attention", "kh = h // G", "kh = h % Hkv", [P_DEC]),
    ("decode scale dropped", C, "decode_attention", "s = scale * (", "s = (", [P_DEC]),
    ("no-shift query at t - 1", C, "decode_attention_original_positions", "np.full((Hq,), t)",
     "np.full((Hq,), t - 1)", [P_ORIG_ROW, P_ORIG_CAUSAL]),
    ("bf16 rounding by truncation", C, "bf16_round",
     "return torch.as_tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()",
     "y = np.asarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFF0000)\n"
     "    return y.view(np.float32).astype(np.float64)", [P_BF16]),
]


def _fails(pins):
    for pin in pins:
        try:
            pin()
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("label,owner,name,old,new,pins", CASES, ids=[c[0] for c in CASES])
def test_planted_mistake_fails_a_pin(label, owner, name, old, new, pins, monkeypatch):
    monkeypatch.setattr(owner, name, _mutant(owner, name, old, new))
    assert _fails(pins), f"no pin catches: {label}"
