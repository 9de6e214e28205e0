"""SepCache streaming-decode oracle (test infrastructure): cache state machine + fp64 decode.

[BD] "SepLLM's Architecture: Composing Efficiency" splits the streaming KV cache into an
Initial Cache (first tokens), a Local Window Cache of capacity w, a Past Window Cache and a
Separator Cache that keeps only separator KV of older tokens, with total capacity c. [SP]
"Limitations & Caveats" and [AS] "Measured effects" (removing positional-encoding shifting)
say positions are taken inside the cache, not in the original text.

Readings where the pages are silent:
* Without a usage threshold (c = None): fixed partitions a + s + w and a Past Window Cache of
  size 0, so compression happens one token at a time: when the window overflows, its oldest
  token moves to the separator cache if it is a separator and is evicted otherwise; when the
  separator cache overflows, its oldest entry is evicted.
* With a usage threshold c (> a + s + w): a token leaving the window goes to the Past Window
  Cache; right after an append that makes initial + separators + past + window reach c, the
  past window's separators move to the separator cache oldest first (which evicts its oldest
  entries beyond s) and the rest of the past window is dropped. The usage after a step is
  therefore always below c.
* The first a tokens go to the initial cache whatever their flag.
* Per step: the update happens first, then the new token's query attends to every retained
  slot, itself included.
* Positional-encoding shifting: the position of a retained key is its rank in the logical
  order [initial | separators oldest first | past window oldest first | window oldest first];
  the query's position is its own rank (occupied - 1). Keys are kept un-rotated and rotated
  afresh at every step.
* RoPE convention: rotate-half pairs (k, k + d/2) with angle p * theta^(-2k/d).
"""

from __future__ import annotations

from collections import deque

import numpy as np


class SepCacheSim:
    """Integer state machine of one SepCache sequence: which original tokens are retained.

    Holds original token positions only; the K/V content is looked up by position.
    """

    def __init__(self, a, s, w, c=None):
        assert a >= 0 and s >= 0 and w >= 1
        assert c is None or c > a + s + w
        self.a, self.s, self.w, self.c = a, s, w, c
        self.initial = []
        self.seps = deque()
        self.past = []
        self.window = deque()
        self.t = 0

    def usage(self):
        return len(self.initial) + len(self.seps) + len(self.past) + len(self.window)

    def _to_separators(self, pos):
        self.seps.append(pos)
        if len(self.seps) > self.s:
            self.seps.popleft()

    def append(self, is_sep):
        """Add the next token (original position self.t) and compress if over capacity."""
        tok = self.t
        self.t += 1
        if tok < self.a:
            self.initial.append(tok)
            return
        self.window.append((tok, bool(is_sep)))
        if len(self.window) > self.w:
            old, old_sep = self.window.popleft()
            if self.c is None:
                if old_sep:
                    self._to_separators(old)
            else:
                self.past.append((old, old_sep))
        if self.c is not None and self.usage() >= self.c:
            for p, p_sep in self.past:
                if p_sep:
                    self._to_separators(p)
            self.past = []

    def order(self):
        """Retained original positions in logical order; a key's rank is its in-cache position."""
        return (list(self.initial) + list(self.seps) + [p for p, _ in self.past] +
                [p for p, _ in self.window])


def rope_rotate(x, pos, theta):
    """Rotate-half RoPE of vectors x [..., d] at integer positions pos (broadcast on [...]).

    out[k] = x[k] cos(p w_k) - x[k + d/2] sin(p w_k), out[k + d/2] = x[k + d/2] cos(p w_k)
    + x[k] sin(p w_k), w_k = theta^(-2k/d), in fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    w = theta ** (-2.0 * np.arange(h) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * w
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def decode_attention(q, k_ret, v_ret, theta, scale):
    """Single-query attention of one step over the retained keys, with in-cache positions.

    q [Hq, d] is the new token's query (un-rotated); k_ret/v_ret [n_ret, Hkv, d] are the
    retained keys/values in logical order (un-rotated keys). Key r sits at position r, the
    query at position n_ret - 1. Returns o [Hq, d] and lse [Hq] (natural log), fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    k_ret = np.asarray(k_ret, dtype=np.float64)
    v_ret = np.asarray(v_ret, dtype=np.float64)
    n_ret = k_ret.shape[0]
    Hq, d = q.shape
    Hkv = k_ret.shape[1]
    G = Hq // Hkv
    kr = rope_rotate(k_ret, np.arange(n_ret)[:, None], theta)
    qr = rope_rotate(q, np.full((Hq,), n_ret - 1), theta)
    o = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for h in range(Hq):
        kh = h // G
        s = scale * (kr[:, kh, :] @ qr[h])
        mx = s.max()
        e = np.exp(s - mx)
        l = e.sum()
        o[h] = (e / l) @ v_ret[:, kh, :]
        lse[h] = mx + np.log(l)
    return o, lse


# ---------------------------------------------------------------- decode without shifting
# Training-free use of the separator mask at inference ([AS] "Key results": training-free
# Llama-3-8B with the cache keeping initial, separator and neighbour tokens): no positional
# shifting, so every retained key keeps its original position. Reading: such a cache stores
# each key rotated once at its original position, in the storage type (bf16), as an ordinary
# rotary KV cache does; only the query is rotated at decode time, at its own position t.
def bf16_round(x):
    """Round to the nearest bfloat16 (ties to even), returned as fp64."""
    import torch
    return torch.as_tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def stored_rotated_key(k, pos, theta):
    """A key as the cache stores it without shifting: RoPE(k, pos) in fp64, rounded to bf16."""
    return bf16_round(rope_rotate(k, pos, theta))


def decode_attention_original_positions(q, k_stored, v_ret, t, theta, scale):
    """Single-query attention over retained keys already rotated at their original positions
    (k_stored [n_ret, Hkv, d]); the query q [Hq, d] is rotated at its own position t.
    Returns o [Hq, d] and lse [Hq] (natural log), fp64."""
    q = np.asarray(q, dtype=np.float64)
    k_stored = np.asarray(k_stored, dtype=np.float64)
    v_ret = np.asarray(v_ret, dtype=np.float64)
    Hq, d = q.shape
    Hkv = k_stored.shape[1]
    G = Hq // Hkv
    qr = rope_rotate(q, np.full((Hq,), t), theta)
    o = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for h in range(Hq):
        kh = h // G
        s = scale * (k_stored[:, kh, :] @ qr[h])
        mx = s.max()
        e = np.exp(s - mx)
        l = e.sum()
        o[h] = (e / l) @ v_ret[:, kh, :]
        lse[h] = mx + np.log(l)
    return o, lse
