"""fp64 oracle: separator-sparse causal attention, forward and backward (test infrastructure).

What SepLLM computes ([AS] "Approach"; [BD] "The Mechanics of Compression", training-from-
scratch setting): every query attends only to the initial tokens, to every preceding separator
and to its n most recent neighbours. [BD] "SepLLM's Architecture" writes the attention as
O = M(A, V, M_b) with a binary n x n mask M_b. This file writes that out as plain masked
softmax attention in float64, plus its analytic gradients, with no blocking or fusion.

Readings where the pages are silent:
* "n neighbours" = the n most recent tokens including the query itself: i - n < j <= i.
* "initial tokens" = positions j < a; every kept pair is causal (j <= i).
* A zero in M_b is a logit of -inf (the pair is dropped from the softmax).
* GQA: query head h reads KV head h // (Hq // Hkv).
* LSE is the natural log of sum_j exp(scale * q_i . k_j) over kept j.
* Tiles for the mask artefacts are BM query rows x BN key columns; the gathered part of a
  query tile is every anchor left of the first key tile that holds a window key of the
  tile's first row (the window/diagonal key tiles are handled as whole tiles).
"""

from __future__ import annotations

import numpy as np

SKIP, PARTIAL, FULL = 0, 1, 2


def anchor_flags(sep, a):
    """Anchor flag f[j] = (j < a) or sep[j]: the keys every later query keeps.

    [AS] "Approach": initial tokens and all preceding separators are kept.
    Works on a 1-D flag row or a [B, L] batch.
    """
    f = np.asarray(sep).astype(bool).copy()
    f[..., : max(0, a)] = True
    return f


def keep_mask(sep_row, a, n):
    """The binary mask M_b of [BD] "SepLLM's Architecture" for one sequence.

    M[i, j] = 1 iff j <= i and (i - j < n or f[j]), i.e. j is an initial token, a
    preceding separator, or one of the n most recent neighbours ([AS] "Approach").
    """
    f = anchor_flags(sep_row, a)
    L = f.shape[0]
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return (j <= i) & (((i - j) < n) | f[None, :])


def keep_block(sep_row, a, n, r0, r1, c0, c1):
    """Rows r0..r1-1 x columns c0..c1-1 of M_b, from the same rule as keep_mask.

    For long sequences, where the full L x L mask does not fit in memory.
    """
    f = anchor_flags(sep_row, a)
    i = np.arange(r0, r1)[:, None]
    j = np.arange(c0, c1)[None, :]
    return (j <= i) & (((i - j) < n) | f[c0:c1][None, :])


def tile_class(sep_row, a, n, bm, bn, t, u):
    """SKIP / PARTIAL / FULL of block (t, u) of M_b (in-bounds pairs only)."""
    L = len(sep_row)
    blk = keep_block(sep_row, a, n, t * bm, min(L, (t + 1) * bm), u * bn, min(L, (u + 1) * bn))
    return SKIP if not blk.any() else (FULL if blk.all() else PARTIAL)


def kept_pairs(sep, a, n):
    """Number of kept (query, key) pairs per batch element, counted on the mask."""
    sep = np.atleast_2d(sep)
    return np.array([int(keep_mask(s, a, n).sum()) for s in sep], dtype=np.int64)


def kept_pairs_closed_form(sep, a, n):
    """Kept pairs per row = min(i + 1, n) + C(i - n), C(x) = #anchors at positions <= x.

    The window gives min(i + 1, n) keys; every anchor left of the window is added once
    (de-duplicated union of the three kept sets of [AS] "Approach").
    """
    sep = np.atleast_2d(sep)
    out = []
    for s in sep:
        f = anchor_flags(s, a)
        L = f.shape[0]
        C = np.cumsum(f.astype(np.int64))
        tot = 0
        for i in range(L):
            tot += min(i + 1, n) + (int(C[i - n]) if i - n >= 0 else 0)
        out.append(tot)
    return np.array(out, dtype=np.int64)


def mask_build(sep, a, n, bm, bn):
    """Mask artefacts the CUDA path consumes, computed from M by plain loops.

    Returns dict with
      anchor_idx [B, L] int32: sorted anchor positions, -1 past anchor_cnt,
      anchor_cnt [B] int32,
      gather_end [B, T] int32: number of anchors left of key tile lo(t), where
          lo(t) = max(0, t*bm - n + 1) // bn is the key tile holding the earliest window key
          of query row t*bm; those anchors are kept by every row of query tile t,
      tile_map [B, T, U] int8: SKIP if no pair of the (t, u) block is kept, FULL if every
          in-bounds pair is kept, PARTIAL otherwise,
      kept [B] int64: kept pairs,
      anchor_bits [B, ceil(L/32)] uint32: bit k of word w is f[32w + k] (0 past L).
    """
    sep = np.atleast_2d(np.asarray(sep))
    B, L = sep.shape
    T = -(-L // bm)
    U = -(-L // bn)
    anchor_idx = np.full((B, L), -1, dtype=np.int32)
    anchor_cnt = np.zeros(B, dtype=np.int32)
    gather_end = np.zeros((B, T), dtype=np.int32)
    tile_map = np.zeros((B, T, U), dtype=np.int8)
    kept = np.zeros(B, dtype=np.int64)
    W = -(-L // 32)
    anchor_bits = np.zeros((B, W), dtype=np.uint32)
    for b in range(B):
        f = anchor_flags(sep[b], a)
        for j in range(L):
            if f[j]:
                anchor_bits[b, j // 32] |= np.uint32(1 << (j % 32))
        M = keep_mask(sep[b], a, n)
        pos = [j for j in range(L) if f[j]]
        anchor_idx[b, : len(pos)] = pos
        anchor_cnt[b] = len(pos)
        kept[b] = int(M.sum())
        for t in range(T):
            lo_key = max(0, t * bm - n + 1)
            lo_tile = lo_key // bn
            gather_end[b, t] = sum(1 for j in pos if j < lo_tile * bn)
            for u in range(U):
                blk = M[t * bm : min(L, (t + 1) * bm), u * bn : min(L, (u + 1) * bn)]
                if not blk.any():
                    tile_map[b, t, u] = SKIP
                elif blk.all():
                    tile_map[b, t, u] = FULL
                else:
                    tile_map[b, t, u] = PARTIAL
    return dict(anchor_idx=anchor_idx, anchor_cnt=anchor_cnt, gather_end=gather_end,
                tile_map=tile_map, kept=kept, anchor_bits=anchor_bits)


def _f64(x):
    x = np.asarray(x)
    return x.astype(np.float64)


def attn_fwd(q, k, v, sep, a, n, scale):
    """O = M(A, V, M_b) ([BD] "SepLLM's Architecture") as masked softmax attention in fp64.

    q [B, L, Hq, d], k/v [B, L, Hkv, d], sep [B, L]. Returns O [B, L, Hq, d] and
    LSE [B, Hq, L] (natural log). A = scale * Q K^T, masked to -inf where M_b is 0.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    sep = np.atleast_2d(np.asarray(sep))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    O = np.zeros((B, L, Hq, d))
    LSE = np.zeros((B, Hq, L))
    for b in range(B):
        M = keep_mask(sep[b], a, n)
        for h in range(Hq):
            kh = h // G
            S = scale * (q[b, :, h, :] @ k[b, :, kh, :].T)
            S = np.where(M, S, -np.inf)
            mx = S.max(axis=1, keepdims=True)
            E = np.exp(S - mx)
            l = E.sum(axis=1, keepdims=True)
            P = E / l
            O[b, :, h, :] = P @ v[b, :, kh, :]
            LSE[b, h, :] = mx[:, 0] + np.log(l[:, 0])
    return O, LSE


def attn_bwd(q, k, v, do, sep, a, n, scale):
    """Analytic gradients of sum(O * dO) for attn_fwd, in fp64.

    With P = softmax(masked A): dV = P^T dO, dP = dO V^T, Delta_i = sum_c dO_ic O_ic,
    dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q. dK/dV of a KV head are
    summed over the query heads that share it. Returns dq, dk, dv (shapes of q, k, v).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    sep = np.atleast_2d(np.asarray(sep))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        M = keep_mask(sep[b], a, n)
        for h in range(Hq):
            kh = h // G
            Q, K, V, dO = q[b, :, h, :], k[b, :, kh, :], v[b, :, kh, :], do[b, :, h, :]
            S = np.where(M, scale * (Q @ K.T), -np.inf)
            mx = S.max(axis=1, keepdims=True)
            E = np.exp(S - mx)
            P = E / E.sum(axis=1, keepdims=True)
            O = P @ V
            dv[b, :, kh, :] += P.T @ dO
            dP = dO @ V.T
            Delta = (dO * O).sum(axis=1, keepdims=True)
            dS = P * (dP - Delta)
            dq[b, :, h, :] = scale * (dS @ K)
            dk[b, :, kh, :] += scale * (dS.T @ Q)
    return dq, dk, dv


def kept_index_set(f, i, n):
    """Sorted key indices kept by query i: the window max(0, i-n+1)..i plus anchors j <= i-n.

    This is the explicit gathered set of [AS] "Approach" (initial tokens, preceding
    separators, n neighbours) with each index once.
    """
    lo = max(0, i - n + 1)
    left = np.nonzero(f[:lo])[0] if lo > 0 else np.zeros(0, dtype=np.int64)
    return np.concatenate([left, np.arange(lo, i + 1)])


def attn_fwd_rows(q, k, v, sep, a, n, scale, b, rows, heads=None):
    """Dense softmax attention over the explicitly gathered kept keys, for chosen rows.

    Second form of the same definition: for each query row i of batch b, gather K(i)
    and run ordinary softmax attention on it. Never builds the L x L mask, so it serves
    long sequences at sampled rows (inputs may be float32 or bf16-valued arrays; only the
    gathered rows are widened to fp64). Returns O [len(rows), H, d] and LSE [len(rows), H]
    for the heads asked for (all query heads by default).
    """
    f = anchor_flags(np.asarray(sep)[b], a)
    L, Hq, d = q.shape[1:]
    Hkv = k.shape[2]
    G = Hq // Hkv
    heads = list(range(Hq)) if heads is None else list(heads)
    O = np.zeros((len(rows), len(heads), d))
    LSE = np.zeros((len(rows), len(heads)))
    for r, i in enumerate(rows):
        i = int(i)
        idx = kept_index_set(f, i, n)
        qi = _f64(q[b, i])
        for kh in sorted({h // G for h in heads}):
            K = _f64(k[b, idx, kh, :])
            V = _f64(v[b, idx, kh, :])
            for c, h in enumerate(heads):
                if h // G != kh:
                    continue
                s = scale * (K @ qi[h])
                mx = s.max()
                e = np.exp(s - mx)
                l = e.sum()
                O[r, c, :] = (e / l) @ V
                LSE[r, c] = mx + np.log(l)
    return O, LSE


def attn_bwd_sampled(q, k, v, do, sep, a, n, scale, b, q_rows, k_rows, kv_heads=None):
    """Gradients at chosen rows without the L x L mask (gathered form of attn_bwd).

    dQ_i = scale * sum_{j in K(i)} P_ij (dP_ij - Delta_i) k_j for each i in q_rows.
    For each key j in k_rows, the queries that keep j are R(j) = j..min(L-1, j+n-1), plus
    every later query when j is an anchor; then
    dK_j = scale * sum_{i in R(j)} dS_ij q_i and dV_j = sum_{i in R(j)} P_ij dO_i,
    summed over the query heads of the KV head. P_ij and Delta_i come from each query's own
    gathered forward. Returns dq [len(q_rows), Hq, d], dk/dv [len(k_rows), Hkv', d].
    """
    f = anchor_flags(np.asarray(sep)[b], a)
    L, Hq, d = q.shape[1:]
    Hkv = k.shape[2]
    G = Hq // Hkv
    kv_heads = list(range(Hkv)) if kv_heads is None else list(kv_heads)

    row_cache = {}

    def row_stats(i):
        # P row over K(i), dP row and Delta_i, for every query head
        if i not in row_cache:
            idx = kept_index_set(f, i, n)
            P = np.zeros((Hq, len(idx)))
            dP = np.zeros((Hq, len(idx)))
            Delta = np.zeros(Hq)
            qi, doi = _f64(q[b, i]), _f64(do[b, i])
            for kh in range(Hkv):
                K = _f64(k[b, idx, kh, :])
                V = _f64(v[b, idx, kh, :])
                for h in range(kh * G, (kh + 1) * G):
                    s = scale * (K @ qi[h])
                    e = np.exp(s - s.max())
                    P[h] = e / e.sum()
                    Delta[h] = float(doi[h] @ (P[h] @ V))
                    dP[h] = V @ doi[h]
            row_cache[i] = (idx, P, dP, Delta)
        return row_cache[i]

    dq = np.zeros((len(q_rows), Hq, d))
    for r, i in enumerate(q_rows):
        i = int(i)
        idx, P, dP, Delta = row_stats(i)
        for h in range(Hq):
            dS = P[h] * (dP[h] - Delta[h])
            dq[r, h, :] = scale * (dS @ _f64(k[b, idx, h // G, :]))

    dk = np.zeros((len(k_rows), len(kv_heads), d))
    dv = np.zeros((len(k_rows), len(kv_heads), d))
    for r, j in enumerate(k_rows):
        j = int(j)
        rows = list(range(j, min(L, j + n)))
        if f[j]:
            rows += list(range(j + n, L))
        for i in rows:
            idx, P, dP, Delta = row_stats(i)
            pos = int(np.searchsorted(idx, j))
            assert idx[pos] == j
            qi, doi = _f64(q[b, i]), _f64(do[b, i])
            for c, kh in enumerate(kv_heads):
                for h in range(kh * G, (kh + 1) * G):
                    p = P[h, pos]
                    ds = p * (dP[h, pos] - Delta[h])
                    dk[r, c, :] += scale * ds * qi[h]
                    dv[r, c, :] += p * doi[h]
    return dq, dk, dv
