"""numpy fp64 brute force used to pin the oracle (tests only).

Written from the definitions, independently of oracle/blasst_oracle.c:
full score matrices, textbook softmax, masked softmax over an explicit key
set, and the vectorised prefix-max form of the skip decision.
"""
from __future__ import annotations

import numpy as np

from synth import bf16_to_f32


def widen(bits):
    return bf16_to_f32(bits).astype(np.float64)


def score_matrix(q, k, scale, causal, b, hq, G, d=None, Lk=None):
    """scale * q k^T for one (batch, query head), [Lq, Lk], -inf where masked."""
    Q = widen(q[b, hq])
    d = Q.shape[1] if d is None else d
    K = widen(k[b, hq // G])[:, :d]
    Lq = Q.shape[0]
    Lk = K.shape[0] if Lk is None else Lk
    K = K[:Lk]
    S = scale * (Q @ K.T)
    if causal:
        pos = np.arange(Lq)[:, None] + (Lk - Lq)
        S = np.where(np.arange(Lk)[None, :] > pos, -np.inf, S)
    return S


def dense_attention(q, k, v, scale, causal, dv=None):
    """Textbook softmax(scale q k^T) v and logsumexp, fp64."""
    B, Hq, Lq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    dv = v.shape[-1] if dv is None else dv
    O = np.zeros((B, Hq, Lq, dv))
    LSE = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            S = score_matrix(q, k, scale, causal, b, h, G, d=d)
            m = S.max(axis=1, keepdims=True)
            e = np.exp(S - m)
            z = e.sum(axis=1, keepdims=True)
            O[b, h] = (e / z) @ widen(v[b, h // G])[:, :dv]
            LSE[b, h] = (m + np.log(z))[:, 0]
    return O, LSE


def tile_rows(is_decode, Hq, Hkv, Lq, BM, tile):
    """(b, list of (hq, pos)) of a flat tile index, in the oracle's row order."""
    G = Hq // Hkv
    if is_decode:
        tph = (G * Lq + BM - 1) // BM
        t = tile % tph
        bh = tile // tph
        b, hkv = divmod(bh, Hkv)
        rows = [(hkv * G + rho // Lq, rho % Lq) for rho in range(t * BM, min(G * Lq, (t + 1) * BM))]
    else:
        tph = (Lq + BM - 1) // BM
        t = tile % tph
        bh = tile // tph
        b, hq = divmod(bh, Hq)
        rows = [(hq, p) for p in range(t * BM, min(Lq, (t + 1) * BM))]
    return b, rows


def closed_form_decisions(q, k, scale, causal, lam, BM, BN, is_decode=False, num_splits=1, d=None,
                          seed_splits=False):
    """Skip mask from per-block row maxima only (prefix-max form).

    skip_j <=> j is not the first visited block of its split and
    max over voting rows r of (m~_rj - max_{j' <= j in split} m~_rj') < ln(lam).
    With seed_splits (decode), block 0's row maxima join the prefix max of every
    later split, which then has no forced first block.
    Returns (skip, visited) as [n_tiles, nb] uint8.
    """
    B, Hq, Lq, _ = q.shape
    Hkv = k.shape[1]
    Lk = k.shape[2]
    G = Hq // Hkv
    nb = (Lk + BN - 1) // BN
    if is_decode:
        n_tiles = B * Hkv * ((G * Lq + BM - 1) // BM)
    else:
        n_tiles = B * Hq * ((Lq + BM - 1) // BM)
        num_splits = 1
    per = (nb + num_splits - 1) // num_splits
    ln_lam = np.log(lam) if lam > 0 else -np.inf
    skip = np.zeros((n_tiles, nb), np.uint8)
    visited = np.zeros((n_tiles, nb), np.uint8)
    cache = {}
    for tile in range(n_tiles):
        b, rows = tile_rows(is_decode, Hq, Hkv, Lq, BM, tile)
        mt = np.full((len(rows), nb), -np.inf)
        for i, (hq, pos) in enumerate(rows):
            key = (b, hq)
            if key not in cache:
                cache[key] = score_matrix(q, k, scale, causal, b, hq, G, d=d)
            srow = cache[key][pos]
            pad = np.full(nb * BN, -np.inf)
            pad[:Lk] = srow
            mt[i] = pad.reshape(nb, BN).max(axis=1)
        vis = np.isfinite(mt).any(axis=0)
        visited[tile] = vis
        for sp in range(num_splits):
            j0, j1 = sp * per, min(nb, (sp + 1) * per)
            if j0 >= j1:
                continue
            seeded = is_decode and seed_splits and sp > 0
            if seeded:
                pm = np.maximum.accumulate(np.concatenate([mt[:, :1], mt[:, j0:j1]], axis=1), axis=1)[:, 1:]
            else:
                pm = np.maximum.accumulate(mt[:, j0:j1], axis=1)
            with np.errstate(invalid="ignore"):
                gap = np.where(np.isfinite(mt[:, j0:j1]), mt[:, j0:j1] - pm, -np.inf).max(axis=0)
            v = vis[j0:j1]
            first = np.argmax(v) if v.any() and not seeded else None
            dec = v & (gap < ln_lam)
            if first is not None:
                dec[first] = False
            skip[tile, j0:j1] = dec
    return skip, visited


def masked_attention(q, k, v, scale, causal, skip, BM, BN, is_decode=False, dv=None, d=None):
    """softmax over the keys of kept blocks only, fp64; (O, lse)."""
    B, Hq, Lq, _ = q.shape
    Hkv = k.shape[1]
    Lk = k.shape[2]
    G = Hq // Hkv
    dv = v.shape[-1] if dv is None else dv
    nb = (Lk + BN - 1) // BN
    O = np.zeros((B, Hq, Lq, dv))
    LSE = np.zeros((B, Hq, Lq))
    for tile in range(skip.shape[0]):
        b, rows = tile_rows(is_decode, Hq, Hkv, Lq, BM, tile)
        keep_keys = np.repeat(skip[tile] == 0, BN)[:Lk]
        for hq, pos in rows:
            s = score_matrix(q, k, scale, causal, b, hq, G, d=d)[pos]
            s = np.where(keep_keys, s, -np.inf)
            m = s.max()
            e = np.exp(s - m)
            z = e.sum()
            O[b, hq, pos] = (e / z) @ widen(v[b, hq // G])[:Lk, :dv]
            LSE[b, hq, pos] = m + np.log(z)
    return O, LSE
