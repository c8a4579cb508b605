"""fp64 CPU oracle for BLASST blocked attention with softmax-threshold skipping.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline and reference legs may import this package.  The
CUDA path in ``block_sparse_flashattention_tcgen05_b200`` never imports it and
shares no code with it.

``attention()`` wraps the plain C implementation in ``blasst_oracle.c`` (fp64,
OpenMP over tiles; it states the method and the readings it follows).
``calibrate_fit()`` and ``threshold_for_sparsity()`` are the calibration steps
(lambda = a/L and lambda*L = alpha*exp(beta*s); xllm-io paper review,
section 3, "threshold calibration" and "calibration model").

Pins (tests/test_oracle_*.py) hold every function here to something other
than itself: numpy brute-force softmax at lambda = 0, hand-built block-max
cases, the prefix-max closed form of the decision, monotonicity in lambda, the
skipped-mass identity and bound, split invariance, and exact recovery of
(alpha, beta).  The relation between real-model sparsity and ``a`` is parity
unpinned (no real-model data here).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "blasst_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BM_PREFILL = 128
BN_PREFILL = 128
BN_DECODE = 64


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP, no BLAS)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            lib.blasst_oracle_attention.restype = ctypes.c_int
            lib.blasst_oracle_attention.argtypes = [
                P, P, P,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_longlong, ctypes.c_longlong,
                ctypes.c_double, ctypes.c_double, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                P, ctypes.c_longlong, P,
                P, P, P, P, P, P,
            ]
            lib.blasst_oracle_num_tiles.restype = ctypes.c_longlong
            lib.blasst_oracle_num_tiles.argtypes = [ctypes.c_int] * 8
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def num_tiles(is_decode, B, Hq, Hkv, Lq, Lk, BM, BN) -> int:
    return int(_load().blasst_oracle_num_tiles(int(is_decode), B, Hq, Hkv, Lq, Lk, BM, BN))


def attention(q, k, v, *, scale, lam, causal, is_decode=False, num_splits=1, BM=None, BN=None,
              dv=None, k_row_stride=None, v_row_stride=None, Lk=None, tiles=None, forced_skip=None,
              Hkv=None, seed_splits=False):
    """Run the oracle.

    q: uint16 [B, Hq, Lq, d] bf16 bits.  k, v: uint16 arrays holding
    [B, Hkv, Lk, row_stride] rows (v may be the same array as k, MLA-style,
    with dv < d).  Returns a dict with o [B,Hq,Lq,dv] f64, lse [B,Hq,Lq] f64
    (natural log), and per (tile, block) arrays skip, visited (uint8) and gaps
    (f64; +inf on a first block, NaN where not visited), plus the counts.
    ``tiles``: optional list of flat tile indices to compute (others: NaN).
    ``seed_splits`` (decode): splits after the first start their running max
    at block 0's row maxima and have no forced first block.
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    B, Hq, Lq, d = q.shape
    Hkv = k.shape[1] if Hkv is None else Hkv
    k_row_stride = k.shape[-1] if k_row_stride is None else k_row_stride
    v_row_stride = v.shape[-1] if v_row_stride is None else v_row_stride
    dv = min(d, v_row_stride) if dv is None else dv
    Lk = k.shape[2] if Lk is None else Lk
    if BM is None:
        BM = 128
    if BN is None:
        BN = BN_DECODE if is_decode else BN_PREFILL
    nt = num_tiles(is_decode, B, Hq, Hkv, Lq, Lk, BM, BN)
    if nt < 0:
        raise ValueError("bad shape")
    nb = (Lk + BN - 1) // BN
    o = np.full((B, Hq, Lq, dv), np.nan)
    lse = np.full((B, Hq, Lq), np.nan)
    skip = np.zeros((nt, nb), np.uint8)
    visited = np.zeros((nt, nb), np.uint8)
    gaps = np.full((nt, nb), np.nan)
    counts = np.zeros(2, np.int64)
    tiles_arr = None
    if tiles is not None:
        tiles_arr = np.ascontiguousarray(np.asarray(tiles, dtype=np.int64))
    fs = None
    if forced_skip is not None:
        fs = np.ascontiguousarray(np.asarray(forced_skip, dtype=np.uint8).reshape(nt, nb))
    rc = _load().blasst_oracle_attention(
        _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Lq, Lk, d, dv, k_row_stride, v_row_stride,
        float(scale), float(lam), int(bool(causal)), BM, BN, int(bool(is_decode)), int(num_splits),
        int(bool(seed_splits)), _ptr(tiles_arr), 0 if tiles_arr is None else len(tiles_arr), _ptr(fs),
        _ptr(o), _ptr(lse), _ptr(skip), _ptr(visited), _ptr(gaps), _ptr(counts))
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return dict(o=o, lse=lse, skip=skip, visited=visited, gaps=gaps,
                n_skipped=int(counts[0]), n_visited=int(counts[1]), n_blocks=nb, n_tiles=nt)


def calibrate_fit(L, lam, s):
    """Least-squares fit of ln(lambda*L) = ln(alpha) + beta*s.

    The calibration model lambda*L = alpha*exp(beta*s) (xllm-io paper review,
    section 3), linear in (s, ln(lambda*L)).  Returns (alpha, beta).
    """
    L = np.asarray(L, dtype=np.float64)
    lam = np.asarray(lam, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    y = np.log(lam * L)
    n = len(s)
    if n < 2:
        raise ValueError("need at least two points")
    sx = s.sum()
    sy = y.sum()
    sxx = (s * s).sum()
    sxy = (s * y).sum()
    den = n * sxx - sx * sx
    if den == 0.0:
        raise ValueError("all sparsities equal")
    beta = (n * sxy - sx * sy) / den
    ln_alpha = (sy - beta * sx) / n
    return math.exp(ln_alpha), beta


def threshold_for_sparsity(gaps, visited, target):
    """Smallest-error lambda for a target block sparsity from decision gaps.

    The skip decision of a pair is ``gap < ln(lambda)`` and its gap does not
    depend on lambda (a skipped block never raises the running max), so the
    achievable sparsities are the steps of the empirical gap distribution.
    Returns (lambda, achieved_sparsity).  First blocks (gap = +inf) count in
    the denominator and are never skipped.
    """
    vis = np.asarray(visited).astype(bool)
    g = np.asarray(gaps, dtype=np.float64)[vis]
    n_vis = g.size
    cand = np.sort(g[np.isfinite(g) & (g < 0.0)])
    want = int(round(target * n_vis))
    want = max(0, min(want, cand.size))
    if want == 0:
        return 0.0, 0.0
    hi = cand[want] if want < cand.size else 0.0
    lo = cand[want - 1]
    ln_lam = 0.5 * (lo + hi) if hi > lo else lo + 0.5 * (hi - lo)
    if not ln_lam > lo:
        ln_lam = np.nextafter(lo, np.inf)
    lam = math.exp(ln_lam)
    lam = min(lam, np.nextafter(1.0, 0.0))
    achieved = float(np.count_nonzero(cand < math.log(lam))) / n_vis
    return lam, achieved


def _as_f64(a):
    """bf16 bit patterns (uint16) or real arrays -> float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def attention_backward(q, k, v, do, *, scale, causal, skip=None, BM=BM_PREFILL, BN=BN_PREFILL):
    """Gradients of blocked attention with a FIXED skip mask (fp64, no blocking).

    The forward is O = softmax_kept(scale * Q K^T) V, where a score (r, c)
    takes part iff key c is visible to query r (c < Lk and, causal,
    c <= r + Lk - Lq) and the (query tile r // BM, key block c // BN) pair is
    not skipped; lse_r = log sum_kept exp(S_rc).  With the mask held constant
    this is plain masked softmax attention, so its gradient is the textbook
    one, written out step by step.  Skipped pairs carry P = 0 and so receive
    no gradient, which is the optional sparsity-aware training the pages
    describe (xllm-io paper review, section 3, "training procedure"):

        P    = exp(S - lse) on kept entries, 0 elsewhere
        dV   = P^T dO                  (summed over the query heads of a KV head)
        dP   = dO V^T
        D_r  = sum_c P_rc dP_rc
        dS   = P * (dP - D)
        dQ   = scale * dS K
        dK   = scale * dS^T Q          (summed over the query heads of a KV head)

    q [B, Hq, Lq, d], k [B, Hkv, Lk, d], v [B, Hkv, Lk, dv], do [B, Hq, Lq, dv]:
    uint16 bf16 bit patterns or real arrays.  skip: None (nothing skipped) or
    uint8 [B * Hq * ceil(Lq / BM), ceil(Lk / BN)], 1 = skipped, tiles ordered
    (b, hq, query tile) -- the prefill mask layout.  A row with no kept score
    has O = 0, lse = -inf and no gradient.
    Returns dict dq, dk, dv, o (float64) and lse (float64, natural log).
    """
    Q, K, V, dO = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    dv = V.shape[3]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    nq = (Lq + BM - 1) // BM
    nb = (Lk + BN - 1) // BN
    if skip is not None:
        skip = np.asarray(skip, dtype=np.uint8).reshape(B, Hq, nq, nb)
    rows = np.arange(Lq)[:, None]
    cols = np.arange(Lk)[None, :]
    visible = np.ones((Lq, Lk), bool)
    if causal:
        visible &= cols <= rows + (Lk - Lq)
    dq = np.zeros((B, Hq, Lq, d))
    dk = np.zeros((B, Hkv, Lk, d))
    dvv = np.zeros((B, Hkv, Lk, dv))
    o = np.zeros((B, Hq, Lq, dv))
    lse = np.full((B, Hq, Lq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            keep = visible.copy()
            if skip is not None:
                keep &= ~skip[b, h][rows // BM, cols // BN].astype(bool)
            S = scale * (Q[b, h] @ K[b, hk].T)
            Sm = np.where(keep, S, -np.inf)
            m = Sm.max(axis=1, keepdims=True)
            has = np.isfinite(m[:, 0])
            m = np.where(np.isfinite(m), m, 0.0)
            E = np.where(keep, np.exp(Sm - m), 0.0)
            ell = E.sum(axis=1, keepdims=True)
            P = np.divide(E, ell, out=np.zeros_like(E), where=ell > 0)
            lse[b, h] = np.where(has, m[:, 0] + np.log(np.where(has, ell[:, 0], 1.0)), -np.inf)
            o[b, h] = P @ V[b, hk]
            dvv[b, hk] += P.T @ dO[b, h]
            dP = dO[b, h] @ V[b, hk].T
            D = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, h] = scale * (dS @ K[b, hk])
            dk[b, hk] += scale * (dS.T @ Q[b, h])
    return dict(dq=dq, dk=dk, dv=dvv, o=o, lse=lse)


def backward_dq_rows(q, k, v, do, rows, *, scale, causal, skip, BM=BM_PREFILL, BN=BN_PREFILL, terms=False):
    """dQ of chosen query rows of the fixed-mask backward, each row on its own.

    A row's gradient needs only that row: its kept, visible scores S_c = scale
    q_r . k_c, its own lse over them, P = exp(S - lse), dP_c = dO_r . v_c,
    D = sum_c P_c dP_c, and dQ_r = scale * sum_c P_c (dP_c - D) k_c -- the same
    definition as attention_backward, restricted to one row (O(Lk * d) work),
    so it can be run at sizes where the whole matrix does not fit.
    rows: iterable of (b, hq, r).  skip as in attention_backward (None: dense).
    Returns float64 [len(rows), d]; with terms=True a dict with that ("dq") and,
    per row, the row's P and dS over all keys ([len(rows), Lk]) and O = P V
    ([len(rows), dv]), for tolerance models built from the same definition.
    """
    Q, K, V, dO = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    G = Hq // Hkv
    nq = (Lq + BM - 1) // BM
    nb = (Lk + BN - 1) // BN
    if skip is not None:
        skip = np.asarray(skip, dtype=np.uint8).reshape(B, Hq, nq, nb)
    cols = np.arange(Lk)
    out = np.zeros((len(rows), d))
    Ps = np.zeros((len(rows), Lk))
    dSs = np.zeros((len(rows), Lk))
    Os = np.zeros((len(rows), V.shape[3]))
    for n, (b, h, r) in enumerate(rows):
        hk = h // G
        keep = np.ones(Lk, bool)
        if causal:
            keep &= cols <= r + (Lk - Lq)
        if skip is not None:
            keep &= ~skip[b, h, r // BM][cols // BN].astype(bool)
        if not keep.any():
            continue
        s = scale * (K[b, hk] @ Q[b, h, r])
        m = s[keep].max()
        e = np.where(keep, np.exp(np.where(keep, s, m) - m), 0.0)
        p = e / e.sum()
        dp = V[b, hk] @ dO[b, h, r]
        dd = (p * dp).sum()
        ds = p * (dp - dd)
        out[n] = scale * (ds @ K[b, hk])
        Ps[n], dSs[n], Os[n] = p, ds, p @ V[b, hk]
    if terms:
        return dict(dq=out, P=Ps, dS=dSs, O=Os)
    return out
