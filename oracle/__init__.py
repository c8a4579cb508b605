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
