"""Helpers for GPU-vs-oracle parity (tests only).

Tolerances (a thresholded approximation compared with its fp64 oracle):
  * skip masks bit-equal except pairs whose oracle gap lies within 1e-3 of
    ln(lambda) (the device decides in fp32, log2 units);
  * outputs compared with the oracle run on the DEVICE's mask (forced-mask
    mode): max-abs <= 1e-2, mean-abs <= 1e-3 (bf16 in/out, fp32 accumulate;
    half a bf16 ulp is 0.0078 for |O| in [2, 4));
  * lse (natural log) within 1e-3.
"""
from __future__ import annotations

import math

import numpy as np

MASK_BAND = 1e-3
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_ABS = 1e-3


def unpack_mask(words, nb):
    """int32 words [rows, W] -> uint8 bits [rows, nb] (bit j%32 of word j//32)."""
    w = np.asarray(words).astype(np.uint32)
    rows = w.shape[0]
    bits = np.zeros((rows, w.shape[1] * 32), np.uint8)
    for b in range(32):
        bits[:, b::32] = (w >> np.uint32(b)) & np.uint32(1)
    return bits[:, :nb]


def bf16_tensor_to_f64(t):
    import torch

    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def compare_masks(gpu_bits, ref, lam, tiles=None):
    """Returns (n_diff_outside_band, n_in_band).  ref = oracle result dict."""
    g = gpu_bits if tiles is None else gpu_bits[np.asarray(tiles)]
    r_skip = ref["skip"] if tiles is None else ref["skip"][np.asarray(tiles)]
    r_gap = ref["gaps"] if tiles is None else ref["gaps"][np.asarray(tiles)]
    r_vis = ref["visited"] if tiles is None else ref["visited"][np.asarray(tiles)]
    if lam > 0:
        band = np.isfinite(r_gap) & (np.abs(r_gap - math.log(lam)) <= MASK_BAND)
    else:
        band = np.zeros_like(r_gap, dtype=bool)
    diff = (g != r_skip)
    assert not np.any(g[r_vis == 0]), "device marked an unvisited pair as skipped"
    return int(np.count_nonzero(diff & ~band)), int(np.count_nonzero(band))


def assert_outputs_close(o_gpu, lse_gpu, o_ref, lse_ref, rows=None, one_hot=False):
    """o_gpu/lse_gpu numpy f64 arrays; rows: optional boolean/index selection.

    one_hot=True is for the hand-built cases whose softmax rows are nearly
    one-hot, so |O| ~ |v| ~ 1: there bf16 output rounding alone averages about
    a quarter ulp (~2e-3 in [1, 2)) and a 1e-3 mean bound cannot hold.  Each
    element must then be within one bf16 ulp of the fp64 value plus the
    rounding of P to bf16 (2^-9 relative, times max |v| <= 4), and max-abs
    stays <= 1e-2.
    """
    if rows is not None:
        o_gpu, o_ref = o_gpu[rows], o_ref[rows]
        lse_gpu, lse_ref = lse_gpu[rows], lse_ref[rows]
    err = np.abs(o_gpu - o_ref)
    assert np.all(np.isfinite(o_gpu)), "non-finite output"
    if one_hot:
        mag = np.maximum(np.abs(o_ref), 2.0 ** -14)
        ulp = np.exp2(np.floor(np.log2(mag)) - 7)
        assert np.all(err <= ulp + 4 * 2.0 ** -9), "element off by more than 1 ulp + P rounding"
        assert err.max() <= O_MAX_ABS, f"max-abs {err.max():.3e}"
        assert np.abs(lse_gpu - lse_ref).max() <= LSE_ABS
        return float(err.max()), float(err.mean()), float(np.abs(lse_gpu - lse_ref).max())
    big = np.abs(o_ref) >= 4.0
    if np.any(big):
        # beyond |O| = 4 half a bf16 ulp exceeds the absolute bound: 1 ulp there
        ulp = np.exp2(np.floor(np.log2(np.abs(o_ref[big]))) - 7)
        assert np.all(err[big] <= ulp), "large-|O| element off by more than one bf16 ulp"
        err = np.where(big, 0.0, err)
    assert err.max() <= O_MAX_ABS, f"max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"mean-abs {err.mean():.3e}"
    lerr = np.abs(lse_gpu - lse_ref)
    assert lerr.max() <= LSE_ABS, f"lse max-abs {lerr.max():.3e}"
    return float(err.max()), float(err.mean()), float(lerr.max())
