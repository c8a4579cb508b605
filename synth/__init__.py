"""Seeded synthetic attention inputs (bf16 bit patterns as numpy uint16).

This module is shared by the tests, the bench and ``__graft_entry__.smoke()``:
it feeds the same bytes to the CUDA path and to the fp64 oracle. It holds no
attention arithmetic (no scores, softmax, maxima or skip rule) -- only random
numbers and the planted structure that stands in for real-model activations,
which the BLASST pages measure on (Llama-3.1-8B / Qwen3-8B attention, RULER and
LongBench; evaluation-setup table of the xllm-io review, section 5).

Planted-direction recipe (one generator for every workload shape):

* ``u`` -- a seeded unit vector per (batch, KV head), shared by all query heads
  of that KV head, so that grouped queries align with their keys.
* ``Q = Z + gamma*u`` on every query row.
* ``K = Z + gamma*u`` on the sink rows {0..3} and on a heavy set H (5% of keys),
  ``K = Z`` elsewhere.  ``V = Z``.  All Z are iid N(0, 1).
* Two readings of gamma and H (both are generated and run):
  - ``"lit"``: gamma = 3 raw and H an iid 5% of keys (the literal text);
  - ``"blk"``: gamma = sqrt(8/scale) (planted logit +8) and H = 5% of keys as
    64-aligned 64-key runs.  Only this reading reaches 50%/75% block sparsity.
* The "+2 boost on keys within 512 positions of the query" is put in the data,
  not in the kernel (the computed function stays softmax(QK^T*scale)V):
  - decode: w perpendicular to u, c = sqrt(2/scale); q += c*w and the last 512
    keys += c*w;
  - prefill: position segments of 256 keys; query i gets c*w[i//256], key j
    gets c*(w[j//256] + w[j//256 + 1]) with w[t] seeded unit vectors
    perpendicular to u, so a key in the query's own or previous segment gains
    about +2 logits.
* MLA (576 = 512 latent + 64 RoPE columns): u and w live in the 512 latent
  columns; the 64 RoPE columns are pure N(0, 1).

Every float is rounded once to bf16 (round-to-nearest-even) here; both paths
read those bytes.  Random streams are keyed by (seed, tensor, batch, head,
chunk) through numpy's SeedSequence/PCG64, so results do not depend on the
number of threads used.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "bf16_bits",
    "bf16_to_f32",
    "AttnInputs",
    "random_normal",
    "planted_prefill",
    "planted_decode",
    "planted_mla",
    "upstream_grad",
    "e4m3_bits",
    "e4m3_to_f32",
]

_TENSOR_ID = {"q": 1, "k": 2, "v": 3, "u": 4, "w": 5, "h": 6, "do": 7}
_CHUNK_ROWS = 1 << 14


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even) and return the uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class AttnInputs:
    """bf16 bit tensors [B, H, L, d] (uint16) plus the workload description."""

    q: np.ndarray
    k: np.ndarray
    v: np.ndarray | None
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, Hq, Lq, d = self.q.shape
        _, Hkv, Lk, dk = self.k.shape
        return B, Hq, Hkv, Lq, Lk, d


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, key)])))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _unit(g: np.ndarray) -> np.ndarray:
    return (g / np.linalg.norm(g)).astype(np.float64)


def _perp_unit(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    g = g.astype(np.float64)
    g = g - (g @ u) * u
    return g / np.linalg.norm(g)


def _fill(out: np.ndarray, seed: int, tid: int, add_fn=None) -> None:
    """out[B, H, L, d] (uint16) <- bf16(N(0,1) + add_fn(b, h, row0, z_chunk))."""
    B, H, L, d = out.shape
    jobs = [(b, h, r0) for b in range(B) for h in range(H) for r0 in range(0, L, _CHUNK_ROWS)]

    def work(job):
        b, h, r0 = job
        r1 = min(L, r0 + _CHUNK_ROWS)
        z = _rng(seed, tid, b, h, r0 // _CHUNK_ROWS).standard_normal((r1 - r0, d), dtype=np.float32)
        if add_fn is not None:
            add_fn(b, h, r0, z)
        out[b, h, r0:r1] = bf16_bits(z)

    if len(jobs) == 1:
        work(jobs[0])
        return
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, jobs))


def random_normal(B, Hq, Hkv, Lq, Lk, d, dv=None, seed=0, scale=None) -> AttnInputs:
    """Plain iid N(0,1) q, k, v (no planted structure)."""
    dv = d if dv is None else dv
    q = np.empty((B, Hq, Lq, d), np.uint16)
    k = np.empty((B, Hkv, Lk, d), np.uint16)
    v = np.empty((B, Hkv, Lk, dv), np.uint16)
    _fill(q, seed, _TENSOR_ID["q"])
    _fill(k, seed, _TENSOR_ID["k"])
    _fill(v, seed, _TENSOR_ID["v"])
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    return AttnInputs(q, k, v, scale, dict(kind="normal", seed=seed))


def _gamma(reading: str, scale: float) -> float:
    if reading == "lit":
        return 3.0
    if reading == "blk":
        return math.sqrt(8.0 / scale)
    raise ValueError(reading)


def _heavy_mask(reading: str, Lk: int, rng: np.random.Generator) -> np.ndarray:
    """Sinks {0..3} plus a 5% heavy set, per the reading."""
    m = np.zeros(Lk, dtype=bool)
    m[: min(4, Lk)] = True
    if reading == "lit":
        m |= rng.random(Lk) < 0.05
    else:
        runs = Lk // 64
        n = int(round(0.05 * runs))
        if n > 0:
            for r in rng.choice(runs, size=n, replace=False):
                m[r * 64 : (r + 1) * 64] = True
    return m


def planted_prefill(B, Hq, Hkv, L, d=128, seed=0, reading="lit", boost=True, scale=None) -> AttnInputs:
    """Prefill workload (Lq = Lk = L) with the planted-direction generator.

    ``boost=False`` gives the plain planted generator of the 1024-token MHA
    workload; ``boost=True`` adds the +2 logit segment boost of the GQA ones.
    """
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    G = Hq // Hkv
    gamma = _gamma(reading, scale)
    c = math.sqrt(2.0 / scale)
    nseg = (L + 255) // 256 + 1
    U = np.empty((B, Hkv, d))
    W = np.empty((B, Hkv, nseg, d))
    HM = np.empty((B, Hkv, L), dtype=bool)
    for b in range(B):
        for h in range(Hkv):
            r = _rng(seed, _TENSOR_ID["u"], b, h)
            U[b, h] = _unit(r.standard_normal(d))
            rw = _rng(seed, _TENSOR_ID["w"], b, h)
            for t in range(nseg):
                W[b, h, t] = _perp_unit(rw.standard_normal(d), U[b, h])
            HM[b, h] = _heavy_mask(reading, L, _rng(seed, _TENSOR_ID["h"], b, h))
    U32 = (gamma * U).astype(np.float32)
    CW = (c * W).astype(np.float32)

    def add_q(b, hq, r0, z):
        h = hq // G
        z += U32[b, h]
        if boost:
            idx = (np.arange(r0, r0 + z.shape[0]) // 256)
            z += CW[b, h][idx]

    def add_k(b, h, r0, z):
        rows = np.arange(r0, r0 + z.shape[0])
        z[HM[b, h, rows]] += U32[b, h]
        if boost:
            seg = rows // 256
            z += CW[b, h][seg] + CW[b, h][seg + 1]

    q = np.empty((B, Hq, L, d), np.uint16)
    k = np.empty((B, Hkv, L, d), np.uint16)
    v = np.empty((B, Hkv, L, d), np.uint16)
    _fill(q, seed, _TENSOR_ID["q"], add_q)
    _fill(k, seed, _TENSOR_ID["k"], add_k)
    _fill(v, seed, _TENSOR_ID["v"])
    meta = dict(kind="planted_prefill", reading=reading, boost=boost, seed=seed, gamma=gamma,
                heavy_fraction=float(HM.mean()))
    return AttnInputs(q, k, v, scale, meta)


def planted_decode(B, Hq, Hkv, Lk, d=128, Lq=1, seed=0, reading="lit", boost=True, scale=None) -> AttnInputs:
    """Decode workload (Lq query tokens per sequence, KV cache of Lk keys)."""
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    G = Hq // Hkv
    gamma = _gamma(reading, scale)
    c = math.sqrt(2.0 / scale)
    U = np.empty((B, Hkv, d))
    Wv = np.empty((B, Hkv, d))
    HM = np.empty((B, Hkv, Lk), dtype=bool)
    for b in range(B):
        for h in range(Hkv):
            U[b, h] = _unit(_rng(seed, _TENSOR_ID["u"], b, h).standard_normal(d))
            Wv[b, h] = _perp_unit(_rng(seed, _TENSOR_ID["w"], b, h).standard_normal(d), U[b, h])
            HM[b, h] = _heavy_mask(reading, Lk, _rng(seed, _TENSOR_ID["h"], b, h))
    U32 = (gamma * U).astype(np.float32)
    CW = (c * Wv).astype(np.float32)

    def add_q(b, hq, r0, z):
        h = hq // G
        z += U32[b, h]
        if boost:
            z += CW[b, h]

    def add_k(b, h, r0, z):
        rows = np.arange(r0, r0 + z.shape[0])
        z[HM[b, h, rows]] += U32[b, h]
        if boost:
            z[rows >= Lk - 512] += CW[b, h]

    q = np.empty((B, Hq, Lq, d), np.uint16)
    k = np.empty((B, Hkv, Lk, d), np.uint16)
    v = np.empty((B, Hkv, Lk, d), np.uint16)
    _fill(q, seed, _TENSOR_ID["q"], add_q)
    _fill(k, seed, _TENSOR_ID["k"], add_k)
    _fill(v, seed, _TENSOR_ID["v"])
    meta = dict(kind="planted_decode", reading=reading, boost=boost, seed=seed, gamma=gamma,
                heavy_fraction=float(HM.mean()))
    return AttnInputs(q, k, v, scale, meta)


def planted_mla(B, Hq, Lk, d_latent=512, d_rope=64, Lq=1, seed=0, reading="lit", boost=True,
                scale=None) -> AttnInputs:
    """MLA decode workload: one latent KV head of d_latent + d_rope columns.

    ``k`` is [B, 1, Lk, d_latent + d_rope]; V is the first d_latent columns of
    the same rows, so ``v`` is None and the caller passes k again with
    dv = d_latent and a row stride of d_latent + d_rope.
    """
    d = d_latent + d_rope
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    gamma = _gamma(reading, scale)
    c = math.sqrt(2.0 / scale)
    U = np.zeros((B, d))
    Wv = np.zeros((B, d))
    HM = np.empty((B, Lk), dtype=bool)
    for b in range(B):
        U[b, :d_latent] = _unit(_rng(seed, _TENSOR_ID["u"], b, 0).standard_normal(d_latent))
        Wv[b, :d_latent] = _perp_unit(_rng(seed, _TENSOR_ID["w"], b, 0).standard_normal(d_latent),
                                      U[b, :d_latent])
        HM[b] = _heavy_mask(reading, Lk, _rng(seed, _TENSOR_ID["h"], b, 0))
    U32 = (gamma * U).astype(np.float32)
    CW = (c * Wv).astype(np.float32)

    def add_q(b, hq, r0, z):
        z += U32[b]
        if boost:
            z += CW[b]

    def add_k(b, h, r0, z):
        rows = np.arange(r0, r0 + z.shape[0])
        z[HM[b, rows]] += U32[b]
        if boost:
            z[rows >= Lk - 512] += CW[b]

    q = np.empty((B, Hq, Lq, d), np.uint16)
    k = np.empty((B, 1, Lk, d), np.uint16)
    _fill(q, seed, _TENSOR_ID["q"], add_q)
    _fill(k, seed, _TENSOR_ID["k"], add_k)
    meta = dict(kind="planted_mla", reading=reading, boost=boost, seed=seed, gamma=gamma,
                d_latent=d_latent, d_rope=d_rope, heavy_fraction=float(HM.mean()))
    return AttnInputs(q, k, None, scale, meta)


def upstream_grad(B, Hq, Lq, dv=128, seed=0) -> np.ndarray:
    """Gradient of the attention output for the backward pass: iid N(0,1), bf16 bits."""
    do = np.empty((B, Hq, Lq, dv), np.uint16)
    _fill(do, seed, _TENSOR_ID["do"])
    return do


def e4m3_to_f32(b: np.ndarray) -> np.ndarray:
    """e4m3 bytes (OCP E4M3FN: sign, 4-bit exponent with bias 7, 3-bit mantissa, no
    infinities, S.1111.111 = NaN) -> float32 values, exactly."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int32)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((e == 15) & ((b & 7) == 7), np.nan, val)
    return (sign * val).astype(np.float32)


def e4m3_bits(x: np.ndarray) -> np.ndarray:
    """float values -> e4m3 bytes, round to nearest even, saturated at +-448 (torch's cast)."""
    import torch

    x = np.clip(np.asarray(x, dtype=np.float32), -448.0, 448.0)
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
