"""Pins of the fp64 oracle against what the BLASST pages and mathematics fix.

Every check here compares the oracle with something other than itself:
numpy brute force of the textbook attention formula, hand-derived golden
cases, the prefix-max closed form of the decision, monotonicity, the
skipped-mass identity and bound, split invariance and exact fit recovery.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from _brute import closed_form_decisions, dense_attention, masked_attention, widen
from synth import bf16_bits, planted_decode, planted_prefill, random_normal

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run(inp, lam, causal, **kw):
    return oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=lam, causal=causal, **kw)


# ---------------------------------------------------------------------------
# lambda = 0: textbook softmax(QK^T * scale) V and logsumexp, to 1e-9
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 1, 300, 300, 16), (2, 4, 2, 130, 130, 32), (1, 3, 3, 57, 57, 8)])
def test_dense_prefill_matches_bruteforce(shape, causal):
    B, Hq, Hkv, Lq, Lk, d = shape
    inp = random_normal(B, Hq, Hkv, Lq, Lk, d, seed=7)
    r = _run(inp, 0.0, causal, BM=64, BN=32)
    O, LSE = dense_attention(inp.q, inp.k, inp.v, inp.scale, causal)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)
    assert r["n_skipped"] == 0


@pytest.mark.parametrize("splits", [1, 3, 16])
@pytest.mark.parametrize("Lq,causal", [(1, False), (3, True)])
def test_dense_decode_matches_bruteforce(splits, Lq, causal):
    inp = random_normal(2, 8, 2, Lq, 700, 16, seed=11)
    r = _run(inp, 0.0, causal, is_decode=True, num_splits=splits, BN=64)
    O, LSE = dense_attention(inp.q, inp.k, inp.v, inp.scale, causal)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)


def test_dense_mla_strided_v_matches_bruteforce():
    # MLA-style: V is the first dv columns of the K rows (row stride d).
    B, Hq, Lk, d, dv = 1, 16, 200, 24, 16
    inp = random_normal(B, Hq, 1, 1, Lk, d, seed=3)
    r = oracle.attention(inp.q, inp.k, inp.k, scale=inp.scale, lam=0.0, causal=False, is_decode=True,
                         num_splits=3, BN=64, dv=dv, v_row_stride=d)
    O, LSE = dense_attention(inp.q, inp.k, inp.k, inp.scale, False, dv=dv)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)


def test_dense_config1_shape_matches_bruteforce():
    # the 1024-token MHA prefill shape with the planted generator, full size
    inp = planted_prefill(1, 1, 1, 1024, 128, seed=1, reading="lit", boost=False)
    r = _run(inp, 0.0, True)
    O, LSE = dense_attention(inp.q, inp.k, inp.v, inp.scale, True)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)
    assert r["n_visited"] == 36


# ---------------------------------------------------------------------------
# hand-built cases with exactly known block maxima (golden fixtures)
# ---------------------------------------------------------------------------
def _hand_inputs(c):
    Hq, Hkv, Lq, Lk = c["Hq"], c["Hkv"], c["Lq"], c["Lk"]
    d = 128
    q = np.zeros((1, Hq, Lq, d), np.float32)
    if c["mode"] == "decode":
        for g in range(Hq):
            q[0, g, :, c["q_axes"][g][0]] = 1.0
    else:
        for r in range(Lq):
            q[0, :, r, c["q_axes"][r][0]] = 1.0
    k = np.zeros((1, Hkv, Lk, d), np.float32)
    for j, coords in enumerate(c["key_coords"]):
        k[0, :, j, : len(coords)] = coords
    if c.get("v_onehot"):
        v = np.zeros((1, Hkv, Lk, d), np.float32)
        for j in range(Lk):
            v[0, :, j, j] = 1.0
    else:
        v = np.random.default_rng(0).standard_normal((1, Hkv, Lk, d)).astype(np.float32)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    # the chosen values are exact in bf16
    assert np.array_equal(widen(kb), k.astype(np.float64))
    return qb, kb, vb


def _hand_cases():
    with open(os.path.join(GOLDEN, "hand_cases.json")) as f:
        data = json.load(f)
    for c in data["cases"]:
        for cl in c["cases_lambda"]:
            yield pytest.param(c, cl, id=f"{c['name']}-{cl.get('ln_lambda', cl.get('lambda'))}")


@pytest.mark.parametrize("case,cl", list(_hand_cases()))
def test_hand_cases(case, cl):
    q, k, v = _hand_inputs(case)
    lam = math.exp(cl["ln_lambda"]) if "ln_lambda" in cl else cl["lambda"]
    r = oracle.attention(q, k, v, scale=1.0, lam=lam, causal=case["causal"],
                         is_decode=case["mode"] == "decode", num_splits=case.get("num_splits", 1),
                         BM=case["BM"], BN=case["BN"], seed_splits=case.get("seed_splits", False))
    assert r["skip"].tolist() == cl["skip"]
    assert r["visited"].tolist() == cl["visited"]
    if "lse" in cl:
        np.testing.assert_allclose(r["lse"].ravel(), cl["lse"], atol=1e-12)
    if "o_row0" in cl:
        np.testing.assert_allclose(r["o"][0, 0, 0, : len(cl["o_row0"])], cl["o_row0"], atol=1e-12)


def test_forced_mask_rejects_first_block():
    inp = random_normal(1, 1, 1, 64, 256, 8, seed=1)
    nb = 4
    forced = np.zeros((1, nb), np.uint8)
    forced[0, 0] = 1
    with pytest.raises(ValueError):
        _run(inp, 0.0, False, BM=64, BN=64, forced_skip=forced)


# ---------------------------------------------------------------------------
# the decision is a function of per-block maxima only (prefix-max form)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lam", [1e-4, 4 / 512, 0.05, 0.3, 0.9])
def test_mask_equals_prefix_max_closed_form_prefill(lam):
    inp = planted_prefill(1, 4, 2, 512, 32, seed=5, reading="blk", boost=True)
    r = _run(inp, lam, True, BM=64, BN=32)
    skip, vis = closed_form_decisions(inp.q, inp.k, inp.scale, True, lam, 64, 32)
    assert np.array_equal(r["visited"], vis)
    assert np.array_equal(r["skip"], skip)
    assert r["n_skipped"] == int(skip.sum()) and r["n_visited"] == int(vis.sum())


@pytest.mark.parametrize("lam", [1e-3, 0.02, 0.2])
@pytest.mark.parametrize("splits", [1, 4])
def test_mask_equals_prefix_max_closed_form_decode(lam, splits):
    inp = planted_decode(2, 8, 2, 1024, 32, Lq=2, seed=9, reading="blk")
    r = _run(inp, lam, True, is_decode=True, num_splits=splits, BN=64)
    skip, vis = closed_form_decisions(inp.q, inp.k, inp.scale, True, lam, 128, 64, is_decode=True,
                                      num_splits=splits)
    assert np.array_equal(r["visited"], vis)
    assert np.array_equal(r["skip"], skip)


def test_outputs_equal_masked_softmax():
    # with lambda > 0 the output is exactly softmax over the keys of kept blocks
    inp = planted_prefill(1, 2, 1, 400, 32, seed=2, reading="blk", boost=True)
    r = _run(inp, 0.05, True, BM=64, BN=32)
    assert r["n_skipped"] > 0
    O, LSE = masked_attention(inp.q, inp.k, inp.v, inp.scale, True, r["skip"], 64, 32)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)


def test_decode_outputs_equal_masked_softmax_across_splits():
    inp = planted_decode(1, 4, 1, 2048, 32, seed=4, reading="blk")
    r = _run(inp, 0.05, False, is_decode=True, num_splits=4, BN=64)
    assert r["n_skipped"] > 0
    O, LSE = masked_attention(inp.q, inp.k, inp.v, inp.scale, False, r["skip"], 128, 64, is_decode=True)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)


# ---------------------------------------------------------------------------
# monotonicity: lambda1 <= lambda2 implies skipset(lambda1) within skipset(lambda2)
# ---------------------------------------------------------------------------
def test_skip_sets_nested_in_lambda():
    inp = planted_prefill(1, 2, 1, 768, 32, seed=8, reading="blk", boost=True)
    prev = None
    counts = []
    for lam in [0.0, 1e-6, 1e-4, 1e-3, 0.01, 0.1, 0.5, 0.99]:
        r = _run(inp, lam, True, BM=64, BN=32)
        if prev is not None:
            assert np.all(prev <= r["skip"])
        prev = r["skip"]
        counts.append(r["n_skipped"])
    assert counts == sorted(counts) and counts[-1] > 0


# ---------------------------------------------------------------------------
# skipped-mass identity and a priori bound
# ---------------------------------------------------------------------------
def test_skipped_mass_identity_and_bound():
    lam = 0.02
    BM, BN = 64, 32
    inp = planted_prefill(1, 2, 1, 512, 32, seed=12, reading="blk", boost=True)
    sp = _run(inp, lam, True, BM=BM, BN=BN)
    dn = _run(inp, 0.0, True, BM=BM, BN=BN)
    assert sp["n_skipped"] > 0
    B, Hq, Lq, _ = inp.q.shape
    Lk = inp.k.shape[2]
    from _brute import score_matrix, tile_rows
    for tile in range(sp["skip"].shape[0]):
        b, rows = tile_rows(False, Hq, 1, Lq, BM, tile)
        skipped_keys = np.repeat(sp["skip"][tile] == 1, BN)[:Lk]
        for hq, pos in rows:
            s = score_matrix(inp.q, inp.k, inp.scale, True, b, hq, Hq)[pos]
            p = np.exp(s - s.max())
            p /= p.sum()
            eps = p[skipped_keys].sum()
            V = widen(inp.v[b, 0])
            if eps > 0:
                o_skip = (p[skipped_keys] @ V[skipped_keys]) / eps
            else:
                o_skip = np.zeros(V.shape[1])
            od, osp = dn["o"][b, hq, pos], sp["o"][b, hq, pos]
            np.testing.assert_allclose(od, (1 - eps) * osp + eps * o_skip, atol=1e-12, rtol=0)
            assert abs((dn["lse"][b, hq, pos] - sp["lse"][b, hq, pos]) + math.log1p(-eps)) < 1e-12
            n_sk = int(np.count_nonzero(skipped_keys & np.isfinite(s)))
            assert eps <= lam * n_sk + 1e-15
            assert np.max(np.abs(od - osp)) <= 2 * eps * np.max(np.abs(V)) + 1e-12


# ---------------------------------------------------------------------------
# split invariance at lambda = 0
# ---------------------------------------------------------------------------
def test_split_invariance_dense():
    inp = planted_decode(2, 8, 2, 1500, 32, seed=6, reading="lit")
    base = _run(inp, 0.0, False, is_decode=True, num_splits=1)
    for s in (2, 5, 16, 40):
        r = _run(inp, 0.0, False, is_decode=True, num_splits=s)
        np.testing.assert_allclose(r["o"], base["o"], atol=1e-12, rtol=0)
        np.testing.assert_allclose(r["lse"], base["lse"], atol=1e-12, rtol=0)


def test_splits_restart_running_max():
    # with several splits each split keeps its own first block
    inp = planted_decode(1, 4, 1, 64 * 32, 32, seed=6, reading="blk")
    r = _run(inp, 0.999, False, is_decode=True, num_splits=4)
    firsts = r["skip"][0, ::8]
    assert np.all(firsts == 0)
    assert r["n_skipped"] > 0


# ---------------------------------------------------------------------------
# split seeding (decode): later splits start their running max at block 0's maxima
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("splits", [2, 5, 16])
def test_seeded_dense_decode_matches_bruteforce(splits):
    # at lambda = 0 nothing is skipped: the seed only moves the exp reference
    inp = planted_decode(2, 8, 2, 1500, 32, Lq=2, seed=21, reading="blk")
    r = _run(inp, 0.0, True, is_decode=True, num_splits=splits, seed_splits=True)
    O, LSE = dense_attention(inp.q, inp.k, inp.v, inp.scale, True)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)


@pytest.mark.parametrize("lam", [1e-3, 0.02, 0.2, 0.9])
@pytest.mark.parametrize("splits", [2, 4, 16])
def test_seeded_mask_equals_prefix_max_closed_form(lam, splits):
    inp = planted_decode(2, 8, 2, 1024, 32, Lq=2, seed=9, reading="blk")
    r = _run(inp, lam, True, is_decode=True, num_splits=splits, BN=64, seed_splits=True)
    skip, vis = closed_form_decisions(inp.q, inp.k, inp.scale, True, lam, 128, 64, is_decode=True,
                                      num_splits=splits, seed_splits=True)
    assert np.array_equal(r["visited"], vis)
    assert np.array_equal(r["skip"], skip)


@pytest.mark.parametrize("splits", [3, 8])
def test_seeded_mask_equals_prefix_max_closed_form_wide_tile(splits):
    # a 64-row tile (64 query heads on one KV head, the shape of the tcgen05 decode): every row's
    # prefix max, block 0 included, must allow the skip
    inp = planted_decode(1, 64, 1, 2048, 32, seed=19, reading="blk")
    for lam in (0.05, 0.3, 0.9):
        r = _run(inp, lam, False, is_decode=True, num_splits=splits, BN=64, seed_splits=True)
        skip, vis = closed_form_decisions(inp.q, inp.k, inp.scale, False, lam, 128, 64, is_decode=True,
                                          num_splits=splits, seed_splits=True)
        assert np.array_equal(r["visited"], vis)
        assert np.array_equal(r["skip"], skip)


def test_seeded_outputs_equal_masked_softmax():
    # block 0 enters later splits only through its maxima, never through l or O
    inp = planted_decode(1, 4, 1, 2048, 32, seed=4, reading="blk")
    r = _run(inp, 0.05, False, is_decode=True, num_splits=8, BN=64, seed_splits=True)
    assert r["n_skipped"] > 0
    O, LSE = masked_attention(inp.q, inp.k, inp.v, inp.scale, False, r["skip"], 128, 64, is_decode=True)
    np.testing.assert_allclose(r["o"], O, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["lse"], LSE, atol=1e-9, rtol=0)


def test_seeded_one_split_is_unseeded():
    inp = planted_decode(2, 8, 2, 1024, 32, seed=3, reading="blk")
    a = _run(inp, 0.1, False, is_decode=True, num_splits=1, seed_splits=True)
    b = _run(inp, 0.1, False, is_decode=True, num_splits=1)
    assert np.array_equal(a["skip"], b["skip"])
    np.testing.assert_array_equal(a["o"], b["o"])


@pytest.mark.parametrize("lam", [0.005, 0.05, 0.5])
def test_seeded_skips_contain_unseeded(lam):
    # the seed can only raise the running max, so every gap shrinks or stays
    inp = planted_decode(2, 8, 2, 4096, 32, seed=11, reading="blk")
    a = _run(inp, lam, False, is_decode=True, num_splits=16, seed_splits=True)
    b = _run(inp, lam, False, is_decode=True, num_splits=16)
    assert np.all(b["skip"] <= a["skip"])
    assert a["n_skipped"] > b["n_skipped"]


# ---------------------------------------------------------------------------
# calibration: lambda * L = alpha * exp(beta * s)
# ---------------------------------------------------------------------------
def test_calibrate_fit_recovers_exact_points():
    alpha, beta = 3.7, 6.25
    Ls = np.array([8192, 16384, 32768, 65536, 8192, 32768], float)
    s = np.array([0.3, 0.4, 0.5, 0.6, 0.7, 0.8])
    lam = alpha * np.exp(beta * s) / Ls
    a, b = oracle.calibrate_fit(Ls, lam, s)
    assert abs(a - alpha) < 1e-9 and abs(b - beta) < 1e-9


def test_calibrate_fit_matches_polyfit_on_noisy_points():
    rng = np.random.default_rng(0)
    s = rng.uniform(0.2, 0.9, 40)
    Ls = rng.choice([8192, 16384, 32768, 65536], 40).astype(float)
    lam = 2.0 * np.exp(5.0 * s + rng.normal(0, 0.1, 40)) / Ls
    a, b = oracle.calibrate_fit(Ls, lam, s)
    pb, pa = np.polyfit(s, np.log(lam * Ls), 1)
    assert abs(b - pb) < 1e-9 and abs(math.log(a) - pa) < 1e-9


def test_threshold_for_sparsity_hits_count():
    inp = planted_prefill(1, 2, 1, 1024, 32, seed=13, reading="blk", boost=True)
    r0 = _run(inp, 0.0, True, BM=64, BN=32)
    for target in (0.3, 0.5, 0.6):
        lam, ach = oracle.threshold_for_sparsity(r0["gaps"], r0["visited"], target)
        r = _run(inp, lam, True, BM=64, BN=32)
        assert abs(r["n_skipped"] / r["n_visited"] - ach) < 1e-12
        assert abs(ach - target) <= 1.0 / r["n_visited"] + 1e-12 or ach < target
