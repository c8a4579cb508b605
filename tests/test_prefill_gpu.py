"""GPU parity of blasst_prefill / blasst_calibrate (tcgen05, 128x128 tiles) against the fp64 oracle."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from _parity import assert_outputs_close, bf16_tensor_to_f64, compare_masks, unpack_mask
from synth import AttnInputs, bf16_bits, planted_prefill, random_normal

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def bl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_tcgen05_b200 as m

    m.lib()
    return m


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def check_prefill(bl, inp, lam, causal, tiles=None, one_hot=False):
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, mask, cnt = bl.prefill(q, k, v, scale=inp.scale, lam=lam, causal=causal, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0, "device wait timed out"
    B, Hq, Lq, d = inp.q.shape
    Lk = inp.k.shape[2]
    nb = (Lk + 127) // 128
    bits = unpack_mask(mask.cpu().numpy(), nb)
    assert int(cnt.item()) == int(bits.sum())
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=lam, causal=causal, tiles=tiles)
    nd, nband = compare_masks(bits, ref, lam, tiles)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=lam, causal=causal, tiles=tiles,
                          forced_skip=bits)
    og = bf16_tensor_to_f64(o)
    lg = lse.cpu().numpy().astype(np.float64)
    rows = None
    if tiles is not None:
        nq = (Lq + 127) // 128
        sel = np.zeros((B, Hq, Lq), bool)
        for t in tiles:
            bh, qt = divmod(int(t), nq)
            b, h = divmod(bh, Hq)
            sel[b, h, qt * 128:(qt + 1) * 128] = True
        rows = sel
    assert_outputs_close(og, lg, fr["o"], fr["lse"], rows, one_hot=one_hot)
    return bits, ref


def test_prefill_single_tile(bl):
    inp = random_normal(1, 1, 1, 128, 128, 128, seed=1)
    check_prefill(bl, inp, 0.0, False)


def test_prefill_one_pair_causal(bl):
    inp = random_normal(1, 1, 1, 256, 256, 128, seed=2)
    check_prefill(bl, inp, 0.0, True)


@pytest.mark.parametrize("lam", [0.0, 4 / 1024, 32 / 1024])
def test_prefill_mha_1024_planted(bl, lam):
    # B=1, H=1, L=1024, causal, literal planted generator (no boost)
    inp = planted_prefill(1, 1, 1, 1024, 128, seed=1, reading="lit", boost=False)
    bits, ref = check_prefill(bl, inp, lam, True)
    assert ref["n_visited"] == 36


@pytest.mark.parametrize("lam", [0.0, 1e-4, 0.01, 0.1, 0.5, 0.999])
def test_prefill_gqa_blk(bl, lam):
    inp = planted_prefill(1, 8, 2, 1536, 128, seed=3, reading="blk")
    bits, _ = check_prefill(bl, inp, lam, True)
    if lam == 0.0:
        assert bits.sum() == 0


@pytest.mark.parametrize("shape", [(2, 4, 2, 300, 300, True), (1, 2, 1, 200, 700, False),
                                   (1, 2, 2, 256, 640, True), (1, 3, 3, 129, 129, True),
                                   (1, 2, 1, 640, 640, False)])
@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_prefill_ragged_and_rectangular(bl, shape, lam):
    B, Hq, Hkv, Lq, Lk, causal = shape
    inp = random_normal(B, Hq, Hkv, Lq, Lk, 128, seed=4)
    check_prefill(bl, inp, lam, causal)


def test_prefill_odd_tile_count(bl):
    # 5 query tiles: the last CTA holds a single tile
    inp = planted_prefill(1, 2, 1, 640, 128, seed=5, reading="blk")
    check_prefill(bl, inp, 0.02, True)


def _expanded_hand_case(name, BN=128):
    with open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")) as f:
        case = [c for c in json.load(f)["cases"] if c["name"] == name][0]
    nkeys = len(case["key_coords"])
    bn0 = case["BN"]  # keys per block in the hand case; each block becomes one BN-key block
    Lk = (nkeys // bn0) * BN
    d = 128
    Lq = case["Lq"]
    q = np.zeros((1, 1, Lq, d), np.float32)
    for r in range(Lq):
        q[0, 0, r, case["q_axes"][r][0]] = 1.0
    k = np.full((1, 1, Lk, d), -64.0, np.float32)
    for j, coords in enumerate(case["key_coords"]):
        k[0, 0, (j // bn0) * BN + j % bn0, : len(coords)] = coords
    v = np.random.default_rng(0).standard_normal((1, 1, Lk, d)).astype(np.float32)
    return case, AttnInputs(bf16_bits(q), bf16_bits(k), bf16_bits(v), 1.0)


@pytest.mark.parametrize("name", ["one_row_four_blocks", "two_rows_one_row_keeps", "lambda_near_one"])
def test_prefill_hand_cases_exact(bl, name):
    # each hand key becomes a 128-key block whose other keys score -64: block maxima are exact
    case, inp = _expanded_hand_case(name)
    for cl in case["cases_lambda"]:
        lam = math.exp(cl["ln_lambda"]) if "ln_lambda" in cl else cl["lambda"]
        bits, _ = check_prefill(bl, inp, lam, False, one_hot=True)
        assert bits.tolist() == cl["skip"]


def test_prefill_calibrate_matches_prefill(bl):
    inp = planted_prefill(1, 4, 2, 2048, 128, seed=6, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    gaps, mc, cc = bl.calibrate(q, k, scale=inp.scale, lam=0.03, causal=True, mode="prefill")
    _, _, mp, cp = bl.prefill(q, k, v, scale=inp.scale, lam=0.03, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(mc, mp) and torch.equal(cc, cp)
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.03, causal=True)
    g = gaps.cpu().numpy().astype(np.float64)
    vis = ref["visited"] == 1
    assert np.array_equal(np.isnan(g), ~vis)
    assert np.array_equal(np.isinf(g), np.isinf(ref["gaps"]) & vis)
    fin = np.isfinite(ref["gaps"]) & vis
    assert np.max(np.abs(g[fin] - ref["gaps"][fin])) < 1e-3
    # the threshold picked from device gaps reproduces its target on the device
    lam, ach = bl.calibrate_threshold(gaps.cpu().numpy(), 0.5)
    _, _, m2, c2 = bl.prefill(q, k, v, scale=inp.scale, lam=lam, causal=True)
    torch.cuda.synchronize()
    assert abs(c2.item() / ref["n_visited"] - ach) < 1e-9


def test_prefill_lambda_monotone_counts(bl):
    inp = planted_prefill(1, 4, 1, 2048, 128, seed=7, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    prev_bits = None
    for lam in [0.0, 1e-5, 1e-3, 0.01, 0.1, 0.5, 0.99]:
        _, _, m, _ = bl.prefill(q, k, v, scale=inp.scale, lam=lam, causal=True)
        torch.cuda.synchronize()
        bits = unpack_mask(m.cpu().numpy(), 16)
        if prev_bits is not None:
            assert np.all(prev_bits <= bits)
        prev_bits = bits


def test_prefill_invalid_arguments(bl):
    inp = random_normal(1, 2, 1, 256, 256, 128, seed=0)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    for lam in (-1e-3, 1.0, float("nan")):
        with pytest.raises(bl.BlasstError) as e:
            bl.prefill(q, k, v, scale=inp.scale, lam=lam)
        assert e.value.status == 1
    qs = to_dev(random_normal(1, 2, 1, 300, 256, 128).q)
    with pytest.raises(bl.BlasstError) as e:
        bl.prefill(qs, k, v, scale=inp.scale, lam=0.0, causal=True)  # Lq > Lk with causal
    assert e.value.status == 1


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 2e-3])
def test_prefill_full_size_sampled(bl, lam):
    # the benchmarked launch: B=1, Hq=32, Hkv=8, L=32768, causal; oracle on sampled tiles
    inp = planted_prefill(1, 32, 8, 32768, 128, seed=2, reading="blk")
    rng = np.random.default_rng(1)
    nq = 256
    tiles = np.sort(np.concatenate([rng.choice(32 * nq, 6, replace=False), [nq - 1, 31 * nq + nq - 1]]))
    check_prefill(bl, inp, lam, True, tiles=tiles)


@pytest.mark.slow
def test_prefill_64k_sampled(bl):
    # the long-context launch: B=1, Hq=32, Hkv=8, L=65536, causal; oracle on sampled tiles
    inp = planted_prefill(1, 32, 8, 65536, 128, seed=4, reading="blk")
    nq = 512
    tiles = [nq - 1, 5 * nq + 200, 17 * nq + 3, 31 * nq + nq - 1]
    check_prefill(bl, inp, 3e-3, True, tiles=tiles)


def test_prefill_novote_instance_equals_dense_prefill(bl):
    # the measurement instance (decision compiled out) computes, at lambda = 0,
    # exactly what the real kernel computes there: nothing is skipped by either
    inp = planted_prefill(1, 4, 2, 1000, 128, seed=8, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    o1, l1, m1, c1 = bl.prefill(q, k, v, scale=inp.scale, lam=0.0, causal=True)
    o2, l2, m2, c2 = bl.measure_prefill_novote(q, k, v, scale=inp.scale, lam=0.0, causal=True)
    torch.cuda.synchronize()
    assert int(c1.item()) == 0 and int(c2.item()) == 0
    assert torch.equal(m1, m2) and torch.equal(o1, o2) and torch.equal(l1, l2)
    check_prefill(bl, inp, 0.0, True)
