"""GPU parity of blasst_decode (split-KV, 64-key blocks) against the fp64 oracle."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from _parity import assert_outputs_close, bf16_tensor_to_f64, compare_masks, unpack_mask
from synth import bf16_bits, planted_decode, random_normal

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


def check_decode(bl, inp, lam, causal, splits, tiles=None, band_ok=True, one_hot=False, seed_splits=False):
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    o, lse, mask, cnt = bl.decode(q, k, v, scale=inp.scale, lam=lam, causal=causal, num_splits=splits,
                                  seed_splits=seed_splits)
    torch.cuda.synchronize()
    B, Hq, Lq, d = inp.q.shape
    Hkv, Lk = inp.k.shape[1], inp.k.shape[2]
    nb = (Lk + 63) // 64
    bits = unpack_mask(mask.cpu().numpy(), nb)
    assert int(cnt.item()) == int(bits.sum())
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=lam, causal=causal, is_decode=True,
                           num_splits=splits, BN=64, tiles=tiles, seed_splits=seed_splits)
    nd, nband = compare_masks(bits, ref, lam, tiles)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    if not band_ok:
        assert nband == 0
    forced = bits.copy()
    fr = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=lam, causal=causal, is_decode=True,
                          num_splits=splits, BN=64, tiles=tiles, forced_skip=forced, seed_splits=seed_splits)
    og = bf16_tensor_to_f64(o)
    lg = lse.cpu().numpy().astype(np.float64)
    rows = None
    if tiles is not None:
        G = Hq // Hkv
        sel = np.zeros((B, Hq, Lq), bool)
        for t in tiles:
            b, h = divmod(int(t), Hkv)
            sel[b, h * G:(h + 1) * G, :] = True
        rows = sel
    assert_outputs_close(og, lg, fr["o"], fr["lse"], rows, one_hot=one_hot)
    return bits, ref


@pytest.mark.parametrize("lam", [0.0, 1e-3, 0.05, 0.5, 0.999])
@pytest.mark.parametrize("reading", ["blk", "lit"])
def test_decode_gqa_small(bl, lam, reading):
    inp = planted_decode(2, 8, 2, 64 * 37 + 13, 128, seed=21, reading=reading)
    bits, ref = check_decode(bl, inp, lam, False, 4)
    if lam == 0.0:
        assert bits.sum() == 0


@pytest.mark.parametrize("lam", [0.0, 0.02])
def test_decode_random_normal(bl, lam):
    inp = random_normal(3, 4, 4, 1, 1000, 128, seed=5)
    check_decode(bl, inp, lam, False, 16)


@pytest.mark.parametrize("lam", [0.0, 0.1])
def test_decode_two_ntiles_causal(bl, lam):
    # G * Lq = 16 rows: the wider tile variant, causal with Lq = 2
    inp = planted_decode(1, 8, 1, 3000, 128, Lq=2, seed=3, reading="blk")
    check_decode(bl, inp, lam, True, 3)


def test_decode_short_cache_many_empty_splits(bl):
    inp = planted_decode(2, 4, 1, 50, 128, seed=8, reading="lit")
    check_decode(bl, inp, 0.3, False, 16)


def test_decode_single_split_long(bl):
    inp = planted_decode(1, 4, 1, 64 * 200, 128, seed=9, reading="blk")
    bits, _ = check_decode(bl, inp, 0.05, False, 1)
    assert bits.sum() > 0


def test_decode_lambda_zero_matches_textbook(bl):
    # lambda = 0 against the dense definition directly (oracle dense == brute force, pinned on CPU)
    inp = random_normal(2, 8, 2, 1, 777, 128, seed=1)
    check_decode(bl, inp, 0.0, False, 5)


def _expanded_hand_case(name, BN):
    with open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")) as f:
        case = [c for c in json.load(f)["cases"] if c["name"] == name][0]
    nkeys = len(case["key_coords"])
    bn0 = case["BN"]  # keys per block in the hand case; each block becomes one BN-key block
    Lk = (nkeys // bn0) * BN
    d = 128
    Hq, Hkv = case["Hq"], case["Hkv"]
    q = np.zeros((1, Hq, 1, d), np.float32)
    for g in range(Hq):
        q[0, g, 0, case["q_axes"][g][0] if case["mode"] == "decode" else case["q_axes"][0][0]] = 1.0
    k = np.full((1, Hkv, Lk, d), -64.0, np.float32)
    for j, coords in enumerate(case["key_coords"]):
        k[0, :, (j // bn0) * BN + j % bn0, : len(coords)] = coords
    v = np.random.default_rng(0).standard_normal((1, Hkv, Lk, d)).astype(np.float32)
    return case, bf16_bits(q), bf16_bits(k), bf16_bits(v)


@pytest.mark.parametrize("name", ["one_row_four_blocks", "decode_group_two_splits", "lambda_near_one"])
def test_decode_hand_cases_exact(bl, name):
    # each hand key becomes a 64-key block whose other keys score -64: block maxima are exact
    case, q, k, v = _expanded_hand_case(name, 64)
    from synth import AttnInputs

    inp = AttnInputs(q, k, v, 1.0)
    splits = case.get("num_splits", 1)
    for cl in case["cases_lambda"]:
        lam = math.exp(cl["ln_lambda"]) if "ln_lambda" in cl else cl["lambda"]
        bits, ref = check_decode(bl, inp, lam, False, splits, one_hot=True)
        assert bits.tolist() == cl["skip"]


def test_decode_invalid_arguments(bl):
    inp = random_normal(1, 4, 1, 1, 256, 128, seed=0)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    for lam in (-0.1, 1.0, float("nan"), float("inf")):
        with pytest.raises(bl.BlasstError) as e:
            bl.decode(q, k, v, scale=inp.scale, lam=lam)
        assert e.value.status == 1
    with pytest.raises(bl.BlasstError) as e:
        bl.decode(q, k, v, scale=-1.0, lam=0.0)
    assert e.value.status == 1
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(bl.BlasstError) as e:
        bl.decode(q, k, v, scale=inp.scale, lam=0.0, workspace=ws)
    assert e.value.status == 3


def test_decode_caller_workspace_and_status_word(bl):
    inp = planted_decode(2, 8, 2, 4000, 128, seed=2, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    nbytes = bl.decode_workspace_bytes(2, 8, 1, 128, 16)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1, m1, c1 = bl.decode(q, k, v, scale=inp.scale, lam=0.05, workspace=ws, status_word=st)
    o2, l2, m2, c2 = bl.decode(q, k, v, scale=inp.scale, lam=0.05)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(m1, m2) and torch.equal(c1, c2)


def test_decode_calibrate_matches_decode_masks(bl):
    inp = planted_decode(2, 8, 2, 5000, 128, seed=4, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    gaps, mc, cc = bl.calibrate(q, k, scale=inp.scale, lam=0.05, mode="decode", num_splits=4)
    _, _, md, cd = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=4)
    torch.cuda.synchronize()
    assert torch.equal(mc, md) and torch.equal(cc, cd)
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.05, causal=False, is_decode=True,
                           num_splits=4, BN=64)
    g = gaps.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref["gaps"])
    assert np.array_equal(np.isinf(g), np.isinf(ref["gaps"]))
    assert np.max(np.abs(g[fin] - ref["gaps"][fin])) < 1e-3


# ----------------------------------------------- wide tiles (17..128 rows, tcgen05)
@pytest.mark.parametrize("lam", [0.0, 1e-3, 0.05, 0.5])
@pytest.mark.parametrize("splits", [1, 4, 16])
def test_decode_mqa_32_heads(bl, lam, splits):
    inp = planted_decode(2, 32, 1, 64 * 41 + 13, 128, seed=51, reading="blk")
    bits, _ = check_decode(bl, inp, lam, False, splits)
    if lam == 0.0:
        assert bits.sum() == 0


@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_decode_mqa_128_heads(bl, lam):
    # every TMEM lane is a row
    inp = planted_decode(2, 128, 1, 3000, 128, seed=52, reading="blk")
    check_decode(bl, inp, lam, False, 4)


def test_decode_gqa_group_32(bl):
    inp = planted_decode(2, 64, 2, 2000, 128, seed=53, reading="blk")
    check_decode(bl, inp, 0.05, False, 3)


def test_decode_wide_causal_two_queries(bl):
    inp = planted_decode(1, 64, 1, 2500, 128, Lq=2, seed=54, reading="blk")
    check_decode(bl, inp, 0.1, True, 5)


def test_decode_wide_short_cache_empty_splits(bl):
    inp = planted_decode(2, 32, 1, 90, 128, seed=55, reading="lit")
    check_decode(bl, inp, 0.3, False, 16)


def test_decode_wide_calibrate_gaps(bl):
    inp = planted_decode(2, 64, 2, 3000, 128, seed=56, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    gaps, mc, cc = bl.calibrate(q, k, scale=inp.scale, lam=0.05, mode="decode", num_splits=4)
    _, _, md, cd = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=4)
    torch.cuda.synchronize()
    assert torch.equal(mc, md) and torch.equal(cc, cd)
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.05, causal=False, is_decode=True,
                           num_splits=4, BN=64)
    g = gaps.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref["gaps"])
    assert np.array_equal(np.isinf(g), np.isinf(ref["gaps"]))
    assert np.max(np.abs(g[fin] - ref["gaps"][fin])) < 1e-3


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_decode_mqa_full_size_sampled(bl, lam):
    # batch 8, 128 query heads on one KV head, 32768-key cache, 16 splits; oracle on sampled sequences
    inp = planted_decode(8, 128, 1, 32768, 128, seed=57, reading="blk")
    check_decode(bl, inp, lam, False, 16, tiles=[0, 5])


# ------------------------------------------------------------- split seeding
@pytest.mark.parametrize("lam", [0.0, 1e-3, 0.05, 0.5, 0.999])
@pytest.mark.parametrize("splits", [4, 16])
def test_decode_seeded(bl, lam, splits):
    inp = planted_decode(2, 8, 2, 64 * 37 + 13, 128, seed=21, reading="blk")
    bits, _ = check_decode(bl, inp, lam, False, splits, seed_splits=True)
    if lam == 0.0:
        assert bits.sum() == 0


@pytest.mark.parametrize("lam", [0.0, 0.1])
def test_decode_seeded_two_ntiles_causal(bl, lam):
    inp = planted_decode(1, 8, 1, 3000, 128, Lq=2, seed=3, reading="blk")
    check_decode(bl, inp, lam, True, 5, seed_splits=True)


def test_decode_seeded_short_cache_empty_splits(bl):
    inp = planted_decode(2, 4, 1, 50, 128, seed=8, reading="lit")
    check_decode(bl, inp, 0.3, False, 16, seed_splits=True)


@pytest.mark.parametrize("name", ["one_row_two_splits_seeded", "one_row_seeded_split_all_skipped"])
def test_decode_seeded_hand_cases_exact(bl, name):
    case, q, k, v = _expanded_hand_case(name, 64)
    from synth import AttnInputs

    inp = AttnInputs(q, k, v, 1.0)
    for cl in case["cases_lambda"]:
        lam = math.exp(cl["ln_lambda"]) if "ln_lambda" in cl else cl["lambda"]
        bits, _ = check_decode(bl, inp, lam, False, case["num_splits"], one_hot=True, seed_splits=True)
        assert bits.tolist() == cl["skip"]


def test_decode_seeded_calibrate_gaps(bl):
    inp = planted_decode(2, 8, 2, 5000, 128, seed=4, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    gaps, mc, cc = bl.calibrate(q, k, scale=inp.scale, lam=0.05, mode="decode", num_splits=8, seed_splits=True)
    _, _, md, cd = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=8, seed_splits=True)
    torch.cuda.synchronize()
    assert torch.equal(mc, md) and torch.equal(cc, cd)
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.05, causal=False, is_decode=True,
                           num_splits=8, BN=64, seed_splits=True)
    g = gaps.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref["gaps"])
    assert np.array_equal(np.isinf(g), np.isinf(ref["gaps"]))
    assert np.max(np.abs(g[fin] - ref["gaps"][fin])) < 1e-3


def test_decode_seeded_skips_contain_unseeded(bl):
    inp = planted_decode(4, 32, 8, 8192, 128, seed=13, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    _, _, m0, c0 = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=16)
    _, _, m1, c1 = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=16, seed_splits=True)
    torch.cuda.synchronize()
    a, b = m0.cpu().numpy().astype(np.uint32), m1.cpu().numpy().astype(np.uint32)
    assert np.all((a & ~b) == 0)
    assert int(c1.item()) > int(c0.item())


# seeded splits on wide tiles (the tcgen05 decode)
@pytest.mark.parametrize("lam", [0.0, 1e-3, 0.05, 0.5, 0.999])
@pytest.mark.parametrize("splits", [4, 16])
def test_decode_mqa_seeded(bl, lam, splits):
    inp = planted_decode(2, 32, 1, 64 * 41 + 13, 128, seed=51, reading="blk")
    bits, _ = check_decode(bl, inp, lam, False, splits, seed_splits=True)
    if lam == 0.0:
        assert bits.sum() == 0


def test_decode_wide_seeded_causal_two_queries(bl):
    inp = planted_decode(1, 64, 1, 2500, 128, Lq=2, seed=54, reading="blk")
    check_decode(bl, inp, 0.1, True, 5, seed_splits=True)


def test_decode_wide_seeded_short_cache_empty_splits(bl):
    inp = planted_decode(2, 32, 1, 90, 128, seed=55, reading="lit")
    check_decode(bl, inp, 0.3, False, 16, seed_splits=True)


def test_decode_wide_seeded_calibrate_gaps(bl):
    inp = planted_decode(2, 64, 2, 3000, 128, seed=56, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    gaps, mc, cc = bl.calibrate(q, k, scale=inp.scale, lam=0.05, mode="decode", num_splits=6, seed_splits=True)
    _, _, md, cd = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=6, seed_splits=True)
    torch.cuda.synchronize()
    assert torch.equal(mc, md) and torch.equal(cc, cd)
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.05, causal=False, is_decode=True,
                           num_splits=6, BN=64, seed_splits=True)
    g = gaps.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref["gaps"])
    assert np.array_equal(np.isinf(g), np.isinf(ref["gaps"]))
    assert np.max(np.abs(g[fin] - ref["gaps"][fin])) < 1e-3


def test_decode_wide_seeded_skips_contain_unseeded(bl):
    inp = planted_decode(2, 128, 1, 8192, 128, seed=58, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    _, _, m0, c0 = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=16)
    _, _, m1, c1 = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=16, seed_splits=True)
    torch.cuda.synchronize()
    a, b = m0.cpu().numpy().astype(np.uint32), m1.cpu().numpy().astype(np.uint32)
    assert np.all((a & ~b) == 0)
    assert int(c1.item()) > int(c0.item())


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_decode_seeded_full_size_sampled(bl, lam):
    inp = planted_decode(32, 32, 8, 32768, 128, seed=3, reading="blk")
    rng = np.random.default_rng(1)
    tiles = np.sort(rng.choice(32 * 8, 8, replace=False))
    check_decode(bl, inp, lam, False, 16, tiles=tiles, seed_splits=True)


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_decode_full_size_sampled(bl, lam):
    # batch 32, Hq 32 / Hkv 8, 32768-key cache, 16 splits: the benchmarked launch; oracle on sampled tiles
    inp = planted_decode(32, 32, 8, 32768, 128, seed=3, reading="blk")
    rng = np.random.default_rng(0)
    tiles = np.sort(rng.choice(32 * 8, 12, replace=False))
    check_decode(bl, inp, lam, False, 16, tiles=tiles)


def test_decode_adaptive_splits(bl):
    # num_splits=-1 picks blasst_decode_pick_splits(B, Hkv, Lk, SMs); same bytes as passing that count
    inp = planted_decode(2, 8, 2, 64 * 300 + 5, 128, seed=29, reading="blk")
    S = bl.decode_pick_splits(2, 2, 64 * 300 + 5)
    assert S == max(1, min(64, 300 // 32, -(-16 * torch.cuda.get_device_properties(0).multi_processor_count // 4)))
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    a = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=-1)
    b = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=S)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    check_decode(bl, inp, 0.05, False, S)


def test_decode_adaptive_splits_wide_tile(bl):
    # a 64-row tile takes the wide rule (floor(4 * SMs / (B * Hkv)) under the cap); -1 equals that count
    inp = planted_decode(4, 64, 1, 64 * 300 + 5, 128, seed=30, reading="blk")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    S = bl.decode_pick_splits(4, 1, 64 * 300 + 5, rows=64)
    assert S == max(1, min(64, 300 // 32, 4 * sms // 4))
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    a = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=-1)
    b = bl.decode(q, k, v, scale=inp.scale, lam=0.05, num_splits=S)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    check_decode(bl, inp, 0.05, False, S)
