"""GPU parity of MLA decode (576-column latent cache, V = its first 512 columns,
all query heads in one tile) against the fp64 oracle."""
import numpy as np
import pytest

import oracle
from _parity import assert_outputs_close, bf16_tensor_to_f64, compare_masks, unpack_mask
from synth import planted_mla

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


def check_mla(bl, inp, lam, splits, causal=False, tiles=None, seed_splits=False):
    q, k = to_dev(inp.q), to_dev(inp.k)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, mask, cnt = bl.decode(q, k, k, scale=inp.scale, lam=lam, causal=causal, num_splits=splits, dv=512,
                                  status_word=st, seed_splits=seed_splits)
    torch.cuda.synchronize()
    assert st.item() == 0
    B, Hq, Lq, d = inp.q.shape
    Lk = inp.k.shape[2]
    nb = (Lk + 63) // 64
    bits = unpack_mask(mask.cpu().numpy(), nb)
    assert int(cnt.item()) == int(bits.sum())
    kw = dict(scale=inp.scale, lam=lam, causal=causal, is_decode=True, num_splits=splits, BN=64, dv=512,
              v_row_stride=576, tiles=tiles, seed_splits=seed_splits)
    ref = oracle.attention(inp.q, inp.k, inp.k, **kw)
    nd, _ = compare_masks(bits, ref, lam, tiles)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, inp.k, inp.k, forced_skip=bits, **kw)
    rows = None
    if tiles is not None:
        rows = np.zeros((B, Hq, Lq), bool)
        rows[np.asarray(tiles)] = True
    assert_outputs_close(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), fr["o"], fr["lse"], rows)
    return bits, ref


@pytest.mark.parametrize("lam", [0.0, 0.02, 0.5])
@pytest.mark.parametrize("splits", [1, 2, 3])
def test_mla_small(bl, lam, splits):
    inp = planted_mla(2, 16, 1000, seed=41, reading="blk")
    check_mla(bl, inp, lam, splits)


@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_mla_full_tile(bl, lam):
    # 128 query heads: every TMEM lane is a row
    inp = planted_mla(2, 128, 4096, seed=42, reading="blk")
    bits, _ = check_mla(bl, inp, lam, 2)
    if lam > 0:
        assert bits.sum() > 0


def test_mla_causal_two_queries(bl):
    inp = planted_mla(1, 64, 2000, Lq=2, seed=43, reading="lit")
    check_mla(bl, inp, 0.1, 2, causal=True)


def test_mla_calibrate_matches_decode(bl):
    inp = planted_mla(2, 32, 3000, seed=44, reading="blk")
    q, k = to_dev(inp.q), to_dev(inp.k)
    gaps, mc, cc = bl.calibrate(q, k, scale=inp.scale, lam=0.05, causal=False, mode="decode", num_splits=2, dv=512)
    _, _, md, cd = bl.decode(q, k, k, scale=inp.scale, lam=0.05, num_splits=2, dv=512)
    torch.cuda.synchronize()
    assert torch.equal(mc, md) and torch.equal(cc, cd)
    ref = oracle.attention(inp.q, inp.k, inp.k, scale=inp.scale, lam=0.05, causal=False, is_decode=True,
                           num_splits=2, BN=64, dv=512, v_row_stride=576)
    g = gaps.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref["gaps"])
    assert np.array_equal(np.isinf(g), np.isinf(ref["gaps"]))
    assert np.max(np.abs(g[fin] - ref["gaps"][fin])) < 1e-3


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_mla_full_size_sampled(bl, lam):
    # batch 64, 128 heads, 32768-key latent cache, 2 splits: the benchmarked launch
    inp = planted_mla(64, 128, 32768, seed=5, reading="blk")
    tiles = [0, 23, 63]
    check_mla(bl, inp, lam, 2, tiles=tiles)


@pytest.mark.parametrize("lam", [0.0, 0.05, 0.5])
@pytest.mark.parametrize("splits", [3, 8])
def test_mla_seeded_splits(bl, lam, splits):
    # every split after the first starts its running max at block 0's row maxima and has no
    # forced first block (the oracle's seeded mode)
    inp = planted_mla(2, 128, 3000, seed=46, reading="blk")
    bits, ref = check_mla(bl, inp, lam, splits, seed_splits=True)
    if lam == 0.0:
        assert bits.sum() == 0


def test_mla_seeded_causal_two_queries(bl):
    inp = planted_mla(1, 64, 2000, Lq=2, seed=47, reading="blk")
    check_mla(bl, inp, 0.1, 4, causal=True, seed_splits=True)


def test_mla_seeded_calibrate_matches_decode(bl):
    inp = planted_mla(2, 128, 3000, seed=48, reading="blk")
    q, k = to_dev(inp.q), to_dev(inp.k)
    gaps, mc, cc = bl.calibrate(q, k, scale=inp.scale, lam=0.05, causal=False, mode="decode", num_splits=8, dv=512,
                                seed_splits=True)
    _, _, md, cd = bl.decode(q, k, k, scale=inp.scale, lam=0.05, num_splits=8, dv=512, seed_splits=True)
    torch.cuda.synchronize()
    assert torch.equal(mc, md) and torch.equal(cc, cd)
    ref = oracle.attention(inp.q, inp.k, inp.k, scale=inp.scale, lam=0.05, causal=False, is_decode=True,
                           num_splits=8, BN=64, dv=512, v_row_stride=576, seed_splits=True)
    g = gaps.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref["gaps"])
    assert np.array_equal(np.isinf(g), np.isinf(ref["gaps"]))
    assert np.max(np.abs(g[fin] - ref["gaps"][fin])) < 1e-3


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 0.01])
def test_mla_seeded_full_size_sampled(bl, lam):
    # batch 64, 128 heads, 32768-key latent cache, 8 seeded splits
    inp = planted_mla(64, 128, 32768, seed=5, reading="blk")
    check_mla(bl, inp, lam, 8, tiles=[0, 31, 63], seed_splits=True)
