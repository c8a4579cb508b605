"""GPU parity of blasst_decode_fp8 (e4m3 K/V cache) against the fp64 oracle.

The cache holds K = k_scale * k8 and V = v_scale * v8.  Every e4m3 value is
exact in bf16, so the oracle runs on the decoded bytes (as bf16) with the
softmax scale multiplied by k_scale, and its O is multiplied by v_scale: the
same function, evaluated in fp64.  Bars as for the bf16 decode (masks outside
the +-1e-3 band, O 1e-2 / 1e-3, lse 1e-3).
"""
import numpy as np
import pytest

import oracle
from _parity import assert_outputs_close, bf16_tensor_to_f64, compare_masks, unpack_mask
from synth import bf16_bits, bf16_to_f32, e4m3_bits, e4m3_to_f32, planted_decode, random_normal

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


def quantize(x_bits):
    """bf16 bits -> (e4m3 bytes, per-tensor scale, the decoded values as bf16 bits)."""
    x = bf16_to_f32(x_bits)
    scale = float(np.abs(x).max()) / 448.0
    q8 = e4m3_bits(x / scale)
    return q8, scale, bf16_bits(e4m3_to_f32(q8))


def check_fp8(bl, inp, lam, splits, causal=False, seed_splits=False):
    k8, ks, kdeq = quantize(inp.k)
    v8, vs, vdeq = quantize(inp.v)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, mask, cnt = bl.decode_fp8(to_dev(inp.q), torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda(),
                                      scale=inp.scale, k_scale=ks, v_scale=vs, lam=lam, causal=causal,
                                      num_splits=splits, status_word=st, seed_splits=seed_splits)
    torch.cuda.synchronize()
    assert st.item() == 0
    nb = (inp.k.shape[2] + 63) // 64
    bits = unpack_mask(mask.cpu().numpy(), nb)
    assert int(cnt.item()) == int(bits.sum())
    kw = dict(scale=inp.scale * ks, lam=lam, causal=causal, is_decode=True, num_splits=splits, BN=64,
              seed_splits=seed_splits)
    ref = oracle.attention(inp.q, kdeq, vdeq, **kw)
    nd, _ = compare_masks(bits, ref, lam)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, kdeq, vdeq, forced_skip=bits, **kw)
    assert_outputs_close(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), fr["o"] * vs, fr["lse"])
    return bits


@pytest.mark.parametrize("lam", [0.0, 0.05, 0.5])
@pytest.mark.parametrize("splits", [1, 4, 16])
def test_fp8_gqa_ragged(bl, lam, splits):
    inp = planted_decode(2, 8, 2, 64 * 37 + 13, 128, seed=71, reading="blk")
    bits = check_fp8(bl, inp, lam, splits)
    if lam == 0.0:
        assert bits.sum() == 0


def test_fp8_sixteen_row_tile(bl):
    # G * Lq = 16: the 16-row variant of the kernel
    inp = planted_decode(2, 16, 1, 3000, 128, seed=72, reading="blk")
    check_fp8(bl, inp, 0.05, 4)


def test_fp8_causal_multi_query(bl):
    inp = planted_decode(2, 4, 1, 2000, 128, Lq=3, seed=73, reading="blk")
    check_fp8(bl, inp, 0.05, 3, causal=True)


def test_fp8_seeded(bl):
    inp = planted_decode(2, 8, 2, 4000, 128, seed=74, reading="blk")
    check_fp8(bl, inp, 0.05, 8, seed_splits=True)


def test_fp8_random_inputs(bl):
    inp = random_normal(2, 4, 2, 1, 1500, 128, seed=75)
    check_fp8(bl, inp, 0.0, 4)


def test_fp8_rejects_wide_tiles_and_bad_scales(bl):
    inp = planted_decode(1, 32, 1, 256, 128, seed=76, reading="blk")
    k8 = torch.zeros((1, 1, 256, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(bl.BlasstError) as e:
        bl.decode_fp8(to_dev(inp.q), k8, k8, scale=inp.scale, k_scale=1.0, v_scale=1.0)
    assert e.value.status == 2
    inp = planted_decode(1, 8, 1, 256, 128, seed=76, reading="blk")
    with pytest.raises(bl.BlasstError) as e:
        bl.decode_fp8(to_dev(inp.q), k8, k8, scale=inp.scale, k_scale=0.0, v_scale=1.0)
    assert e.value.status == 1


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_fp8_full_size_sampled(bl, lam):
    # the benchmarked FP8 launch: batch 32, Hq 32 / Hkv 8, 32768-key cache, 16 splits, per-tensor
    # scales; the oracle runs on sampled (sequence, KV head) tiles of the decoded cache
    inp = planted_decode(32, 32, 8, 32768, 128, seed=3, reading="blk")
    k, v = to_dev(inp.k), to_dev(inp.v)

    def quant(x):  # on the device: the same nearest-even, saturating cast as synth.e4m3_bits
        sc = float(x.float().abs().max().item()) / 448.0
        return (x.float() / sc).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8), sc

    k8, ks = quant(k)
    v8, vs = quant(v)
    del k, v
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, mask, cnt = bl.decode_fp8(to_dev(inp.q), k8, v8, scale=inp.scale, k_scale=ks, v_scale=vs, lam=lam,
                                      num_splits=16, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rng = np.random.default_rng(2)
    tiles = np.sort(rng.choice(32 * 8, 8, replace=False))
    kdeq = np.zeros_like(inp.k)
    vdeq = np.zeros_like(inp.v)
    for t in tiles:
        b, h = divmod(int(t), 8)
        kdeq[b, h] = bf16_bits(e4m3_to_f32(k8[b, h].cpu().numpy()))
        vdeq[b, h] = bf16_bits(e4m3_to_f32(v8[b, h].cpu().numpy()))
    bits = unpack_mask(mask.cpu().numpy(), 512)
    kw = dict(scale=inp.scale * ks, lam=lam, causal=False, is_decode=True, num_splits=16, BN=64, tiles=tiles)
    ref = oracle.attention(inp.q, kdeq, vdeq, **kw)
    nd, _ = compare_masks(bits, ref, lam, tiles)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, kdeq, vdeq, forced_skip=bits, **kw)
    sel = np.zeros((32, 32, 1), bool)
    for t in tiles:
        b, h = divmod(int(t), 8)
        sel[b, h * 4:(h + 1) * 4, :] = True
    assert_outputs_close(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), fr["o"] * vs, fr["lse"], sel)


def test_fp8_cache_shorter_than_a_block_more_splits_than_blocks(bl):
    inp = planted_decode(3, 8, 2, 40, 128, seed=77, reading="blk")
    check_fp8(bl, inp, 0.05, 4)
    inp = planted_decode(2, 8, 2, 64 * 3 + 1, 128, seed=78, reading="blk")
    check_fp8(bl, inp, 0.3, 16)
