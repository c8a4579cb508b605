"""The e4m3 codec the FP8 decode tests use to build inputs and the oracle's view of them.

The decoder is written from the OCP E4M3FN definition; it is pinned to that
definition's landmark values and to torch's float8_e4m3fn conversion (all 256
codes), and the encoder to a brute-force nearest-value search.
"""
import numpy as np
import pytest

from synth import e4m3_bits, e4m3_to_f32

torch = pytest.importorskip("torch")


def test_landmark_values():
    d = e4m3_to_f32(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0xB8, 0x7E, 0xFE, 0x40, 0x3C], np.uint8))
    assert d[0] == 0.0
    assert d[1] == 2.0 ** -9            # smallest subnormal
    assert d[2] == 7 * 2.0 ** -9        # largest subnormal
    assert d[3] == 2.0 ** -6            # smallest normal
    assert d[4] == 1.0 and d[5] == -1.0
    assert d[6] == 448.0 and d[7] == -448.0
    assert d[8] == 2.0 and d[9] == 1.5
    assert np.isnan(e4m3_to_f32(np.array([0x7F, 0xFF], np.uint8))).all()


def test_decoder_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3_to_f32(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_encoder_is_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4000) * 30, rng.standard_normal(1000) * 0.01, [500.0, -1e6, 0.0]])
    got = e4m3_to_f32(e4m3_bits(x)).astype(np.float64)
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3_to_f32(codes).astype(np.float64)
    ok = ~np.isnan(vals)
    vals, codes = vals[ok], codes[ok]
    xc = np.clip(x, -448, 448)
    dist = np.abs(xc[:, None] - vals[None, :])
    best = dist.min(axis=1)
    assert np.all(np.abs(got - xc) == best)          # a nearest representable value
    ties = (dist == best[:, None]).sum(axis=1) > 1
    even = (codes[np.argmin(np.where(dist == best[:, None], codes[None, :] & 1, 9), axis=1)] & 1) == 0
    assert np.all(~ties | even)


def test_e4m3_values_are_exact_in_bf16():
    from synth import bf16_bits, bf16_to_f32

    v = e4m3_to_f32(np.arange(256, dtype=np.uint8))
    v = v[~np.isnan(v)]
    assert np.array_equal(bf16_to_f32(bf16_bits(v)), v)
