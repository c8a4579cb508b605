"""Parity at the benchmarked points.

Every (workload, sparsity target) that bench.py times is rebuilt here exactly as
the bench builds it -- same configuration, seed and input generator, same
device tensors -- and its lambda is taken exactly as the bench takes it: one
decision-only calibration pass, then the gap quantile for the target (the
highest reachable sparsity when the target is out of reach); the paged, ragged
cache by bisection on the device's skip count.  The launch at that lambda is
then compared with the fp64 oracle on sampled tiles (or whole sequences):

  * skip masks bit-equal outside the +-1e-3 band around ln(lambda);
  * O against the oracle run on the device's mask: max-abs <= 1e-2, mean-abs
    <= 1e-3; lse within 1e-3;
  * the device's skip count reproduces the sparsity the calibration promised.

The sampled prefill tiles include the first tile, the last tile, and the
diagonal tiles of the longest rows of several heads, whose rows visit every
block.
"""
import numpy as np
import pytest

import bench
import oracle
from _parity import assert_outputs_close, bf16_tensor_to_f64, compare_masks, unpack_mask
from synth import bf16_bits, bf16_to_f32, e4m3_bits, e4m3_to_f32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
torch = pytest.importorskip("torch")

TARGETS = (0.0, 0.5, 0.75)
_WL = {}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_tcgen05_b200 as m

    m.lib()
    yield torch.device("cuda", 0)
    _WL.clear()
    torch.cuda.empty_cache()


def workload(name, dev):
    """The bench's workload object and its lambdas, built once per module."""
    if name not in _WL:
        if name == "prefill":
            wl = bench.Prefill(bench.PREFILL, dev)
        elif name == "prefill_64k":
            wl = bench.Prefill(bench.PREFILL_64K, dev)
        elif name == "decode":
            wl = bench.Decode(bench.DECODE, dev)
        elif name == "decode_seeded":
            src = workload("decode", dev)[0]
            wl = bench.DecodeSeeded.__new__(bench.DecodeSeeded)
            wl.__dict__.update(src.__dict__)
        elif name == "decode_mqa":
            wl = bench.DecodeMqa(bench.MQA, dev)
        elif name == "decode_mqa_seeded":
            src = workload("decode_mqa", dev)[0]
            wl = bench.DecodeMqaSeeded.__new__(bench.DecodeMqaSeeded)
            wl.__dict__.update(src.__dict__)
        elif name == "mla":
            wl = bench.Mla(bench.MLA, dev)
        elif name == "decode_paged":
            src = workload("decode", dev)[0]
            wl = bench.DecodePaged(src, dev, min_len=min(8192, src.cfg["Lk"] // 4))
        else:
            raise KeyError(name)
        wl.count = torch.zeros(1, dtype=torch.int64, device=dev)
        lams = wl.lambdas() if hasattr(wl, "lambdas") else bench.lambdas_for_targets(wl, wl.calibrate())
        _WL[name] = (wl, lams)
    return _WL[name]


def _prefill_tiles(Hq, nq, rng, extra=3):
    fixed = [0, nq - 1, 7 * nq + nq - 1, 16 * nq + nq // 2, 24 * nq + nq - 2, (Hq - 1) * nq + nq - 1]
    pool = np.setdiff1d(np.arange(Hq * nq), fixed)
    return np.sort(np.concatenate([fixed, rng.choice(pool, extra, replace=False)]))


@pytest.mark.parametrize("name", ["prefill", "prefill_64k"])
@pytest.mark.parametrize("target", TARGETS)
def test_prefill_at_bench_lambda(dev, name, target):
    import block_sparse_flashattention_tcgen05_b200 as bl

    wl, lams = workload(name, dev)
    lam, achieved = lams[target]
    inp = wl.inp
    B, Hq, Lq, _ = inp.q.shape
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse, mask, cnt = bl.prefill(wl.q, wl.k, wl.v, scale=inp.scale, lam=lam, causal=True, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert abs(int(cnt.item()) / wl.visited - achieved) < 1e-9, "sparsity differs from the calibration's"
    nq = (Lq + 127) // 128
    nb = (inp.k.shape[2] + 127) // 128
    bits = unpack_mask(mask.cpu().numpy(), nb)
    assert int(cnt.item()) == int(bits.sum())
    tiles = _prefill_tiles(Hq, nq, np.random.default_rng(int(target * 100) + nq))
    kw = dict(scale=inp.scale, lam=lam, causal=True, tiles=tiles)
    ref = oracle.attention(inp.q, inp.k, inp.v, **kw)
    nd, _ = compare_masks(bits, ref, lam, tiles)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, inp.k, inp.v, forced_skip=bits, **kw)
    rows = np.zeros((B, Hq, Lq), bool)
    for t in tiles:
        bh, qt = divmod(int(t), nq)
        rows.reshape(B * Hq, Lq)[bh, qt * 128:(qt + 1) * 128] = True
    assert_outputs_close(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), fr["o"], fr["lse"], rows)


def _decode_check(inp, lam, splits, o, lse, mask, tiles, seed_splits=False, k=None, v=None, scale=None,
                  o_scale=1.0):
    B, Hq, Lq, _ = inp.q.shape
    Hkv = inp.k.shape[1]
    nb = (inp.k.shape[2] + 63) // 64
    bits = unpack_mask(mask.cpu().numpy(), nb)
    k = inp.k if k is None else k
    v = inp.v if v is None else v
    kw = dict(scale=inp.scale if scale is None else scale, lam=lam, causal=False, is_decode=True,
              num_splits=splits, BN=64, tiles=tiles, seed_splits=seed_splits)
    ref = oracle.attention(inp.q, k, v, **kw)
    nd, _ = compare_masks(bits, ref, lam, tiles)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, k, v, forced_skip=bits, **kw)
    G = Hq // Hkv
    rows = np.zeros((B, Hq, Lq), bool)
    for t in tiles:
        b, h = divmod(int(t), Hkv)
        rows[b, h * G:(h + 1) * G] = True
    assert_outputs_close(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), fr["o"] * o_scale,
                         fr["lse"], rows)
    return bits


@pytest.mark.parametrize("name", ["decode", "decode_seeded", "decode_mqa", "decode_mqa_seeded"])
@pytest.mark.parametrize("target", TARGETS)
def test_decode_at_bench_lambda(dev, name, target):
    import block_sparse_flashattention_tcgen05_b200 as bl

    wl, lams = workload(name, dev)
    lam, achieved = lams[target]
    inp = wl.inp
    B, Hq, _, _ = inp.q.shape
    Hkv = inp.k.shape[1]
    splits = wl.cfg["splits"]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse, mask, cnt = bl.decode(wl.q, wl.k, wl.v, scale=inp.scale, lam=lam, num_splits=splits,
                                  seed_splits=wl.seed_splits, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert abs(int(cnt.item()) / wl.visited - achieved) < 1e-9, "sparsity differs from the calibration's"
    rng = np.random.default_rng(int(target * 100) + 7)
    n = B * Hkv
    tiles = np.unique(np.concatenate([[0, n - 1], rng.choice(n, min(n, 48 if Hkv > 1 else 6), replace=False)]))
    _decode_check(inp, lam, splits, o, lse, mask, tiles, seed_splits=wl.seed_splits)


def _quantize(x_bits):
    """bf16 bits -> (e4m3 bytes, per-tensor scale, decoded values as bf16 bits): the
    bench's rule (max |x| / 448, nearest even, saturating), computed on the host."""
    x = bf16_to_f32(x_bits)
    scale = float(np.abs(x).max()) / 448.0
    q8 = e4m3_bits(x / np.float32(scale))
    return q8, scale, bf16_bits(e4m3_to_f32(q8))


@pytest.mark.parametrize("target", TARGETS)
def test_decode_fp8_at_bench_lambda(dev, target):
    # the bench times the FP8 cache at the bf16 decode's lambdas
    import block_sparse_flashattention_tcgen05_b200 as bl

    wl, lams = workload("decode", dev)
    lam, _ = lams[target]
    inp = wl.inp
    if "fp8" not in _WL:
        _WL["fp8"] = (_quantize(inp.k), _quantize(inp.v))
    (k8, ks, kdeq), (v8, vs, vdeq) = _WL["fp8"]
    B, Hq, _, _ = inp.q.shape
    Hkv = inp.k.shape[1]
    splits = wl.cfg["splits"]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse, mask, cnt = bl.decode_fp8(wl.q, torch.from_numpy(k8).to(dev), torch.from_numpy(v8).to(dev),
                                      scale=inp.scale, k_scale=ks, v_scale=vs, lam=lam, num_splits=splits,
                                      status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rng = np.random.default_rng(int(target * 100) + 11)
    n = B * Hkv
    tiles = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 48, replace=False)]))
    bits = _decode_check(inp, lam, splits, o, lse, mask, tiles, k=kdeq, v=vdeq, scale=inp.scale * ks,
                         o_scale=vs)
    assert int(cnt.item()) == int(bits.sum())


@pytest.mark.parametrize("target", TARGETS)
def test_mla_at_bench_lambda(dev, target):
    import block_sparse_flashattention_tcgen05_b200 as bl

    wl, lams = workload("mla", dev)
    lam, achieved = lams[target]
    inp = wl.inp
    B, Hq, Lq, _ = inp.q.shape
    splits = wl.cfg["splits"]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    seeded = wl.cfg.get("seed_splits", False)
    o, lse, mask, cnt = bl.decode(wl.q, wl.k, wl.k, scale=inp.scale, lam=lam, num_splits=splits, dv=512,
                                  status_word=st, seed_splits=seeded)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert abs(int(cnt.item()) / wl.visited - achieved) < 1e-9, "sparsity differs from the calibration's"
    nb = (inp.k.shape[2] + 63) // 64
    bits = unpack_mask(mask.cpu().numpy(), nb)
    tiles = [0, B // 2 + int(target * 10), B - 1]
    kw = dict(scale=inp.scale, lam=lam, causal=False, is_decode=True, num_splits=splits, BN=64, dv=512,
              v_row_stride=576, tiles=tiles, seed_splits=seeded)
    ref = oracle.attention(inp.q, inp.k, inp.k, **kw)
    nd, _ = compare_masks(bits, ref, lam, tiles)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, inp.k, inp.k, forced_skip=bits, **kw)
    rows = np.zeros((B, Hq, Lq), bool)
    rows[np.asarray(tiles)] = True
    assert_outputs_close(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), fr["o"], fr["lse"], rows)


@pytest.mark.parametrize("target", TARGETS)
def test_decode_paged_at_bench_lambda(dev, target):
    import block_sparse_flashattention_tcgen05_b200 as bl

    wl, lams = workload("decode_paged", dev)
    lam, achieved = lams[target]
    inp = wl.inp
    B, Hq, _, _ = inp.q.shape
    Hkv = inp.k.shape[1]
    splits = wl.cfg["splits"]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse, mask, cnt = bl.decode_paged(wl.q, wl.kp, wl.vp, wl.table, wl.lens_dev, scale=inp.scale, lam=lam,
                                        num_splits=splits, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert abs(int(cnt.item()) / wl.visited - achieved) < 1e-9, "sparsity differs from the bisection's"
    max_pages = wl.table.shape[1]
    bits = unpack_mask(mask.cpu().numpy(), max_pages).reshape(B, Hkv, max_pages)
    og = bf16_tensor_to_f64(o)
    lg = lse.cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(int(target * 100) + 13)
    longest, shortest = int(np.argmax(wl.lens)), int(np.argmin(wl.lens))
    for b in np.unique(np.concatenate([[longest, shortest], rng.choice(B, 4, replace=False)])):
        n = int(wl.lens[b])
        nbk = (n + 63) // 64
        assert not bits[b, :, nbk:].any(), "mask bit past the sequence's last block"
        kw = dict(scale=inp.scale, lam=lam, causal=False, is_decode=True, num_splits=splits, BN=64)
        qb, kb, vb = inp.q[b:b + 1], inp.k[b:b + 1, :, :n], inp.v[b:b + 1, :, :n]
        ref = oracle.attention(qb, kb, vb, **kw)
        nd, _ = compare_masks(bits[b, :, :nbk], ref, lam)
        assert nd == 0, f"sequence {b}: {nd} mask bits differ outside the band"
        fr = oracle.attention(qb, kb, vb, forced_skip=bits[b, :, :nbk], **kw)
        assert_outputs_close(og[b:b + 1], lg[b:b + 1], fr["o"], fr["lse"])


@pytest.mark.parametrize("target", TARGETS)
def test_backward_at_bench_lambda(dev, target):
    """The fixed-mask backward the bench times: the 32K GQA prefill inputs, the forward's mask at the
    bench's lambda, the bench's upstream gradient.  Sampled dq rows against the oracle's row function
    within the per-element bound of tests/test_backward_gpu.py (bf16 dS, the bf16 forward O in D, the
    output rounding), and over every key sum_k dK_k = 0 and sum_k dV_k = the group's sum of dO rows."""
    import block_sparse_flashattention_tcgen05_b200 as bl
    from synth import upstream_grad

    wl, lams = workload("prefill", dev)
    lam, achieved = lams[target]
    inp = wl.inp
    B, Hq, L, _ = inp.q.shape
    Hkv = inp.k.shape[1]
    G = Hq // Hkv
    o, lse, mask, cnt = bl.prefill(wl.q, wl.k, wl.v, scale=inp.scale, lam=lam, causal=True)
    do_bits = upstream_grad(B, Hq, L, 128, seed=wl.cfg["seed"])  # the bench's dO (bench.Backward)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    dq, dk, dv = bl.prefill_backward(wl.q, wl.k, wl.v, o, lse, bench.to_dev(do_bits, dev), scale=inp.scale,
                                     causal=True, skip_mask=mask, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert abs(int(cnt.item()) / wl.visited - achieved) < 1e-9
    bits = unpack_mask(mask.cpu().numpy(), (L + 127) // 128)
    rows = [(0, 0, 0), (0, 3, 4097), (0, 9, 12345), (0, 17, 20000), (0, 26, 30001), (0, Hq - 1, L - 1)]
    ref = oracle.backward_dq_rows(inp.q, inp.k, inp.v, do_bits, rows, scale=inp.scale, causal=True, skip=bits,
                                  terms=True)
    dqh = dq.float().cpu().numpy()
    Kf = bf16_to_f32(inp.k).astype(np.float64)[0]
    Vf = bf16_to_f32(inp.v).astype(np.float64)[0]
    Dof = bf16_to_f32(do_bits).astype(np.float64)[0]
    for n, (b, h, r) in enumerate(rows):
        kk, vv = Kf[h // G], Vf[h // G]
        p_, ds_, o_ = ref["P"][n], ref["dS"][n], ref["O"][n]
        dD = (np.abs(Dof[h, r]) * (2.0 ** -8 * (p_ @ np.abs(vv)) + 2.0 ** -9 * np.abs(o_))).sum()
        bound = (2.0 ** -9 * (np.abs(ref["dq"][n]) + inp.scale * (np.abs(ds_) @ np.abs(kk))) +
                 inp.scale * dD * (p_ @ np.abs(kk)))
        err = np.abs(dqh[b, h, r] - ref["dq"][n])
        assert np.all(err <= bound + 1e-7), f"row {(b, h, r)}: worst {np.max(err / (bound + 1e-7)):.2f} of bound"
    dkh = dk.double().cpu().numpy()[0]
    dvh = dv.double().cpu().numpy()[0]
    dov = torch.from_numpy(do_bits.view(np.int16)).view(torch.bfloat16).double().numpy()[0]
    for hk in range(Hkv):
        tot = np.abs(dkh[hk]).sum(axis=0)
        assert np.all(np.abs(dkh[hk].sum(axis=0)) <= 2.0 ** -6 * tot)
        want = dov[hk * G:(hk + 1) * G].sum(axis=(0, 1))
        tot_v = np.abs(dvh[hk]).sum(axis=0)
        assert np.all(np.abs(dvh[hk].sum(axis=0) - want) <= 2.0 ** -6 * tot_v)
