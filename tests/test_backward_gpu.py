"""GPU parity of blasst_prefill_backward (fixed-mask backward, tcgen05) against the fp64 oracle.

The GPU forward gives o, lse and the skip mask; the GPU backward then gives
dq, dk, dv, which must match oracle.attention_backward run with the GPU's
mask.  Tolerance (per tensor X in dq, dk, dv, relative to max |X_ref|):
every output element is a sum of products in which one factor (P or dS) is
rounded to bf16 before the tensor-core product (relative error <= 2^-9 each)
and D = rowsum(dO * O) uses the bf16 forward output (relative error <= 2^-9
per term), then the sum is rounded to bf16 once more (2^-9 of |X|).  Summed
over up to a few hundred terms of mixed sign these stay well below 2^-7 of
the tensor's largest element, so the bounds are max-abs <= 2^-7 * max|X_ref|
and mean-abs <= 2^-10 * max|X_ref|.
"""
import numpy as np
import pytest

import oracle
from _parity import bf16_tensor_to_f64, unpack_mask
from synth import bf16_to_f32, planted_prefill, random_normal, upstream_grad

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

MAX_REL = 2.0 ** -7
MEAN_REL = 2.0 ** -10


@pytest.fixture(scope="module")
def bl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_tcgen05_b200 as m

    m.lib()
    return m


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def grad_errors(got, ref):
    err = np.abs(got - ref)
    top = max(np.abs(ref).max(), 1e-30)
    return float(err.max() / top), float(err.mean() / top)


def run_backward(bl, inp, lam, causal, seed=0, forced=None):
    """GPU forward (or the oracle's forward under a forced mask) + GPU backward.

    Returns the GPU gradients (f64), the mask the backward used (uint8 [tiles, nb]) and the oracle's gradients."""
    B, Hq, Lq, d = inp.q.shape
    Lk = inp.k.shape[2]
    nb = (Lk + 127) // 128
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    do_bits = upstream_grad(B, Hq, Lq, d, seed=seed)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if forced is None:
        o, lse, mask, _ = bl.prefill(q, k, v, scale=inp.scale, lam=lam, causal=causal, status_word=st)
        torch.cuda.synchronize()
        bits = unpack_mask(mask.cpu().numpy(), nb)
    else:
        bits = forced
        fr = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.0, causal=causal, forced_skip=bits)
        o = torch.from_numpy(fr["o"].astype(np.float32)).to(torch.bfloat16).cuda()
        lse = torch.from_numpy(fr["lse"].astype(np.float32)).cuda()
        words = (nb + 31) // 32
        packed = np.zeros((bits.shape[0], words), np.uint32)
        for jj in range(nb):
            packed[:, jj // 32] |= bits[:, jj].astype(np.uint32) << np.uint32(jj % 32)
        mask = torch.from_numpy(packed.view(np.int32)).cuda()
    dq, dk, dv = bl.prefill_backward(q, k, v, o, lse, to_dev(do_bits), scale=inp.scale, causal=causal,
                                     skip_mask=mask, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0, "device status word set"
    ref = oracle.attention_backward(inp.q, inp.k, inp.v, do_bits, scale=inp.scale, causal=causal, skip=bits)
    got = dict(dq=bf16_tensor_to_f64(dq), dk=bf16_tensor_to_f64(dk), dv=bf16_tensor_to_f64(dv))
    return got, bits, ref


def check_backward(bl, inp, lam, causal, seed=0, forced=None):
    got, bits, ref = run_backward(bl, inp, lam, causal, seed, forced)
    for n in ("dq", "dk", "dv"):
        assert np.all(np.isfinite(got[n])), f"{n}: non-finite"
        mx, mean = grad_errors(got[n], ref[n])
        assert mx <= MAX_REL, f"{n}: max-abs {mx:.3e} of max|ref|"
        assert mean <= MEAN_REL, f"{n}: mean-abs {mean:.3e} of max|ref|"
    return got, bits, ref


@pytest.mark.parametrize("lam", [0.0, 0.2, 0.6])
def test_backward_causal_gqa(bl, lam):
    inp = planted_prefill(1, 4, 2, 640, 128, seed=61, reading="blk")
    _, bits, _ = check_backward(bl, inp, lam, True, seed=1)
    if lam > 0:
        assert bits.any(), "expected some skipped pairs"


def test_backward_noncausal_ragged(bl):
    inp = random_normal(2, 2, 1, 200, 330, 128, seed=62)
    check_backward(bl, inp, 0.0, False, seed=2)


def test_backward_causal_shorter_queries(bl):
    # Lq < Lk: bottom-right causal alignment, ragged tails on both sides
    full = planted_prefill(1, 2, 1, 500, 128, seed=63, reading="blk")
    full.q = np.ascontiguousarray(full.q[:, :, 500 - 300:])
    check_backward(bl, full, 0.05, True, seed=3)


def test_backward_mqa_eight_heads(bl):
    inp = planted_prefill(1, 8, 1, 384, 128, seed=64, reading="blk")
    check_backward(bl, inp, 0.05, True, seed=4)


def test_backward_forced_mask_zero_gradient_block(bl):
    # a mask that skips KV block 2 in every tile that visits it: its keys get exactly zero dK, dV
    inp = planted_prefill(1, 2, 1, 640, 128, seed=65, reading="blk")
    nq = nb = 5
    rng = np.random.default_rng(7)
    forced = (rng.random((2 * nq, nb)) < 0.3).astype(np.uint8)
    forced[:, 0] = 0
    forced[:, 2] = 1
    for t in range(2 * nq):  # blocks past the causal diagonal are never visited: 0
        forced[t, (t % nq) + 1:] = 0
    got, _, _ = check_backward(bl, inp, 0.0, True, seed=5, forced=forced)
    assert np.all(got["dk"][:, :, 256:384] == 0) and np.all(got["dv"][:, :, 256:384] == 0)


def test_backward_dense_mask_equals_no_mask(bl):
    inp = planted_prefill(1, 2, 1, 384, 128, seed=66, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    o, lse, mask, _ = bl.prefill(q, k, v, scale=inp.scale, lam=0.0, causal=True)
    do = to_dev(upstream_grad(1, 2, 384, 128, seed=6))
    a = bl.prefill_backward(q, k, v, o, lse, do, scale=inp.scale, causal=True, skip_mask=mask)
    b = bl.prefill_backward(q, k, v, o, lse, do, scale=inp.scale, causal=True, skip_mask=None)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])  # dk, dv: no atomics, deterministic
    assert (a[0].float() - b[0].float()).abs().max().item() <= 2.0 ** -6 * a[0].float().abs().max().item()


def test_backward_caller_workspace(bl):
    inp = planted_prefill(1, 2, 1, 256, 128, seed=67, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    o, lse, mask, _ = bl.prefill(q, k, v, scale=inp.scale, lam=0.05, causal=True)
    do = to_dev(upstream_grad(1, 2, 256, 128, seed=7))
    ws = torch.empty(bl.backward_workspace_bytes(1, 2, 256), dtype=torch.uint8, device="cuda")
    a = bl.prefill_backward(q, k, v, o, lse, do, scale=inp.scale, causal=True, skip_mask=mask, workspace=ws)
    b = bl.prefill_backward(q, k, v, o, lse, do, scale=inp.scale, causal=True, skip_mask=mask)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_backward_full_size_sampled_rows_and_invariants(bl):
    """The benchmark's 32K GQA shape (B=1, Hq=32, Hkv=8, causal): dq of sampled rows against the
    oracle row by row, and, over every key, the two sums the gradient fixes at any size:
    sum_k dK_k = 0 (softmax does not change when every key moves by the same vector) and
    sum_k dV_k = sum of the group's dO rows (each row's P sums to 1)."""
    L = 32768
    inp = planted_prefill(1, 32, 8, L, 128, seed=3, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    o, lse, mask, cnt = bl.prefill(q, k, v, scale=inp.scale, lam=0.0128, causal=True)
    do_bits = upstream_grad(1, 32, L, 128, seed=9)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = bl.prefill_backward(q, k, v, o, lse, to_dev(do_bits), scale=inp.scale, causal=True,
                                     skip_mask=mask, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    bits = unpack_mask(mask.cpu().numpy(), L // 128)
    assert 0.3 < bits.sum() / bl.visited_pairs(1, 32, 8, L, L, True, False) < 0.95
    rows = [(0, 0, 0), (0, 5, 127), (0, 9, 12345), (0, 17, 20000), (0, 26, 30001), (0, 31, L - 1)]
    ref = oracle.backward_dq_rows(inp.q, inp.k, inp.v, do_bits, rows, scale=inp.scale, causal=True, skip=bits,
                                  terms=True)
    dqh = dq.float().cpu().numpy()
    got = np.stack([dqh[b, h, r] for b, h, r in rows])
    # A full-size row sums dS_k K_k over up to 32K keys while dq itself cancels (sum_k dS_k = 0), so
    # the bound is per element, from the terms of those sums (worst case, no cancellation of errors):
    #   dS_k is rounded to bf16:            2^-9 scale sum_k |dS_k K_kd|
    #   D = rowsum(dO O) uses the forward's bf16 O, normalised by the sum of the bf16-rounded P it used,
    #   so |dO| (2^-8 sum_k P_k |V_k| + 2^-9 |O|) bounds D's error dD, which moves dq by at most
    #                                       scale dD sum_k P_k |K_kd|
    #   the output is rounded to bf16:      2^-9 |dq|
    Kf = bf16_to_f32(inp.k).astype(np.float64)[0]
    Vf = bf16_to_f32(inp.v).astype(np.float64)[0]
    Dof = bf16_to_f32(do_bits).astype(np.float64)[0]
    for n, (b, h, r) in enumerate(rows):
        kk, vv = Kf[h // 4], Vf[h // 4]
        p_, ds_, o_ = ref["P"][n], ref["dS"][n], ref["O"][n]
        dD = (np.abs(Dof[h, r]) * (2.0 ** -8 * (p_ @ np.abs(vv)) + 2.0 ** -9 * np.abs(o_))).sum()
        bound = (2.0 ** -9 * (np.abs(ref["dq"][n]) + inp.scale * (np.abs(ds_) @ np.abs(kk))) +
                 inp.scale * dD * (p_ @ np.abs(kk)))
        err = np.abs(got[n] - ref["dq"][n])
        assert np.all(err <= bound + 1e-7), f"row {(b, h, r)}: worst {np.max(err / (bound + 1e-7)):.2f} of bound"
    dkh = dk.double().cpu().numpy()[0]
    dvh = dv.double().cpu().numpy()[0]
    dov = torch.from_numpy(do_bits.view(np.int16)).view(torch.bfloat16).double().numpy()[0]
    for hk in range(8):
        tot = np.abs(dkh[hk]).sum(axis=0)
        assert np.all(np.abs(dkh[hk].sum(axis=0)) <= 2.0 ** -6 * tot)
        want = dov[hk * 4:(hk + 1) * 4].sum(axis=(0, 1))
        tot_v = np.abs(dvh[hk]).sum(axis=0)
        assert np.all(np.abs(dvh[hk].sum(axis=0) - want) <= 2.0 ** -6 * tot_v)


def test_backward_long_sequence_partial_last_chunk(bl):
    """261 KV blocks (33408 keys): the launch orders CTAs in chunks of 64 KV blocks, the last chunk
    holding 5. Sampled dq rows against the oracle (rows seeing the last blocks included) and the key
    sums sum_k dK_k = 0 and sum_k dV_k = sum of the group's dO rows, which miss a block whose CTA was
    left out or run twice; the last block's dK and dV rows are nonzero."""
    L = 261 * 128
    inp = planted_prefill(1, 8, 2, L, 128, seed=71, reading="blk")
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    o, lse, mask, cnt = bl.prefill(q, k, v, scale=inp.scale, lam=0.0128, causal=True)
    do_bits = upstream_grad(1, 8, L, 128, seed=10)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = bl.prefill_backward(q, k, v, o, lse, to_dev(do_bits), scale=inp.scale, causal=True,
                                     skip_mask=mask, status_word=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    bits = unpack_mask(mask.cpu().numpy(), L // 128)
    rows = [(0, 0, 5), (0, 3, 20000), (0, 4, L - 300), (0, 7, L - 1)]
    ref = oracle.backward_dq_rows(inp.q, inp.k, inp.v, do_bits, rows, scale=inp.scale, causal=True, skip=bits,
                                  terms=True)
    dqh = dq.float().cpu().numpy()
    Kf = bf16_to_f32(inp.k).astype(np.float64)[0]
    Vf = bf16_to_f32(inp.v).astype(np.float64)[0]
    Dof = bf16_to_f32(do_bits).astype(np.float64)[0]
    for n, (b, h, r) in enumerate(rows):
        # the per-element bound of the 32K test: bf16 dS, the forward's bf16 O in D, the bf16 output
        kk, vv = Kf[h // 4], Vf[h // 4]
        p_, ds_, o_ = ref["P"][n], ref["dS"][n], ref["O"][n]
        dD = (np.abs(Dof[h, r]) * (2.0 ** -8 * (p_ @ np.abs(vv)) + 2.0 ** -9 * np.abs(o_))).sum()
        bound = (2.0 ** -9 * (np.abs(ref["dq"][n]) + inp.scale * (np.abs(ds_) @ np.abs(kk))) +
                 inp.scale * dD * (p_ @ np.abs(kk)))
        err = np.abs(dqh[b, h, r] - ref["dq"][n])
        assert np.all(err <= bound + 1e-7), f"row {(b, h, r)}: worst {np.max(err / (bound + 1e-7)):.2f} of bound"
    dkh = dk.double().cpu().numpy()[0]
    dvh = dv.double().cpu().numpy()[0]
    dov = torch.from_numpy(do_bits.view(np.int16)).view(torch.bfloat16).double().numpy()[0]
    for hk in range(2):
        tot = np.abs(dkh[hk]).sum(axis=0)
        assert np.all(np.abs(dkh[hk].sum(axis=0)) <= 2.0 ** -6 * tot)
        want = dov[hk * 4:(hk + 1) * 4].sum(axis=(0, 1))
        tot_v = np.abs(dvh[hk]).sum(axis=0)
        assert np.all(np.abs(dvh[hk].sum(axis=0) - want) <= 2.0 ** -6 * tot_v)
        assert np.abs(dvh[hk, L - 128:]).sum() > 0 and np.abs(dkh[hk, L - 128:]).sum() > 0


def test_backward_noncausal_more_queries_than_keys(bl):
    inp = random_normal(1, 4, 2, 500, 200, 128, seed=68)
    check_backward(bl, inp, 0.0, False, seed=8)


def test_backward_group_of_sixteen(bl):
    inp = planted_prefill(1, 16, 1, 384, 128, seed=69, reading="blk")
    check_backward(bl, inp, 0.1, True, seed=9)


@pytest.mark.parametrize("lam", [0.5, 0.999])
def test_backward_heavy_skipping_batch_three_ragged(bl, lam):
    inp = planted_prefill(3, 2, 1, 250 + 128 * 3, 128, seed=70, reading="blk")
    _, bits, _ = check_backward(bl, inp, lam, True, seed=10)
    assert bits.any()
