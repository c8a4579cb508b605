"""blasst_decode_noalloc: the decode entry point that allocates nothing.

It serves callers that cannot allocate device memory while they run (an
engine that has reserved the device's memory for its own pool, a
latency-critical loop where an allocation could stall the device).  Its split
partials live in a fixed device array inside the library.  This file is named
to be collected last, so that a run stopping at the first failure has already
run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

import oracle
from _parity import (LSE_ABS, O_MAX_ABS, O_MEAN_ABS, assert_outputs_close, bf16_tensor_to_f64, compare_masks,
                     unpack_mask)
from synth import planted_decode, planted_mla

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


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    err = np.abs(a - b)
    return err.max(), err.mean()


def test_noalloc_matches_decode_on_two_calls_in_a_row(bl):
    # two different problems back to back through the fixed scratch: the second
    # call must not see anything left over from the first
    cases = [
        (planted_decode(4, 8, 2, 5000, 128, seed=31, reading="blk"), 0.05, 16),
        (planted_decode(2, 8, 1, 3000, 128, Lq=2, seed=32, reading="lit"), 0.2, 5),
    ]
    for inp, lam, splits in cases:
        q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
        causal = inp.q.shape[2] > 1
        o1, l1, m1, c1 = bl.decode_noalloc(q, k, v, scale=inp.scale, lam=lam, causal=causal, num_splits=splits)
        o2, l2, m2, c2 = bl.decode(q, k, v, scale=inp.scale, lam=lam, causal=causal, num_splits=splits)
        torch.cuda.synchronize()
        assert torch.equal(m1, m2) and torch.equal(c1, c2)
        emax, emean = _close(o1, o2)
        assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS
        assert float((l1 - l2).abs().max()) <= LSE_ABS


def _against_oracle(inp, lam, splits, o, lse, mask, mla=False):
    """Mask against the oracle's (outside the +-1e-3 band), outputs against the
    oracle run on the device's own mask."""
    Lk = inp.k.shape[2]
    nb = (Lk + 63) // 64
    bits = unpack_mask(mask.cpu().numpy(), nb)
    causal = inp.q.shape[2] > 1
    v = inp.k if mla else inp.v
    kw = dict(scale=inp.scale, lam=lam, causal=causal, is_decode=True, num_splits=splits, BN=64)
    if mla:
        kw.update(dv=512, v_row_stride=576)
    ref = oracle.attention(inp.q, inp.k, v, **kw)
    nd, _ = compare_masks(bits, ref, lam)
    assert nd == 0, f"{nd} mask bits differ outside the band"
    fr = oracle.attention(inp.q, inp.k, v, forced_skip=bits, **kw)
    assert_outputs_close(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), fr["o"], fr["lse"])


def test_noalloc_wide_tile_and_mla_after_another_call(bl):
    # a 32-row tile (32 query heads on one KV head: the tcgen05 decode) and a
    # 128-head MLA decode at its default split count (2), run back to back after
    # a different call has left its partials in the array; each checked against
    # the oracle on its own mask and against the allocating entry point
    warm = planted_decode(3, 16, 4, 4000, 128, seed=33, reading="blk")
    bl.decode_noalloc(to_dev(warm.q), to_dev(warm.k), to_dev(warm.v), scale=warm.scale, lam=0.1, num_splits=7)
    wide = planted_decode(2, 32, 1, 6000, 128, seed=34, reading="blk")
    mla = planted_mla(4, 128, 3000, seed=35, reading="blk")
    runs = []
    for inp, lam, splits, is_mla in ((wide, 0.05, 16, False), (mla, 0.05, None, True)):
        q, k = to_dev(inp.q), to_dev(inp.k)
        v = k if is_mla else to_dev(inp.v)
        kw = dict(scale=inp.scale, lam=lam, num_splits=splits, dv=512 if is_mla else None)
        runs.append((inp, lam, 2 if is_mla else splits, is_mla, bl.decode_noalloc(q, k, v, **kw),
                     bl.decode(q, k, v, **kw)))
    torch.cuda.synchronize()
    for inp, lam, splits, is_mla, (o1, l1, m1, c1), (o2, l2, m2, c2) in runs:
        assert torch.equal(m1, m2) and torch.equal(c1, c2)
        emax, emean = _close(o1, o2)
        assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS
        assert float((l1 - l2).abs().max()) <= LSE_ABS
        _against_oracle(inp, lam, splits, o1, l1, m1, mla=is_mla)


def test_noalloc_rejects_sizes_beyond_the_scratch(bl):
    limit = bl.NOALLOC_SCRATCH_BYTES
    B, Hq, splits = 64, 128, 16
    assert bl.decode_workspace_bytes(B, Hq, 1, 128, splits) > limit
    q = torch.zeros((B, Hq, 1, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, 8, 128, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bl.BlasstError) as e:
        bl.decode_noalloc(q, k, k, scale=0.1, num_splits=splits)
    assert e.value.status == 3
    assert "scratch" in str(e.value)
