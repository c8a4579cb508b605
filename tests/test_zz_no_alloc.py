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

from _parity import O_MAX_ABS, O_MEAN_ABS, LSE_ABS
from synth import planted_decode

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
