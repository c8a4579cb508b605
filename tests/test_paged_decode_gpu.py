"""GPU parity of decode over a paged, ragged KV cache (blasst_decode_paged).

The cache is only a storage layout: per sequence, the result must equal the
oracle run on that sequence's keys gathered back into a contiguous cache, with
the same split count.
"""
import numpy as np
import pytest

import oracle
from _parity import assert_outputs_close, bf16_tensor_to_f64, compare_masks, unpack_mask
from synth import planted_decode

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
PAGE = 64


@pytest.fixture(scope="module")
def bl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_tcgen05_b200 as m

    m.lib()
    return m


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def make_paged(inp, lens, seed, spare_pages=5, max_pages=None):
    """Scatter each sequence's first lens[b] keys into randomly placed pages.

    Keys past a sequence's end inside its last page hold junk (other keys), so
    masking is exercised; table entries past a sequence's pages are invalid."""
    rng = np.random.default_rng(seed)
    B, Hkv, Lmax, d = inp.k.shape
    npg = [(n + PAGE - 1) // PAGE for n in lens]
    max_pages = max(max(npg), 1) if max_pages is None else max_pages
    num_pages = sum(npg) + spare_pages
    order = rng.permutation(num_pages)
    kp = rng.integers(0, 1 << 15, size=(num_pages, Hkv, PAGE, d)).astype(np.uint16) & np.uint16(0x3F7F)
    vp = kp.copy()
    table = np.full((B, max_pages), 1 << 30, np.int32)
    nxt = 0
    for b in range(B):
        for i in range(npg[b]):
            pg = int(order[nxt])
            nxt += 1
            table[b, i] = pg
            lo, hi = i * PAGE, min((i + 1) * PAGE, Lmax)
            kp[pg, :, : hi - lo] = inp.k[b, :, lo:hi]
            vp[pg, :, : hi - lo] = inp.v[b, :, lo:hi]
    return kp, vp, table, num_pages


def run_paged(bl, inp, lens, lam, splits, causal=False, seed_splits=False, seed=0, max_pages=None):
    kp, vp, table, _ = make_paged(inp, lens, seed, max_pages=max_pages)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, mask, cnt = bl.decode_paged(
        to_dev(inp.q), to_dev(kp), to_dev(vp), torch.from_numpy(table).cuda(),
        torch.tensor(lens, dtype=torch.int32, device="cuda"), scale=inp.scale, lam=lam, causal=causal,
        num_splits=splits, status_word=st, seed_splits=seed_splits)
    torch.cuda.synchronize()
    return o, lse, mask, cnt, st.item(), table.shape[1]


def check_paged(bl, inp, lens, lam, splits, causal=False, seed_splits=False, seed=0):
    o, lse, mask, cnt, status, max_pages = run_paged(bl, inp, lens, lam, splits, causal, seed_splits, seed)
    assert status == 0
    B, Hq, Lq, d = inp.q.shape
    Hkv = inp.k.shape[1]
    bits = unpack_mask(mask.cpu().numpy(), max_pages).reshape(B, Hkv, max_pages)
    og = bf16_tensor_to_f64(o)
    lg = lse.cpu().numpy().astype(np.float64)
    total = 0
    for b, n in enumerate(lens):
        nb = (n + PAGE - 1) // PAGE
        assert not bits[b, :, nb:].any(), "mask bit past the sequence's last block"
        kw = dict(scale=inp.scale, lam=lam, causal=causal, is_decode=True, num_splits=splits, BN=PAGE,
                  seed_splits=seed_splits)
        qb, kb, vb = inp.q[b:b + 1], inp.k[b:b + 1, :, :n], inp.v[b:b + 1, :, :n]
        ref = oracle.attention(qb, kb, vb, **kw)
        nd, _ = compare_masks(bits[b, :, :nb], ref, lam)
        assert nd == 0, f"sequence {b}: {nd} mask bits differ outside the band"
        fr = oracle.attention(qb, kb, vb, forced_skip=bits[b, :, :nb], **kw)
        assert_outputs_close(og[b:b + 1], lg[b:b + 1], fr["o"], fr["lse"])
        total += int(bits[b].sum())
    assert int(cnt.item()) == total
    return bits


@pytest.mark.parametrize("lam", [0.0, 0.02, 0.5])
@pytest.mark.parametrize("splits", [1, 4, 16])
def test_paged_ragged(bl, lam, splits):
    inp = planted_decode(4, 8, 2, 2600, 128, seed=31, reading="blk")
    check_paged(bl, inp, [2600, 64, 65, 1000], lam, splits, seed=splits)


def test_paged_causal_two_queries(bl):
    inp = planted_decode(3, 8, 1, 3000, 128, Lq=2, seed=32, reading="blk")
    check_paged(bl, inp, [3000, 700, 129], 0.1, 3, causal=True)


@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_paged_seeded(bl, lam):
    inp = planted_decode(3, 8, 2, 4000, 128, seed=33, reading="blk")
    check_paged(bl, inp, [4000, 1500, 333], lam, 8, seed_splits=True)


def test_paged_mqa_wide_tile(bl):
    inp = planted_decode(3, 64, 1, 2600, 128, seed=38, reading="blk")
    check_paged(bl, inp, [2600, 65, 1300], 0.05, 4)


@pytest.mark.parametrize("lam", [0.0, 0.05])
def test_paged_mqa_wide_tile_seeded(bl, lam):
    # seeded splits on the tcgen05 decode over ragged pages (one sequence shorter than a split)
    inp = planted_decode(3, 64, 1, 2600, 128, seed=38, reading="blk")
    check_paged(bl, inp, [2600, 65, 1300], lam, 6, seed_splits=True)


def test_paged_single_key_sequences(bl):
    inp = planted_decode(3, 4, 1, 200, 128, seed=34, reading="lit")
    check_paged(bl, inp, [1, 63, 200], 0.3, 16)


def test_paged_identity_table_equals_contiguous(bl):
    # pages laid out in sequence order: same bytes through both tensor maps, same result bit for bit
    inp = planted_decode(2, 8, 2, 64 * 40, 128, seed=35, reading="blk")
    B, Hkv, L, d = inp.k.shape
    kp = np.ascontiguousarray(inp.k.reshape(B, Hkv, L // PAGE, PAGE, d).transpose(0, 2, 1, 3, 4)).reshape(-1, Hkv,
                                                                                                           PAGE, d)
    vp = np.ascontiguousarray(inp.v.reshape(B, Hkv, L // PAGE, PAGE, d).transpose(0, 2, 1, 3, 4)).reshape(-1, Hkv,
                                                                                                           PAGE, d)
    table = np.arange(B * (L // PAGE), dtype=np.int32).reshape(B, L // PAGE)
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    q = to_dev(inp.q)
    o1, l1, m1, c1 = bl.decode_paged(q, to_dev(kp), to_dev(vp), torch.from_numpy(table).cuda(), lens,
                                     scale=inp.scale, lam=0.05, num_splits=4)
    o2, l2, m2, c2 = bl.decode(q, to_dev(inp.k), to_dev(inp.v), scale=inp.scale, lam=0.05, num_splits=4)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(m1, m2) and torch.equal(c1, c2)


def test_paged_empty_sequence(bl):
    inp = planted_decode(2, 4, 1, 500, 128, seed=36, reading="blk")
    o, lse, mask, cnt, status, _ = run_paged(bl, inp, [500, 0], 0.05, 4, max_pages=8)
    assert status == 0
    assert torch.all(o[1] == 0) and torch.all(torch.isneginf(lse[1]))
    assert int(mask[1].abs().sum().item()) == 0


def test_paged_bad_page_and_length_are_reported(bl):
    # an out-of-range page reads zeros and a too-long length is clamped; both raise status bit 2
    inp = planted_decode(2, 4, 1, 300, 128, seed=37, reading="lit")
    kp, vp, table, num_pages = make_paged(inp, [300, 300], 1)
    table[0, 2] = num_pages + 7
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bl.decode_paged(to_dev(inp.q), to_dev(kp), to_dev(vp), torch.from_numpy(table).cuda(),
                    torch.tensor([300, 300], dtype=torch.int32, device="cuda"), scale=inp.scale, num_splits=2,
                    status_word=st)
    torch.cuda.synchronize()
    assert st.item() & 2
    st.zero_()
    kp, vp, table, _ = make_paged(inp, [300, 300], 2)
    bl.decode_paged(to_dev(inp.q), to_dev(kp), to_dev(vp), torch.from_numpy(table).cuda(),
                    torch.tensor([300, 10 ** 6], dtype=torch.int32, device="cuda"), scale=inp.scale, num_splits=2,
                    status_word=st)
    torch.cuda.synchronize()
    assert st.item() & 2
