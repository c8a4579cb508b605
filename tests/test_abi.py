"""The C-ABI library: it loads, exports what include/blasst.h declares, and its
host-only logic (argument checks, calibration fit and threshold, visited-pair
counts, workspace size) behaves as specified.  No GPU needed: every call here
returns before any CUDA work."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
from synth import planted_prefill, random_normal

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bl():
    from block_sparse_flashattention_tcgen05_b200 import build

    build.build()
    import block_sparse_flashattention_tcgen05_b200 as m

    m.lib()
    return m


def declared_symbols():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            with open(os.path.join(ROOT, "include", h)) as f:
                names += re.findall(r"BLASST_API\s+[\w\s\*]+?\b(blasst_\w+)\s*\(", f.read())
    return names


def test_exports_every_declared_symbol(bl):
    names = declared_symbols()
    assert len(names) >= 9
    L = bl.lib()
    for n in names:
        assert hasattr(L, n), n


FAKE = 0x10000  # an aligned non-null address; never dereferenced on these paths


def _call(bl, fn, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=1, Lq=1, Lk=256, d=128, scale=0.088,
                lam=0.0, causal=0, mask=None, count=None, stream=None, opts=None)
    args.update(over)
    opts = args["opts"] or bl.Opts()
    f = getattr(bl.lib(), fn)
    return f(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["Hq"], args["Hkv"],
             args["Lq"], args["Lk"], args["d"], args["scale"], args["lam"], args["causal"], args["mask"],
             args["count"], args["stream"], ctypes.byref(opts))


@pytest.mark.parametrize("fn", ["blasst_decode", "blasst_prefill"])
def test_invalid_arguments_rejected_before_launch(bl, fn):
    assert _call(bl, fn, q=None) == 1
    assert _call(bl, fn, k=None) == 1
    assert _call(bl, fn, v=None) == 1
    assert _call(bl, fn, o=None) == 1
    assert _call(bl, fn, lse=None) == 1
    assert _call(bl, fn, B=0) == 1
    assert _call(bl, fn, Hq=6, Hkv=4) == 1
    assert _call(bl, fn, lam=-0.5) == 1
    assert _call(bl, fn, lam=1.0) == 1
    assert _call(bl, fn, lam=float("nan")) == 1
    assert _call(bl, fn, lam=float("inf")) == 1
    assert _call(bl, fn, scale=0.0) == 1
    assert _call(bl, fn, scale=float("nan")) == 1
    assert _call(bl, fn, causal=1, Lq=300, Lk=256) == 1
    assert _call(bl, fn, q=FAKE + 8) == 1                    # misaligned
    assert _call(bl, fn, d=64) == 2                          # head dim not built
    assert _call(bl, fn, opts=bl.Opts(k_row_stride=130)) == 1  # stride not a multiple of 8
    assert _call(bl, fn, opts=bl.Opts(block_n=32)) == 2


def test_decode_unsupported_tile_and_small_workspace(bl):
    assert _call(bl, "blasst_decode", Hq=256, Hkv=1) == 2     # G * Lq > 128
    assert _call(bl, "blasst_decode", opts=bl.Opts(workspace=FAKE, workspace_bytes=64)) == 3
    assert _call(bl, "blasst_decode", opts=bl.Opts(workspace=FAKE + 16, workspace_bytes=1 << 30)) == 1


def test_split_seeding_only_on_decode(bl):
    assert _call(bl, "blasst_prefill", opts=bl.Opts(seed_splits=1)) == 2     # prefill has no splits
    mla = dict(dv=512, k_row_stride=576, v_row_stride=576)
    # MLA takes seeding: the arguments pass (no device here, so the call then fails on CUDA)
    assert _call(bl, "blasst_decode", d=576, Hq=128, opts=bl.Opts(seed_splits=1, **mla)) not in (1, 2, 3)
    # so do wide d = 128 tiles (64 query heads on one KV head: the tcgen05 decode)
    assert _call(bl, "blasst_decode", Hq=64, Hkv=1, opts=bl.Opts(seed_splits=1)) not in (1, 2, 3)


def _paged(bl, **over):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, o=FAKE, lse=FAKE, table=FAKE, lens=FAKE, B=2, Hq=4, Hkv=1, Lq=1,
             max_pages=8, num_pages=16, d=128, scale=0.088, lam=0.0, causal=0)
    a.update(over)
    return bl.lib().blasst_decode_paged(a["q"], a["kp"], a["vp"], a["o"], a["lse"], a["table"], a["lens"], a["B"],
                                        a["Hq"], a["Hkv"], a["Lq"], a["max_pages"], a["num_pages"], a["d"],
                                        a["scale"], a["lam"], a["causal"], None, None, None,
                                        ctypes.byref(a.get("opts") or bl.Opts()))


def test_paged_decode_arguments_rejected_before_launch(bl):
    assert _paged(bl, table=None) == 1
    assert _paged(bl, lens=None) == 1
    assert _paged(bl, table=FAKE + 2) == 1                     # misaligned int32 array
    assert _paged(bl, max_pages=0) == 1
    assert _paged(bl, num_pages=0) == 1
    assert _paged(bl, d=576) == 2                               # paged MLA cache: not built
    assert _paged(bl, Hq=256) == 2                              # G * Lq > 128
    assert _paged(bl, lam=1.0) == 1
    assert _paged(bl, opts=bl.Opts(k_row_stride=256)) == 2      # pages are dense rows


def _bwd(bl, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, Hq=4, Hkv=2, Lq=256,
             Lk=256, d=128, scale=0.088, causal=1, mask=None)
    a.update(over)
    return bl.lib().blasst_prefill_backward(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"],
                                            a["dv"], a["B"], a["Hq"], a["Hkv"], a["Lq"], a["Lk"], a["d"],
                                            a["scale"], a["causal"], a["mask"], None,
                                            ctypes.byref(a.get("opts") or bl.Opts()))


def test_backward_arguments_rejected_before_launch(bl):
    for name in ("q", "k", "v", "o", "lse", "do", "dq", "dk", "dv"):
        assert _bwd(bl, **{name: None}) == 1, name
    for name in ("q", "k", "v", "o", "do", "dq", "dk", "dv"):
        assert _bwd(bl, **{name: FAKE + 8}) == 1, name
    assert _bwd(bl, lse=FAKE + 2) == 1
    assert _bwd(bl, mask=FAKE + 2) == 1
    assert _bwd(bl, Hq=3) == 1                      # Hq not a multiple of Hkv
    assert _bwd(bl, Lq=300, Lk=256) == 1            # causal needs Lq <= Lk
    assert _bwd(bl, scale=-1.0) == 1
    assert _bwd(bl, d=64) == 2
    assert _bwd(bl, opts=bl.Opts(dv=64)) == 2
    assert _bwd(bl, opts=bl.Opts(k_row_stride=256)) == 2
    assert _bwd(bl, opts=bl.Opts(block_n=64)) == 2
    assert _bwd(bl, opts=bl.Opts(seed_splits=1)) == 2
    assert _bwd(bl, opts=bl.Opts(workspace=FAKE, workspace_bytes=64)) == 3
    assert _bwd(bl, opts=bl.Opts(workspace=FAKE + 16, workspace_bytes=1 << 30)) == 1


def test_backward_workspace_bytes(bl):
    f = bl.lib().blasst_backward_workspace_bytes
    # 2 x 32 rows padded to 2 tiles: fp32 accumulator of 128 columns + two fp32 rows, 256-byte rounded
    rows = 2 * 32 * 256
    assert f(2, 32, 200) == rows * 128 * 4 + 2 * rows * 4
    assert f(1, 1, 1) == 128 * 128 * 4 + 2 * 512
    assert f(0, 1, 1) == 0 and f(1, 1, 0) == 0


def _fp8(bl, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=8, Hkv=1, Lq=1, Lk=256, d=128, scale=0.088,
             ks=0.01, vs=0.01, lam=0.0, causal=0)
    a.update(over)
    return bl.lib().blasst_decode_fp8(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Lq"],
                                      a["Lk"], a["d"], a["scale"], a["ks"], a["vs"], a["lam"], a["causal"], None,
                                      None, None, ctypes.byref(a.get("opts") or bl.Opts()))


def test_fp8_decode_arguments_rejected_before_launch(bl):
    assert _fp8(bl, v=None) == 1
    assert _fp8(bl, k=FAKE + 8) == 1
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert _fp8(bl, ks=bad) == 1 and _fp8(bl, vs=bad) == 1
    assert _fp8(bl, d=64) == 2
    assert _fp8(bl, Hq=32) == 2                      # more than 16 rows per tile
    assert _fp8(bl, opts=bl.Opts(k_row_stride=256)) == 2
    assert _fp8(bl, lam=1.0) == 1


def test_pick_splits(bl):
    f = bl.lib().blasst_decode_pick_splits
    assert f(32, 8, 32768, 148) == 10       # ceil(16 * 148 / 256)
    assert f(1, 8, 32768, 148) == 16        # capped at 32 blocks (2048 keys) per split
    assert f(4, 8, 32768, 148) == 16
    assert f(1, 1, 1 << 20, 148) == 64      # never more than 64
    assert f(1, 8, 2047, 148) == 1          # short cache: one split
    assert f(4096, 8, 32768, 148) == 1      # large batch fills the device by itself
    for B in (1, 2, 8, 64, 512):
        s = f(B, 8, 65536, 132)
        assert 1 <= s <= max(1, 1024 // 32) and s == max(1, min(min(64, 1024 // 32), -(-16 * 132 // (B * 8))))
    assert f(0, 8, 100, 148) == 1 and f(1, 8, 100, 0) == 1


def test_pick_splits_wide_tiles(bl):
    f = bl.lib().blasst_decode_pick_splits_rows
    narrow = bl.lib().blasst_decode_pick_splits
    for B, Hkv, rows in ((32, 8, 4), (1, 8, 16), (4, 2, 1)):   # tiles of up to 16 rows: the narrow rule
        assert f(B, Hkv, rows, 32768, 148) == narrow(B, Hkv, 32768, 148)
    assert f(64, 1, 128, 32768, 148) == 9     # floor(4 * 148 / 64): 576 CTAs, under two waves of two per SM
    assert f(32, 1, 128, 32768, 148) == 16    # floor(592 / 32) = 18, capped at 32 blocks per split
    assert f(256, 1, 128, 32768, 148) == 2
    assert f(1024, 1, 64, 32768, 148) == 1    # the batch fills two waves by itself
    assert f(8, 1, 17, 2047, 148) == 1        # short cache: one split
    for B in (1, 3, 16, 64, 200):
        want = 4 * 132 // (B * 2)
        assert f(B, 2, 32, 65536, 132) == max(1, min(min(64, 1024 // 32), want))
    assert f(0, 1, 128, 100, 148) == 1 and f(1, 1, 128, 100, 0) == 1


def test_adaptive_splits_only_where_supported(bl):
    mla = dict(num_splits=-1, dv=512, k_row_stride=576, v_row_stride=576)
    assert _call(bl, "blasst_decode", d=576, opts=bl.Opts(**mla)) == 1   # MLA
    assert _call(bl, "blasst_decode_noalloc", d=576, opts=bl.Opts(**mla)) == 1
    assert _call(bl, "blasst_decode", opts=bl.Opts(num_splits=-2)) == 1
    assert _call(bl, "blasst_decode_noalloc", opts=bl.Opts(num_splits=-2)) == 1


def test_noalloc_sizes_partials_as_the_decode_does(bl):
    """The no-allocation call sizes its partials with the split count and value
    width blasst_decode will use: MLA (d = 576, dv = 512) defaults to 2 splits,
    so batch 4 x 128 heads needs about 2 MiB and passes the size check, while
    16 splits at batch 64 exceed the fixed array and are refused up front."""
    mla = dict(dv=512, k_row_stride=576, v_row_stride=576)
    limit = bl.NOALLOC_SCRATCH_BYTES
    assert bl.decode_workspace_bytes(4, 128, 1, 512, 2) < limit < bl.decode_workspace_bytes(4, 128, 1, 512, 16)
    # the 2-split size passes; what follows needs the device (no device here: a CUDA error, not a size error)
    assert _call(bl, "blasst_decode_noalloc", B=4, Hq=128, d=576, opts=bl.Opts(**mla)) != 3
    assert bl.decode_workspace_bytes(64, 128, 1, 512, 16) > limit
    assert _call(bl, "blasst_decode_noalloc", B=64, Hq=128, d=576, opts=bl.Opts(num_splits=16, **mla)) == 3
    assert _call(bl, "blasst_decode_noalloc", B=64, Hq=128, opts=bl.Opts(num_splits=16)) == 3
    assert _call(bl, "blasst_decode_noalloc", opts=bl.Opts(workspace=FAKE, workspace_bytes=1 << 20)) == 1


def test_calibrate_requires_gaps_and_valid_mode(bl):
    assert _call(bl, "blasst_calibrate") == 1                 # no gaps_out
    assert _call(bl, "blasst_calibrate", opts=bl.Opts(mode=7, gaps_out=FAKE)) == 1


def test_old_struct_size_reads_as_defaults(bl):
    # an older caller that only knows the first field: everything else defaults
    o = bl.Opts(block_n=32)
    o.struct_size = ctypes.sizeof(ctypes.c_size_t)
    assert _call(bl, "blasst_decode", d=64, opts=o) == 2      # d=64 unsupported, block_n ignored


def test_status_strings(bl):
    L = bl.lib()
    for s in range(6):
        assert L.blasst_status_string(s)
    assert L.blasst_last_error() is not None


def test_calibrate_fit_exact(bl):
    alpha, beta = 2.5, 7.0
    Ls = np.array([8192, 16384, 32768, 65536.0])
    s = np.array([0.3, 0.5, 0.6, 0.75])
    lam = alpha * np.exp(beta * s) / Ls
    a, b = bl.calibrate_fit(Ls, lam, s)
    assert abs(a - alpha) < 1e-9 and abs(b - beta) < 1e-9
    ao, bo = oracle.calibrate_fit(Ls, lam * (1 + 0.01 * np.arange(4)), s)
    a2, b2 = bl.calibrate_fit(Ls, lam * (1 + 0.01 * np.arange(4)), s)
    assert abs(a2 - ao) < 1e-9 * ao and abs(b2 - bo) < 1e-9


def test_calibrate_fit_rejects_bad_input(bl):
    with pytest.raises(bl.BlasstError):
        bl.calibrate_fit([8192], [0.001], [0.5])
    with pytest.raises(bl.BlasstError):
        bl.calibrate_fit([8192, 8192], [0.001, 0.002], [0.5, 0.5])


def test_calibrate_threshold_agrees_with_oracle_gaps(bl):
    inp = planted_prefill(1, 2, 1, 2048, 32, seed=13, reading="blk", boost=True)
    r = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.0, causal=True, BM=64, BN=32)
    gaps = np.where(r["visited"] == 1, r["gaps"], np.nan).astype(np.float32)
    for target in (0.2, 0.5, 0.7):
        lam, ach = bl.calibrate_threshold(gaps, target)
        lam_o, ach_o = oracle.threshold_for_sparsity(r["gaps"], r["visited"], target)
        assert abs(ach - ach_o) <= 2.0 / r["n_visited"]
        rr = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=lam, causal=True, BM=64, BN=32)
        assert abs(rr["n_skipped"] / rr["n_visited"] - ach) <= 2.0 / r["n_visited"]


@pytest.mark.parametrize("shape", [(1, 4, 2, 300, 300, 1), (2, 2, 1, 1024, 1024, 1), (1, 2, 2, 100, 700, 1),
                                   (1, 2, 2, 100, 700, 0), (1, 1, 1, 128, 128, 1)])
def test_visited_pairs_prefill_matches_oracle(bl, shape):
    B, Hq, Hkv, Lq, Lk, causal = shape
    inp = random_normal(B, Hq, Hkv, Lq, Lk, 8, seed=0)
    r = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.0, causal=bool(causal), BM=128, BN=128)
    assert bl.visited_pairs(B, Hq, Hkv, Lq, Lk, causal, False) == r["n_visited"]


@pytest.mark.parametrize("shape", [(2, 8, 2, 1, 1000, 0), (1, 4, 1, 3, 777, 1)])
def test_visited_pairs_decode_matches_oracle(bl, shape):
    B, Hq, Hkv, Lq, Lk, causal = shape
    inp = random_normal(B, Hq, Hkv, Lq, Lk, 8, seed=0)
    r = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=0.0, causal=bool(causal), is_decode=True,
                         num_splits=4, BN=64)
    assert bl.visited_pairs(B, Hq, Hkv, Lq, Lk, causal, True) == r["n_visited"]


def test_visited_pairs_of_benchmark_shapes(bl):
    # 1024-token MHA prefill: 36 pairs; 32K and 64K GQA prefill; decode 32 x 8 x 512
    assert bl.visited_pairs(1, 1, 1, 1024, 1024, 1, False) == 36
    assert bl.visited_pairs(1, 32, 8, 32768, 32768, 1, False) == 32 * 256 * 257 // 2
    assert bl.visited_pairs(1, 32, 8, 65536, 65536, 1, False) == 32 * 512 * 513 // 2
    assert bl.visited_pairs(32, 32, 8, 1, 32768, 0, True) == 32 * 8 * 512


def test_workspace_bytes(bl):
    rows, S, dv = 32 * 32, 16, 128
    # partial O, partial lse, one skip-count slot per split CTA (bounded by B * Hq * S)
    expect = -(-rows * S * dv * 4 // 256) * 256 + -(-rows * S * 4 // 256) * 256 + -(-32 * 32 * S * 4 // 256) * 256
    assert bl.decode_workspace_bytes(32, 32, 1, 128, 16) == expect
    assert bl.decode_workspace_bytes(32, 32, 1, 0, 0) == expect
