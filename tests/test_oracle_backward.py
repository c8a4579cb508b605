"""Pins of oracle.attention_backward (the fixed-mask gradient), CPU only.

Each pin holds the oracle to something other than its own formulas:
  - central finite differences of a separately written masked-attention
    forward (explicit loops) on tiny fp64 inputs, with a skip mask, causal
    alignment and two query heads per KV head;
  - its forward part (o, lse) against the C oracle's forward run with the
    same forced mask on bf16 inputs (ties the mask indexing to that code);
  - torch autograd of scaled_dot_product_attention in fp64 when nothing is
    skipped (a library routine);
  - invariants that hold for any mask: keys' gradients sum to zero (softmax
    does not change when every key moves by the same vector), values'
    gradients sum to the summed dO of rows that see a key, a key block that
    every tile skipped gets exactly zero gradient, and linearity in dO.
"""
import math

import numpy as np
import pytest

import oracle
from synth import planted_prefill

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def loop_forward(Q, K, V, scale, causal, skip, BM, BN):
    """O for masked attention, by explicit loops over rows and keys (tiny sizes)."""
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    G = Hq // Hkv
    O = np.zeros((B, Hq, Lq, V.shape[3]))
    for b in range(B):
        for h in range(Hq):
            for r in range(Lq):
                ks = [c for c in range(Lk)
                      if (not causal or c <= r + Lk - Lq) and not (skip is not None and skip[b, h, r // BM, c // BN])]
                if not ks:
                    continue
                sc = [scale * sum(Q[b, h, r, i] * K[b, h // G, c, i] for i in range(d)) for c in ks]
                mx = max(sc)
                w = [math.exp(x - mx) for x in sc]
                z = sum(w)
                for c, wc in zip(ks, w):
                    O[b, h, r] += (wc / z) * V[b, h // G, c]
    return O


def tiny_case(seed, causal, Lq=5, Lk=7):
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, d, dv, BM, BN = 1, 2, 1, 3, 2, 2, 3
    Q = rng.standard_normal((B, Hq, Lq, d))
    K = rng.standard_normal((B, Hkv, Lk, d))
    V = rng.standard_normal((B, Hkv, Lk, dv))
    W = rng.standard_normal((B, Hq, Lq, dv))
    nq, nb = -(-Lq // BM), -(-Lk // BN)
    skip = (rng.random((B, Hq, nq, nb)) < 0.4).astype(np.uint8)
    skip[..., 0] = 0  # the first block of every tile is kept
    return Q, K, V, W, skip, BM, BN


@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(causal):
    Q, K, V, W, skip, BM, BN = tiny_case(3 + causal, causal)
    scale = 0.7
    g = oracle.attention_backward(Q, K, V, W, scale=scale, causal=causal, skip=skip, BM=BM, BN=BN)

    def loss(Q_, K_, V_):
        return float((loop_forward(Q_, K_, V_, scale, causal, skip, BM, BN) * W).sum())

    h = 1e-6
    for name, X, grad in (("q", Q, g["dq"]), ("k", K, g["dk"]), ("v", V, g["dv"])):
        fd = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args_p = [Xp if n == name else Y for n, Y in (("q", Q), ("k", K), ("v", V))]
            args_m = [Xm if n == name else Y for n, Y in (("q", Q), ("k", K), ("v", V))]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8, err_msg=f"d{name}")


def test_forward_part_matches_c_oracle_with_forced_mask():
    inp = planted_prefill(1, 4, 2, 300, 128, seed=5, reading="blk")
    scale = 1 / math.sqrt(128)
    rng = np.random.default_rng(9)
    nq, nb = 3, 3
    skip = (rng.random((1 * 4 * nq, nb)) < 0.5).astype(np.uint8)
    skip[:, 0] = 0
    ref = oracle.attention(inp.q, inp.k, inp.v, scale=scale, lam=0.0, causal=True, forced_skip=skip)
    do = np.zeros(inp.q.shape, np.uint16)
    g = oracle.attention_backward(inp.q, inp.k, inp.v, do, scale=scale, causal=True, skip=skip)
    np.testing.assert_allclose(g["o"], ref["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["lse"], ref["lse"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,Lq,Lk", [(False, 40, 56), (True, 40, 56), (True, 64, 64)])
def test_dense_matches_torch_autograd(causal, Lq, Lk):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(11)
    B, Hq, Hkv, d = 2, 4, 2, 16
    Q = rng.standard_normal((B, Hq, Lq, d))
    K = rng.standard_normal((B, Hkv, Lk, d))
    V = rng.standard_normal((B, Hkv, Lk, d))
    W = rng.standard_normal((B, Hq, Lq, d))
    scale = 0.3
    g = oracle.attention_backward(Q, K, V, W, scale=scale, causal=causal, BM=16, BN=16)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    G = Hq // Hkv
    mask = None
    if causal:
        mask = torch.tensor(np.arange(Lk)[None, :] <= np.arange(Lq)[:, None] + (Lk - Lq))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1), attn_mask=mask, scale=scale)
    (out * torch.tensor(W)).sum().backward()
    np.testing.assert_allclose(g["o"], out.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dq"], tq.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dk"], tk.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dv"], tv.grad.numpy(), rtol=0, atol=1e-11)


def masked_case(seed, causal):
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, Lq, Lk, d, BM, BN = 2, 4, 2, 48, 64, 8, 8, 8
    Q = rng.standard_normal((B, Hq, Lq, d))
    K = rng.standard_normal((B, Hkv, Lk, d))
    V = rng.standard_normal((B, Hkv, Lk, d))
    W = rng.standard_normal((B, Hq, Lq, d))
    skip = (rng.random((B * Hq * (Lq // BM), Lk // BN)) < 0.5).astype(np.uint8)
    skip[:, 0] = 0
    return Q, K, V, W, skip, BM, BN


@pytest.mark.parametrize("causal", [False, True])
def test_invariants_any_mask(causal):
    Q, K, V, W, skip, BM, BN = masked_case(21, causal)
    skip.reshape(2, 4, 6, 8)[:, :, :, 5] = 1  # key block 5 skipped by every tile
    g = oracle.attention_backward(Q, K, V, W, scale=0.5, causal=causal, skip=skip, BM=BM, BN=BN)
    np.testing.assert_allclose(g["dk"].sum(axis=2), 0.0, atol=1e-11)
    G = 2
    want = W.reshape(2, 2, G, 48, 8).sum(axis=(2, 3))  # every row sees key 0
    np.testing.assert_allclose(g["dv"].sum(axis=2), want, atol=1e-11)
    assert np.all(g["dk"][:, :, 40:48] == 0.0) and np.all(g["dv"][:, :, 40:48] == 0.0)
    # linearity in dO
    rng = np.random.default_rng(2)
    W2 = rng.standard_normal(W.shape)
    g2 = oracle.attention_backward(Q, K, V, W2, scale=0.5, causal=causal, skip=skip, BM=BM, BN=BN)
    g3 = oracle.attention_backward(Q, K, V, 2 * W + W2, scale=0.5, causal=causal, skip=skip, BM=BM, BN=BN)
    for n in ("dq", "dk", "dv"):
        np.testing.assert_allclose(g3[n], 2 * g[n] + g2[n], atol=1e-11)


def test_skipping_a_pair_only_changes_that_tiles_query_gradient():
    Q, K, V, W, skip, BM, BN = masked_case(23, False)
    skip[:] = 0
    a = oracle.attention_backward(Q, K, V, W, scale=0.5, causal=False, skip=skip, BM=BM, BN=BN)
    skip2 = skip.copy()
    skip2[3, 4] = 1  # (b=0, hq=0, tile 3) skips key block 4
    b = oracle.attention_backward(Q, K, V, W, scale=0.5, causal=False, skip=skip2, BM=BM, BN=BN)
    diff = np.abs(a["dq"] - b["dq"]).max(axis=3)
    changed = np.argwhere(diff > 0)
    assert changed.size and np.all(changed[:, 0] == 0) and np.all(changed[:, 1] == 0)
    assert np.all((changed[:, 2] >= 24) & (changed[:, 2] < 32))


@pytest.mark.parametrize("causal", [False, True])
def test_dq_rows_match_the_full_backward(causal):
    Q, K, V, W, skip, BM, BN = masked_case(31, causal)
    full = oracle.attention_backward(Q, K, V, W, scale=0.5, causal=causal, skip=skip, BM=BM, BN=BN)
    rows = [(0, 0, 0), (0, 3, 17), (1, 1, 47), (1, 2, 23), (0, 1, 8)]
    got = oracle.backward_dq_rows(Q, K, V, W, rows, scale=0.5, causal=causal, skip=skip, BM=BM, BN=BN)
    want = np.stack([full["dq"][b, h, r] for b, h, r in rows])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_two_key_closed_form():
    """One query, two keys (blocks of one key): with p = sigmoid(s0 - s1) the gradient is
    dq = scale p (1-p) (dO.(v0 - v1)) (k0 - k1), dk0 = -dk1 = scale p (1-p) (dO.(v0 - v1)) q,
    dv0 = p dO, dv1 = (1 - p) dO; skipping key 1's block leaves dq = dk = 0, dv0 = dO, dv1 = 0."""
    rng = np.random.default_rng(41)
    d = 5
    q = rng.standard_normal((1, 1, 1, d))
    k = rng.standard_normal((1, 1, 2, d))
    v = rng.standard_normal((1, 1, 2, d))
    do = rng.standard_normal((1, 1, 1, d))
    scale = 0.8
    s0, s1 = scale * q[0, 0, 0] @ k[0, 0, 0], scale * q[0, 0, 0] @ k[0, 0, 1]
    p = 1.0 / (1.0 + math.exp(s1 - s0))
    g = p * (1 - p) * (do[0, 0, 0] @ (v[0, 0, 0] - v[0, 0, 1]))
    out = oracle.attention_backward(q, k, v, do, scale=scale, causal=False, BM=1, BN=1)
    np.testing.assert_allclose(out["dq"][0, 0, 0], scale * g * (k[0, 0, 0] - k[0, 0, 1]), atol=1e-13)
    np.testing.assert_allclose(out["dk"][0, 0, 0], scale * g * q[0, 0, 0], atol=1e-13)
    np.testing.assert_allclose(out["dk"][0, 0, 1], -scale * g * q[0, 0, 0], atol=1e-13)
    np.testing.assert_allclose(out["dv"][0, 0], np.stack([p * do[0, 0, 0], (1 - p) * do[0, 0, 0]]), atol=1e-13)
    skipped = oracle.attention_backward(q, k, v, do, scale=scale, causal=False, BM=1, BN=1,
                                        skip=np.array([[0, 1]], np.uint8))
    assert np.all(skipped["dq"] == 0) and np.all(skipped["dk"] == 0)
    np.testing.assert_allclose(skipped["dv"][0, 0], np.stack([do[0, 0, 0], np.zeros(d)]), atol=1e-15)
