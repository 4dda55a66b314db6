"""Pins of the fp64 oracle to things other than itself.

Each test checks the oracle against a closed form, a library routine, a
special case with a textbook answer, an invariant, or an independent brute
force; the pages ("STILL: Selecting Tokens for Intra-Layer Hybrid Attention to
Linearize LLMs": [p1] jsqmd.com "Self-Saliency Score", "NP-Map",
"Chunk-Wise"; [p4] atlas.scime.ai "Approach") print no worked example.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special as sps
import torch

from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _problem(rng, B=1, H=2, Hkv=1, N=40, d=8, D=6, spread=1.5):
    q = _rand(rng, B, H, N, d) * np.exp(rng.normal(0, 0.5, (B, H, N, 1))) * spread
    k = _rand(rng, B, Hkv, N, d) * np.exp(rng.normal(0, 0.5, (B, Hkv, N, 1))) * spread
    v = _rand(rng, B, Hkv, N, d)
    wq = _rand(rng, H, d, D, scale=1 / math.sqrt(d))
    wk = _rand(rng, Hkv, d, D, scale=1 / math.sqrt(d))
    return q, k, v, wq, wk


# ---------------------------------------------------------------- saliency

@pytest.mark.parametrize("w", [1, 4, 8, 64])
def test_saliency_equals_closed_form(oracle_mod, w):
    """KL(p'||p) summed term by term equals -ln(1-p_ii) = softplus(s_ii - LSE_{j!=i} s_ij)."""
    rng = np.random.default_rng(1)
    q, k, *_ = _problem(rng, H=3, Hkv=1, N=70, d=16)
    dims = oracle_mod.Dims(B=1, H=3, Hkv=1, N=70, d=16, D=4, w=w, C=w, k=0 if w == 0 else 1)
    sigma, r = oracle_mod.saliency(dims, q, k)
    tau = 1 / math.sqrt(16)
    for h in range(3):
        for i in range(70):
            lo = max(0, i - w + 1)
            s = tau * (k[0, 0, lo:i + 1] @ q[0, h, i])
            if len(s) == 1:
                assert sigma[0, h, i] == math.inf
                continue
            closed = np.logaddexp(0.0, s[-1] - sps.logsumexp(s[:-1]))
            assert sigma[0, h, i] == pytest.approx(closed, rel=1e-11, abs=1e-13)
    assert np.allclose(r[0, 0], sigma[0].mean(0))


def test_saliency_window_beyond_sequence(oracle_mod):
    """A window longer than the sequence clips to [0, i]: the scores equal those of w = N."""
    rng = np.random.default_rng(14)
    q, k, *_ = _problem(rng, H=2, Hkv=1, N=30, d=8)
    base = dict(B=1, H=2, Hkv=1, N=30, d=8, D=4, k=1)
    s_n, _ = oracle_mod.saliency(oracle_mod.Dims(w=30, C=30, **base), q, k)
    s_big, _ = oracle_mod.saliency(oracle_mod.Dims(w=40, C=40, **base), q, k)
    np.testing.assert_array_equal(s_n, s_big)


def test_saliency_zero_query(oracle_mod):
    """q = 0: every logit is 0, so p_ii = 1/n and sigma = ln(n/(n-1)) with n the band size."""
    rng = np.random.default_rng(2)
    N, w = 50, 16
    k = _rand(rng, 1, 1, N, 8)
    q = np.zeros((1, 1, N, 8))
    sigma, _ = oracle_mod.saliency(oracle_mod.Dims(1, 1, 1, N, 8, 4, w, 16, 2), q, k)
    for i in range(N):
        n = min(w, i + 1)
        want = math.inf if n == 1 else math.log(n / (n - 1))
        assert sigma[0, 0, i] == pytest.approx(want, rel=1e-13)


def test_saliency_gqa_identical_heads(oracle_mod):
    """G identical query heads: the group score equals the single-head score."""
    rng = np.random.default_rng(3)
    q1, k, *_ = _problem(rng, H=1, Hkv=1, N=45, d=8)
    q4 = np.repeat(q1, 4, axis=1)
    s1, r1 = oracle_mod.saliency(oracle_mod.Dims(1, 1, 1, 45, 8, 4, 8, 8, 2), q1, k)
    s4, r4 = oracle_mod.saliency(oracle_mod.Dims(1, 4, 1, 45, 8, 4, 8, 8, 2), q4, k)
    np.testing.assert_allclose(r4, r1, rtol=1e-14)
    np.testing.assert_allclose(r1[0, 0], s1[0, 0], rtol=0)


def test_saliency_golden(oracle_mod):
    """Hand-derived values (tests/golden/saliency_hand.json)."""
    with open(os.path.join(GOLDEN, "saliency_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = np.array(c["q"], dtype=np.float64)[None, None, :, :]
        k = np.array(c["k"], dtype=np.float64)[None, None, :, :]
        N, d = q.shape[2], q.shape[3]
        dims = oracle_mod.Dims(1, 1, 1, N, d, 2, c["w"], c["w"], 1, scale=c["scale"])
        sigma, _ = oracle_mod.saliency(dims, q, k)
        for i, want in enumerate(c["sigma"]):
            want = math.inf if want == "inf" else want
            assert sigma[0, 0, i] == pytest.approx(want, rel=1e-9), (c["name"], i)


def test_merge_golden(oracle_mod):
    """Hand-derived outputs of two six-token layers (tests/golden/merge_hand.json): kept token,
    window, linear branch over the unkept token of the one decided chunk, one normaliser.  Checked
    for the C oracle and the numpy brute force, and, where the case says so, for the decode state
    machine run token by token (the chunk close at position 3 decides chunk 0 for positions 4, 5)."""
    from oracle import brute
    with open(os.path.join(GOLDEN, "merge_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        dm, x = c["dims"], c["inputs"]
        N, H = dm["N"], dm["H"]
        q = np.array(x["q"], dtype=np.float64).reshape(1, H, N, 1)
        k = np.array(x["k"], dtype=np.float64).reshape(1, 1, N, 1)
        v = np.array(x["v"], dtype=np.float64).reshape(1, 1, N, 1)
        wq = np.array(x["wq"], dtype=np.float64).reshape(H, 1, 1)
        wk = np.array(x["wk"], dtype=np.float64).reshape(1, 1, 1)
        idx = np.array(x["idx"], dtype=np.int32).reshape(1, 1, -1, 1) if "idx" in x else None
        dims = oracle_mod.Dims(1, H, 1, N, 1, 1, dm["w"], dm["C"], dm["k"], scale=dm["scale"])
        o = oracle_mod.prefill(dims, q, k, v, wq, wk, idx_in=idx)["o"]
        ob, _, _ = brute.layer(q, k, v, wq, wk, dm["w"], dm["C"], dm["k"], scale=dm["scale"], idx_in=idx)
        od = None
        if c.get("decode"):
            dec = oracle_mod.Decoder(dims, wq, wk)
            od = np.stack([dec.step(q[:, :, t], k[:, :, t], v[:, :, t])[0] for t in range(N)], axis=2)
        for e in c["expected"]:
            assert o[0, e["h"], e["i"], 0] == pytest.approx(e["o"], rel=1e-12), (c["name"], e)
            assert ob[0, e["h"], e["i"], 0] == pytest.approx(e["o"], rel=1e-12), (c["name"], e)
            if od is not None:
                assert od[0, e["h"], e["i"], 0] == pytest.approx(e["o"], rel=1e-12), (c["name"], e)


# ---------------------------------------------------------------- top-k

# ---------------------------------------------------------------- diagonal-only router

def test_diagonal_score_self_match_is_squared_norm(oracle_mod):
    """q_hi = k_gi for every head of the group: r_gi = tau * ||k_gi||^2 (norm from numpy's routine)."""
    rng = np.random.default_rng(21)
    B, H, Hkv, N, d = 2, 6, 2, 33, 16
    k = _rand(rng, B, Hkv, N, d)
    q = np.repeat(k, H // Hkv, axis=1)
    dims = oracle_mod.Dims(B=B, H=H, Hkv=Hkv, N=N, d=d, D=4, w=8, C=8, k=2)
    r = oracle_mod.diagonal_score(dims, q, k)
    np.testing.assert_allclose(r, np.linalg.norm(k, axis=-1) ** 2 / math.sqrt(d), rtol=1e-12)


def test_diagonal_score_gqa_mean_cancels(oracle_mod):
    """Heads of a group in pairs (q, -q): the group mean of the diagonal logits is 0."""
    rng = np.random.default_rng(22)
    q1 = _rand(rng, 1, 2, 20, 8)
    q = np.concatenate([q1, -q1], axis=1)  # heads 0,1 | 2,3 = -(0,1); one group of 4
    k = _rand(rng, 1, 1, 20, 8)
    dims = oracle_mod.Dims(B=1, H=4, Hkv=1, N=20, d=8, D=4, w=4, C=4, k=1)
    assert np.abs(oracle_mod.diagonal_score(dims, q, k)).max() < 1e-14


def test_diagonal_router_selects_like_saliency_when_band_logits_vanish(oracle_mod):
    """Keys orthogonal to every other token's query: each band logit s_ij (j != i) is 0, so
    sigma = softplus(s_ii - ln(n-1)) is increasing in s_ii at a fixed band size n; the per-chunk
    top-k of the diagonal router then equals that of the Self-Saliency Score."""
    rng = np.random.default_rng(23)
    N, C, w, kk = 64, 16, 16, 5
    d = N
    k = np.zeros((1, 1, N, d))
    q = np.zeros((1, 1, N, d))
    for i in range(N):  # token i lives on coordinate i only: <q_i, k_j> = 0 for j != i
        k[0, 0, i, i] = rng.uniform(0.5, 3.0)
        q[0, 0, i, i] = rng.uniform(0.5, 3.0)
    dims = oracle_mod.Dims(B=1, H=1, Hkv=1, N=N, d=d, D=4, w=w, C=C, k=kk)
    rd = oracle_mod.diagonal_score(dims, q, k)
    _, rs = oracle_mod.saliency(dims, q, k)
    # chunks past the first have full bands (n = w) for every row
    sel_d = oracle_mod.topk(dims, rd)[:, :, 1:]
    sel_s = oracle_mod.topk(dims, rs)[:, :, 1:]
    np.testing.assert_array_equal(sel_d, sel_s)


def test_npmap_single_feature_is_the_norm(oracle_mod):
    """D = 1: f(xW) = [1], so phi(x) = ||x|| whatever W is."""
    rng = np.random.default_rng(15)
    for _ in range(5):
        x, W = rng.standard_normal(7), rng.standard_normal((7, 1))
        np.testing.assert_allclose(oracle_mod.npmap(x[None, :], W)[0], [np.linalg.norm(x)], rtol=1e-15)


def test_topk_matches_sort(oracle_mod):
    """Top-k = first k of a sort by (score desc, index asc), reported ascending; ties and +inf."""
    rng = np.random.default_rng(4)
    B, Hkv, C, T, kk = 2, 3, 16, 5, 5
    N = C * T + 7
    r = rng.integers(0, 6, size=(B, Hkv, N)).astype(np.float64)   # many ties
    r[0, 0, 3] = math.inf
    r[1, 2, 20] = math.inf
    r[1, 2, 21] = math.inf
    idx = oracle_mod.topk(oracle_mod.Dims(B, 2 * Hkv, Hkv, N, 8, 8, C, C, kk), r)
    for b in range(B):
        for g in range(Hkv):
            for c in range(T):
                mem = list(range(c * C, (c + 1) * C))
                want = sorted(sorted(mem, key=lambda j: (-r[b, g, j], j))[:kk])
                assert list(idx[b, g, c]) == want


def test_topk_permutation(oracle_mod):
    """Distinct scores: permuting the scores inside a chunk permutes the kept set."""
    rng = np.random.default_rng(5)
    C, kk = 32, 7
    r = rng.standard_normal((1, 1, C))
    perm = rng.permutation(C)
    d = oracle_mod.Dims(1, 1, 1, C, 8, 8, C, C, kk)
    a = set(oracle_mod.topk(d, r)[0, 0, 0])
    bset = set(oracle_mod.topk(d, r[:, :, perm])[0, 0, 0])
    assert {int(perm[j]) for j in bset} == {int(j) for j in a}


# ---------------------------------------------------------------- NP-Map

def test_npmap_norm_and_direction(oracle_mod):
    """||phi(x)|| = ||x||; direction = softmax(xW) normalised (scipy); W = 0 gives ||x|| 1/sqrt(D); phi(0) = 0."""
    rng = np.random.default_rng(6)
    x = _rand(rng, 33, 16) * np.exp(rng.normal(0, 1, (33, 1)))
    W = _rand(rng, 16, 24, scale=0.5)
    phi = oracle_mod.npmap(x, W)
    np.testing.assert_allclose(np.linalg.norm(phi, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    f = sps.softmax(x @ W, axis=1)
    np.testing.assert_allclose(phi / np.linalg.norm(phi, axis=1, keepdims=True),
                               f / np.linalg.norm(f, axis=1, keepdims=True), rtol=1e-12)
    phi0 = oracle_mod.npmap(x, np.zeros((16, 24)))
    np.testing.assert_allclose(phi0, np.linalg.norm(x, axis=1, keepdims=True) / math.sqrt(24) * np.ones((1, 24)),
                               rtol=1e-13)
    assert np.all(oracle_mod.npmap(np.zeros((2, 16)), W) == 0)


# ---------------------------------------------------------------- routing + merge limits

@pytest.mark.parametrize("B,H,Hkv,N,C,m", [(1, 2, 1, 50, 8, 1), (2, 4, 2, 37, 6, 2), (1, 3, 3, 64, 16, 1)])
def test_all_kept_is_causal_softmax(oracle_mod, B, H, Hkv, N, C, m):
    """k = C: every decided chunk is kept whole, so the layer is exact causal softmax attention (torch SDPA)."""
    rng = np.random.default_rng(7)
    q, k, v, wq, wk = _problem(rng, B, H, Hkv, N, 8, 6)
    out = oracle_mod.prefill(oracle_mod.Dims(B, H, Hkv, N, 8, 6, m * C, C, C), q, k, v, wq, wk)
    G = H // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(np.repeat(k, G, axis=1)), torch.from_numpy(np.repeat(v, G, axis=1)),
        is_causal=True).numpy()
    np.testing.assert_allclose(out["o"], ref, rtol=1e-10, atol=1e-12)


def test_no_window_is_linear_attention_closed_form(oracle_mod):
    """w = 0, k = 0, W = 0: <phi(q),phi(k)> = ||q|| ||k||, so o_i = sum_{j<=i} ||k_j|| v_j / sum_{j<=i} ||k_j||."""
    rng = np.random.default_rng(8)
    B, H, Hkv, N, d, D = 1, 2, 1, 45, 8, 6
    q, k, v, _, _ = _problem(rng, B, H, Hkv, N, d, D)
    out = oracle_mod.prefill(oracle_mod.Dims(B, H, Hkv, N, d, D, 0, 8, 0), q, k, v,
                             np.zeros((H, d, D)), np.zeros((Hkv, d, D)))
    nk = np.linalg.norm(k[0, 0], axis=1)
    want = np.cumsum(nk[:, None] * v[0, 0], axis=0) / np.cumsum(nk)[:, None]
    for h in range(H):
        np.testing.assert_allclose(out["o"][0, h], want, rtol=1e-12)


@pytest.mark.parametrize("m", [1, 2])
def test_window_plus_linear_closed_form(oracle_mod, m):
    """k = 0, w = mC, W = 0: <phi(q_i), phi(k_j)> = ||q_i|| ||k_j||, so row i of query chunk t mixes the
    window [(t-m)C, i] under exp(tau q.k) with every earlier token under ||q_i|| ||k_j|| weights, one
    normaliser for both (chunk-SWA plus linear attention, written out with plain ranges)."""
    rng = np.random.default_rng(12)
    B, H, Hkv, N, d, D, C = 1, 2, 1, 70, 8, 5, 8
    q, k, v, _, _ = _problem(rng, B, H, Hkv, N, d, D, spread=0.7)
    out = oracle_mod.prefill(oracle_mod.Dims(B, H, Hkv, N, d, D, m * C, C, 0), q, k, v,
                             np.zeros((H, d, D)), np.zeros((Hkv, d, D)))
    tau = 1 / math.sqrt(d)
    nk = np.linalg.norm(k[0, 0], axis=1)
    for h in range(H):
        for i in range(N):
            lo = max(0, (i // C - m) * C)
            e = np.exp(tau * (k[0, 0, lo:i + 1] @ q[0, h, i]))
            wl = np.linalg.norm(q[0, h, i]) * nk[:lo]
            want = (e @ v[0, 0, lo:i + 1] + wl @ v[0, 0, :lo]) / (e.sum() + wl.sum())
            np.testing.assert_allclose(out["o"][0, h, i], want, rtol=1e-11, atol=1e-13)


def test_no_window_equals_recurrence(oracle_mod):
    """w = 0, k = 0: the layer equals the token-by-token linear recurrence S_i = S_{i-1} + phi(k_i) v_i^T."""
    rng = np.random.default_rng(9)
    B, H, Hkv, N, d, D = 1, 2, 2, 41, 8, 6
    q, k, v, wq, wk = _problem(rng, B, H, Hkv, N, d, D)
    out = oracle_mod.prefill(oracle_mod.Dims(B, H, Hkv, N, d, D, 0, 8, 0), q, k, v, wq, wk)
    for h in range(H):
        pq = oracle_mod.npmap(q[0, h], wq[h])
        pk = oracle_mod.npmap(k[0, h], wk[h])
        S = np.zeros((D, d))
        z = np.zeros(D)
        for i in range(N):
            S += np.outer(pk[i], v[0, h, i])
            z += pk[i]
            np.testing.assert_allclose(out["o"][0, h, i], (pq[i] @ S) / (pq[i] @ z), rtol=1e-11)


@pytest.mark.parametrize("m,kk", [(1, 0), (1, 3), (2, 3), (1, 8)])
def test_zero_query_routing_sets(oracle_mod, m, kk):
    """q = 0: logits are 0 and phi(q) = 0, so o_i is the plain mean of v over Soft(i); the scores are
    ln(n/(n-1)), so each chunk keeps its first k tokens.  Soft(i) = window [(t-m)C, i] plus the first k
    tokens of every chunk c <= t-m-1 (chunk-granular delay)."""
    rng = np.random.default_rng(10)
    C, N, d = 8, 61, 8
    k = _rand(rng, 1, 1, N, d)
    v = _rand(rng, 1, 1, N, d)
    q = np.zeros((1, 1, N, d))
    out = oracle_mod.prefill(oracle_mod.Dims(1, 1, 1, N, d, 4, m * C, C, kk), q, k, v,
                             _rand(rng, 1, d, 4), _rand(rng, 1, d, 4))
    for i in range(N):
        t = i // C
        soft = set(range(max(0, (t - m) * C), i + 1))
        for c in range(0, t - m):
            soft |= set(range(c * C, c * C + kk))
        want = v[0, 0, sorted(soft)].mean(0)
        np.testing.assert_allclose(out["o"][0, 0, i], want, rtol=1e-12, atol=1e-14)


def test_linear_state_closed_form(oracle_mod):
    """W = 0: phi(k) = ||k|| 1/sqrt(D), so S_t = 1/sqrt(D) * sum over unkept decided tokens of ||k_j|| v_j."""
    rng = np.random.default_rng(11)
    C, N, d, D, kk, m = 8, 48, 8, 5, 3, 1
    q, k, v, _, _ = _problem(rng, 1, 1, 1, N, d, D)
    dims = oracle_mod.Dims(1, 1, 1, N, d, D, m * C, C, kk)
    idx = oracle_mod.prefill(dims, q, k, v, np.zeros((1, d, D)), np.zeros((1, d, D)))["idx"]
    for t in range(N // C + 1):
        S, z = oracle_mod.linear_state(dims, k, v, np.zeros((1, d, D)), idx, 0, 0, t)
        lin = [j for c in range(0, min(t - m, N // C)) for j in range(c * C, (c + 1) * C) if j not in idx[0, 0, c]]
        nk = np.linalg.norm(k[0, 0, lin], axis=1) if lin else np.zeros(0)
        wantS = np.outer(np.ones(D), (nk[:, None] * v[0, 0, lin]).sum(0)) / math.sqrt(D)
        np.testing.assert_allclose(S, wantS, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(z, np.full(D, nk.sum() / math.sqrt(D)), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("B,H,Hkv,N,d,D,w,C,kk", [
    (1, 2, 1, 24, 4, 3, 4, 4, 1),
    (2, 4, 2, 29, 8, 5, 8, 4, 2),    # GQA, ragged tail, m = 2
    (1, 1, 1, 33, 6, 4, 8, 8, 8),    # k = C
    (1, 2, 2, 20, 4, 4, 0, 4, 0),    # no window: pure linear
    (1, 3, 1, 40, 4, 6, 8, 8, 0),    # k = 0: chunked SWA + linear
    (1, 2, 1, 6, 4, 3, 8, 8, 2),     # N < C
])
def test_brute_force_agrees(oracle_mod, B, H, Hkv, N, d, D, w, C, kk):
    rng = np.random.default_rng(12)
    q, k, v, wq, wk = _problem(rng, B, H, Hkv, N, d, D)
    out = oracle_mod.prefill(oracle_mod.Dims(B, H, Hkv, N, d, D, w, C, kk), q, k, v, wq, wk)
    o, r, sel = brute.layer(q, k, v, wq, wk, w, C, kk)
    np.testing.assert_allclose(out["o"], o, rtol=1e-11, atol=1e-13)
    if w > 0:
        np.testing.assert_allclose(out["r"], r, rtol=1e-11, atol=1e-14)
    for (b, g, c), lst in sel.items():
        assert list(out["idx"][b, g, c]) == lst


def test_injected_selection(oracle_mod):
    rng = np.random.default_rng(13)
    B, H, Hkv, N, d, D, w, C, kk = 1, 2, 1, 32, 4, 3, 8, 8, 3
    q, k, v, wq, wk = _problem(rng, B, H, Hkv, N, d, D)
    idx = np.stack([np.sort(rng.choice(np.arange(c * C, (c + 1) * C), kk, replace=False)) for c in range(N // C)])
    idx = idx[None, None]
    out = oracle_mod.prefill(oracle_mod.Dims(B, H, Hkv, N, d, D, w, C, kk), q, k, v, wq, wk, idx_in=idx)
    o, _, _ = brute.layer(q, k, v, wq, wk, w, C, kk, idx_in=idx)
    np.testing.assert_allclose(out["o"], o, rtol=1e-11)


def test_rows_subset(oracle_mod):
    rng = np.random.default_rng(14)
    dims = oracle_mod.Dims(2, 4, 2, 40, 8, 5, 8, 8, 2)
    q, k, v, wq, wk = _problem(rng, 2, 4, 2, 40, 8, 5)
    full = oracle_mod.prefill(dims, q, k, v, wq, wk)["o"]
    rows = np.array([[0, 0, 0], [1, 3, 39], [0, 2, 17], [1, 1, 8]])
    part = oracle_mod.prefill(dims, q, k, v, wq, wk, rows=rows)["o"]
    for b, h, i in rows:
        np.testing.assert_array_equal(part[b, h, i], full[b, h, i])


def test_given_key_features_change_nothing(oracle_mod):
    """prefill with phi(k) supplied (from the oracle's own npmap, per KV head with its Wk) gives the
    same outputs, bit for bit, as prefill computing phi(k) itself -- whole layer and a row subset."""
    rng = np.random.default_rng(16)
    dims = oracle_mod.Dims(2, 4, 2, 40, 8, 5, 8, 8, 2)
    q, k, v, wq, wk = _problem(rng, 2, 4, 2, 40, 8, 5)
    phik = np.stack([np.stack([oracle_mod.npmap(k[b, g], wk[g]) for g in range(2)]) for b in range(2)])
    ref = oracle_mod.prefill(dims, q, k, v, wq, wk)
    got = oracle_mod.prefill(dims, q, k, v, wq, None, phik=phik)
    np.testing.assert_array_equal(got["o"], ref["o"])
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    rows = np.array([[0, 0, 0], [1, 3, 39], [0, 2, 17]])
    part = oracle_mod.prefill(dims, q, k, v, wq, None, idx_in=ref["idx"], rows=rows, phik=phik)["o"]
    for b, h, i in rows:
        np.testing.assert_array_equal(part[b, h, i], ref["o"][b, h, i])
    with pytest.raises(ValueError):
        oracle_mod.prefill(dims, q, k, v, wq, None, phik=phik[:, :1])


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("w,C,kk,Hkv", [(8, 8, 2, 1), (16, 8, 3, 2), (0, 8, 0, 1), (8, 8, 8, 1), (8, 8, 0, 2)])
def test_decode_state_machine_equals_prefill(oracle_mod, w, C, kk, Hkv):
    """Feeding tokens one at a time through the chunk-delayed state machine gives the prefill's rows."""
    rng = np.random.default_rng(15)
    B, H, N, d, D = 2, 2 * Hkv, 53, 8, 5
    q, k, v, wq, wk = _problem(rng, B, H, Hkv, N, d, D)
    dims = oracle_mod.Dims(B, H, Hkv, N, d, D, w, C, kk)
    full = oracle_mod.prefill(dims, q, k, v, wq, wk)
    dec = oracle_mod.Decoder(dims, wq, wk)
    for p in range(N):
        o, r = dec.step(q[:, :, p], k[:, :, p], v[:, :, p])
        np.testing.assert_allclose(o, full["o"][:, :, p], rtol=1e-11, atol=1e-13)
        if w > 0:
            np.testing.assert_allclose(r, full["r"][:, :, p], rtol=1e-12, atol=1e-14)
    assert dec.pos == N
