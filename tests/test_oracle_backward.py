"""Pins of the oracle's backward pass (oracle/backward.py) to central finite differences of the C
forward oracle, with the per-chunk selection held fixed; plus the NP-Map backward alone."""
import math

import numpy as np
import pytest

from oracle import backward


def _problem(rng, B, H, Hkv, N, d, D):
    q = rng.standard_normal((B, H, N, d)) * np.exp(rng.normal(0, 0.4, (B, H, N, 1)))
    k = rng.standard_normal((B, Hkv, N, d)) * np.exp(rng.normal(0, 0.4, (B, Hkv, N, 1)))
    v = rng.standard_normal((B, Hkv, N, d))
    wq = rng.standard_normal((H, d, D)) / math.sqrt(d)
    wk = rng.standard_normal((Hkv, d, D)) / math.sqrt(d)
    do = rng.standard_normal((B, H, N, d))
    return q, k, v, wq, wk, do


def _fd_check(oracle_mod, dims, args, idx, grads, eps=1e-5, tol=1e-6):
    names = ("q", "k", "v", "wq", "wk")
    q, k, v, wq, wk, do = args

    def loss(q_, k_, v_, wq_, wk_):
        o = oracle_mod.prefill(dims, q_, k_, v_, wq_, wk_, idx_in=idx, nthreads=1)["o"]
        return float(np.sum(o * do))

    base = [q, k, v, wq, wk]
    for a, (name, g) in enumerate(zip(names, grads)):
        x = base[a]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            ix = it.multi_index
            plus = [t.copy() for t in base]
            minus = [t.copy() for t in base]
            plus[a][ix] += eps
            minus[a][ix] -= eps
            fd[ix] = (loss(*plus) - loss(*minus)) / (2 * eps)
        err = np.abs(fd - g).max() / max(np.abs(fd).max(), 1e-12)
        assert err < tol, (name, err)


@pytest.mark.parametrize("w,C,kk,Hkv", [(4, 4, 2, 1), (8, 4, 1, 2), (0, 4, 0, 1), (4, 4, 4, 1)])
def test_backward_matches_finite_differences(oracle_mod, w, C, kk, Hkv):
    """Hybrid (window + kept + linear), a two-chunk window with GQA, pure linear (w = 0), and every
    token kept (k = C: causal softmax)."""
    rng = np.random.default_rng(31 + w + kk)
    B, H, N, d, D = 1, 2, 14, 3, 3
    args = _problem(rng, B, H, Hkv, N, d, D)
    dims = oracle_mod.Dims(B=B, H=H, Hkv=Hkv, N=N, d=d, D=D, w=w, C=C, k=kk)
    q, k, v, wq, wk, do = args
    idx = oracle_mod.prefill(dims, q, k, v, wq, wk)["idx"] if (w > 0 and kk > 0) else None
    grads = backward.layer_backward(q, k, v, wq, wk, do, idx, w, C)
    _fd_check(oracle_mod, dims, args, idx, grads)


def test_npmap_backward_matches_finite_differences():
    rng = np.random.default_rng(5)
    x, W, dphi = rng.standard_normal(5), rng.standard_normal((5, 4)), rng.standard_normal(4)
    dx, dW = backward.npmap_backward(x, W, dphi)
    eps = 1e-6
    for a in range(5):
        xp, xm = x.copy(), x.copy()
        xp[a] += eps
        xm[a] -= eps
        fd = (backward.npmap_forward(xp, W) - backward.npmap_forward(xm, W)) @ dphi / (2 * eps)
        assert abs(fd - dx[a]) < 1e-8 * max(1.0, abs(fd))
    for a in range(5):
        for c in range(4):
            Wp, Wm = W.copy(), W.copy()
            Wp[a, c] += eps
            Wm[a, c] -= eps
            fd = (backward.npmap_forward(x, Wp) - backward.npmap_forward(x, Wm)) @ dphi / (2 * eps)
            assert abs(fd - dW[a, c]) < 1e-8 * max(1.0, abs(fd))


def test_backward_golden():
    """Hand-derived gradient of one output row (tests/golden/backward_hand.json) of the six-token
    layer of tests/golden/merge_hand.json: dv = weight / Z, dk from e_j (v_j - o) / Z and the
    linear token's |q| (v_0 - o) / Z, dq in closed form, and dWq = dWk = 0 because a one-feature
    NP-Map is the norm."""
    import json
    import os
    here = os.path.join(os.path.dirname(__file__), "golden")
    with open(os.path.join(here, "backward_hand.json")) as f:
        gold = json.load(f)
    with open(os.path.join(here, "merge_hand.json")) as f:
        case = next(c for c in json.load(f)["cases"] if c["name"] == gold["case"])
    dm, x = case["dims"], case["inputs"]
    N, H = dm["N"], dm["H"]
    q = np.array(x["q"], dtype=np.float64).reshape(1, H, N, 1)
    k = np.array(x["k"], dtype=np.float64).reshape(1, 1, N, 1)
    v = np.array(x["v"], dtype=np.float64).reshape(1, 1, N, 1)
    wq = np.array(x["wq"], dtype=np.float64).reshape(H, 1, 1)
    wk = np.array(x["wk"], dtype=np.float64).reshape(1, 1, 1)
    idx = np.array(x["idx"], dtype=np.int32).reshape(1, 1, -1, 1)
    do = np.zeros_like(q)
    up = gold["upstream"]
    do[0, up["h"], up["i"], 0] = up["value"]
    dq, dk, dv, dwq, dwk = backward.layer_backward(q, k, v, wq, wk, do, idx, dm["w"], dm["C"], scale=dm["scale"])
    want_dq = np.zeros_like(q)
    want_dq[0, gold["dq"]["h"], gold["dq"]["i"], 0] = gold["dq"]["value"]
    np.testing.assert_allclose(dq, want_dq, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dk[0, 0, :, 0], gold["dk"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0, :, 0], gold["dv"], rtol=1e-12, atol=1e-14)
    assert np.all(dwq == 0.0) and np.all(dwk == 0.0)


def test_output_rounded_in_d_reaches_every_gradient_but_dv():
    """The backward form that takes D_i = <do_i, o_i> from the forward's stored bf16 output: on the
    seeded inputs of the GPU case tc_bf16_gqa_ragged, rounding o alone moves dq and dk by under 1e-2 of
    their largest entry and leaves dv exactly as it is (dv = P^T do does not involve D_i).  The GPU
    parity test of still_hybrid_backward_saved allows 2e-2 for the gradients D_i reaches."""
    import oracle
    from linear_attention_still_b200.synth import Shape, make_inputs, round_to_bf16
    shape = Shape(B=2, H=8, Hkv=2, N=700, d=64, D=64, w=128, C=128, k=16)
    inp = make_inputs(shape)
    do = round_to_bf16(np.random.default_rng(77).standard_normal(inp.q.shape).astype(np.float32))[0]
    idx = oracle.prefill(oracle.Dims.of(shape), inp.q, inp.k, inp.v, inp.wq, inp.wk)["idx"]
    exact = backward.layer_backward(inp.q, inp.k, inp.v, inp.wq, inp.wk, do, idx, shape.w, shape.C)
    rounded = backward.layer_backward(inp.q, inp.k, inp.v, inp.wq, inp.wk, do, idx, shape.w, shape.C,
                                      d_from_output="bf16")
    rel = [float(np.abs(a - b).max() / np.abs(b).max()) for a, b in zip(rounded, exact)]
    assert rel[2] == 0.0                                   # dv
    assert 0.0 < rel[0] < 1e-2 and 0.0 < rel[1] < 1e-2     # dq, dk
    assert rel[3] < 1e-2 and rel[4] < 1e-2                 # dWq, dWk
