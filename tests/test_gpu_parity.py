"""GPU parity: every step of the CUDA path, called through the C ABI, against the fp64 oracle on
the same seeded inputs (sizes the oracle finishes in seconds, several tiles, ragged tails)."""
import numpy as np
import pytest
import torch

from linear_attention_still_b200.synth import WORKLOADS, Shape, make_inputs

pytestmark = pytest.mark.gpu

from tests._gpu import (OUT_TOL, SCORE_TOL, check_selection, dev, gpu_prefill, odims, row_rel_err,  # noqa: E402
                        score_err)

CASES = {
    "f32_b1_h2_n512": WORKLOADS["still_f32_b1_h2_n512"],
    "bf16_gqa_ragged": Shape(B=2, H=8, Hkv=2, N=1000, d=64, D=64, w=128, C=128, k=16),
    "bf16_d128_two_chunk_window": Shape(B=1, H=4, Hkv=1, N=1300, d=128, D=128, w=256, C=128, k=32),
    "bf16_keep_all": Shape(B=1, H=4, Hkv=2, N=700, d=64, D=64, w=128, C=128, k=128),
    "bf16_keep_none": Shape(B=1, H=4, Hkv=2, N=700, d=64, D=64, w=128, C=128, k=0),
    "f32_no_window": Shape(B=1, H=2, Hkv=1, N=300, d=64, D=32, w=0, C=64, k=0, dtype="f32"),
    "bf16_no_window": Shape(B=2, H=4, Hkv=2, N=333, d=64, D=64, w=0, C=128, k=0),
    # w = 0 on the tensor-core path with chunks of four query tiles, D = 128, groups of 4, ragged tail
    "bf16_no_window_c512_D128": Shape(B=1, H=8, Hkv=2, N=1300, d=64, D=128, w=0, C=512, k=0),
    "f32_shorter_than_chunk": Shape(B=1, H=2, Hkv=2, N=50, d=64, D=64, w=64, C=64, k=8, dtype="f32"),
    "bf16_one_token": Shape(B=1, H=4, Hkv=1, N=1, d=64, D=64, w=128, C=128, k=8),
    "f32_gqa_d128_D64": Shape(B=1, H=4, Hkv=2, N=520, d=128, D=64, w=128, C=64, k=8, dtype="f32"),
    "bf16_d128_g8": Shape(B=1, H=16, Hkv=2, N=1100, d=128, D=128, w=256, C=256, k=40),
    # largest head dim, feature width and group the library takes (SIMT path)
    "f32_max_d_D_group": Shape(B=1, H=32, Hkv=1, N=200, d=256, D=256, w=64, C=64, k=8, dtype="f32"),
    "bf16_max_d_D": Shape(B=1, H=4, Hkv=2, N=260, d=256, D=256, w=128, C=64, k=16),
    # a window covering the whole sequence with k = 0: exact causal softmax attention in the window
    # phase alone (the flash-style dense comparator `bench.py --keep window` times)
    "bf16_window_covers_sequence": Shape(B=1, H=4, Hkv=2, N=700, d=64, D=64, w=768, C=128, k=0),
    "bf16_d128_window_covers_sequence": Shape(B=1, H=4, Hkv=1, N=600, d=128, D=128, w=640, C=128, k=0),
}


@pytest.fixture(scope="module")
def lib():
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    assert torch.cuda.is_available()
    return still


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_parity(lib, oracle_mod, name):
    shape = CASES[name]
    inp = make_inputs(shape)
    out = gpu_prefill(shape, inp)
    assert out["status"] == 0
    d = odims(shape)
    if shape.w > 0:
        _, ora_r = oracle_mod.saliency(d, inp.q, inp.k)
        assert score_err(out["r"], ora_r) <= SCORE_TOL if shape.k > 0 else True
        if shape.k > 0 and shape.T > 0:
            ora_idx = oracle_mod.topk(d, ora_r)
            check_selection(shape, shape.N, out["idx"], out["r"], ora_r, ora_idx)
    ref = oracle_mod.prefill(d, inp.q, inp.k, inp.v, inp.wq, inp.wk,
                             idx_in=out["idx"] if shape.k > 0 and shape.T > 0 else None)["o"]
    err = row_rel_err(out["o"], ref)
    assert err <= OUT_TOL[shape.dtype], err


@pytest.mark.parametrize("name", ["f32_b1_h2_n512", "bf16_gqa_ragged", "bf16_d128_g8"])
def test_saliency_entry_point(lib, oracle_mod, name):
    shape = CASES[name]
    inp = make_inputs(shape)
    d = lib.dims_of(shape)
    r = torch.empty(shape.B, shape.Hkv, shape.N, device="cuda")
    rq = torch.empty(shape.B, shape.H, shape.N, device="cuda")
    lib.still_saliency(d, dev(inp.q, shape), dev(inp.k, shape), r, rq)
    assert lib.still_get_device_status() == 0
    sig, ora_r = oracle_mod.saliency(odims(shape), inp.q, inp.k)
    assert score_err(r.cpu().numpy(), ora_r) <= SCORE_TOL
    assert score_err(rq.cpu().numpy(), sig) <= SCORE_TOL
    assert np.isposinf(r.cpu().numpy()[:, :, 0]).all()


def test_topk_bit_exact_with_ties(lib, oracle_mod):
    rng = np.random.default_rng(3)
    shape = Shape(B=2, H=6, Hkv=3, N=5 * 96 + 17, d=64, D=64, w=96, C=96, k=11, dtype="f32")
    r = rng.integers(0, 9, size=(shape.B, shape.Hkv, shape.N)).astype(np.float32) * np.float32(0.25)
    r[0, 0, 5] = np.inf
    r[1, 2, 96:110] = np.inf
    r[0, 1, 200:230] = -1.0
    r[1, 0, 300] = -np.inf
    r_dev = torch.from_numpy(r).cuda()
    idx = torch.full((shape.B, shape.Hkv, shape.T, shape.k), -1, dtype=torch.int32, device="cuda")
    lib.still_select_topk(lib.dims_of(shape), r_dev, idx)
    want = oracle_mod.topk(odims(shape), r.astype(np.float64))
    np.testing.assert_array_equal(idx.cpu().numpy(), want)


@pytest.mark.parametrize("dtype,d,D", [("f32", 64, 64), ("bf16", 64, 64), ("bf16", 128, 128), ("f32", 128, 32)])
def test_npmap_entry_point(lib, oracle_mod, dtype, d, D):
    shape = Shape(B=2, H=3, Hkv=3, N=77, d=d, D=D, w=64, C=64, k=4, dtype=dtype)
    inp = make_inputs(shape)
    phi = torch.empty(shape.B, shape.H, shape.N, D, device="cuda")
    lib.still_npmap(shape.B, shape.H, shape.N, d, D, dtype, dev(inp.q, shape), dev(inp.wq, shape), phi)
    assert lib.still_get_device_status() == 0
    got = phi.cpu().numpy()
    for b in range(shape.B):
        for h in range(shape.H):
            ref = oracle_mod.npmap(inp.q[b, h], inp.wq[h])
            assert row_rel_err(got[b, h], ref) <= 1e-5


# The linear state is an intermediate: fp32 features on the SIMT path; on the bf16 tensor-core path
# phi(k) enters the Phi^T V product rounded to bf16 (relative 2^-9 per element).
STATE_TOL = {"f32": 1e-4, "bf16": 5e-3}


@pytest.mark.parametrize("name", ["bf16_gqa_ragged", "bf16_d128_two_chunk_window", "f32_gqa_d128_D64",
                                  "bf16_d128_g8"])
def test_linear_state_parity(lib, oracle_mod, name):
    shape = CASES[name]
    inp = make_inputs(shape)
    out = gpu_prefill(shape, inp)
    d = odims(shape)
    T = shape.T
    for b, g, t in {(0, 0, 0), (0, shape.Hkv - 1, min(2, T)), (shape.B - 1, 0, min(3, T)),
                    (shape.B - 1, shape.Hkv - 1, T)}:
        S, z = oracle_mod.linear_state(d, inp.k, inp.v, inp.wk, out["idx"], b, g, t)
        gs, gz = out["S"][b, g, t], out["z"][b, g, t]
        tol = STATE_TOL[shape.dtype]
        if np.abs(S).max() == 0:
            assert np.abs(gs).max() == 0 and np.abs(gz).max() == 0
            continue
        assert np.abs(gs - S).max() / np.abs(S).max() <= tol, (b, g, t)
        assert np.abs(gz - z).max() / np.abs(z).max() <= tol, (b, g, t)


def test_injected_selection(lib, oracle_mod):
    shape = CASES["bf16_gqa_ragged"]
    inp = make_inputs(shape)
    rng = np.random.default_rng(9)
    T = shape.T
    idx = np.empty((shape.B, shape.Hkv, T, shape.k), dtype=np.int32)
    for b in range(shape.B):
        for g in range(shape.Hkv):
            for c in range(T):
                idx[b, g, c] = np.sort(rng.choice(np.arange(c * shape.C, (c + 1) * shape.C), shape.k, replace=False))
    out = gpu_prefill(shape, inp, idx_in=idx)
    assert out["status"] == 0
    ref = oracle_mod.prefill(odims(shape), inp.q, inp.k, inp.v, inp.wq, inp.wk, idx_in=idx)["o"]
    assert row_rel_err(out["o"], ref) <= OUT_TOL["bf16"]


def test_injected_index_outside_chunk_is_reported(lib):
    shape = CASES["bf16_gqa_ragged"]
    inp = make_inputs(shape)
    idx = np.tile(np.arange(shape.k, dtype=np.int32), (shape.B, shape.Hkv, shape.T, 1))
    idx += (np.arange(shape.T, dtype=np.int32) * shape.C)[None, None, :, None]
    idx[1, 1, 2, 3] = 5  # belongs to chunk 0, not chunk 2
    out = gpu_prefill(shape, inp, idx_in=idx)
    assert out["status"] == 5  # STILL_ERR_DEVICE_CHECK
    assert lib.still_get_device_status() == 0  # cleared by the read


def test_empty_inputs_are_noops(lib):
    shape = Shape(B=1, H=2, Hkv=1, N=0, d=64, D=64, w=64, C=64, k=4)
    d = lib.dims_of(shape)
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    n0 = lib.still_launch_count()
    lib.still_hybrid_prefill(d, x, x, x, x, x, x, workspace=torch.zeros(256, dtype=torch.uint8, device="cuda"))
    assert lib.still_launch_count() == n0
    assert lib.still_get_device_status() == 0


@pytest.mark.parametrize("name", ["f32_b1_h2_n512", "bf16_gqa_ragged", "bf16_d128_g8", "bf16_no_window"])
def test_diagonal_score_entry_point(lib, oracle_mod, name):
    """Diagonal-only router score against the oracle's definition."""
    shape = CASES[name]
    inp = make_inputs(shape)
    r = torch.empty(shape.B, shape.Hkv, shape.N, device="cuda")
    lib.still_diagonal_score(lib.dims_of(shape), dev(inp.q, shape), dev(inp.k, shape), r)
    assert lib.still_get_device_status() == 0
    assert score_err(r.cpu().numpy(), oracle_mod.diagonal_score(odims(shape), inp.q, inp.k)) <= SCORE_TOL


@pytest.mark.parametrize("name", ["bf16_gqa_ragged", "bf16_d128_two_chunk_window"])
def test_diagonal_router_layer(lib, oracle_mod, name):
    """The layer with the diagonal-only router: GPU score -> GPU per-chunk top-k -> prefill with that
    selection, against the oracle's score, selection and layer output on the GPU's selection."""
    shape = CASES[name]
    inp = make_inputs(shape)
    d = lib.dims_of(shape)
    r = torch.empty(shape.B, shape.Hkv, shape.N, device="cuda")
    lib.still_diagonal_score(d, dev(inp.q, shape), dev(inp.k, shape), r)
    idx = torch.full((shape.B, shape.Hkv, shape.T, shape.k), -1, dtype=torch.int32, device="cuda")
    lib.still_select_topk(d, r, idx)
    od = odims(shape)
    ora_r = oracle_mod.diagonal_score(od, inp.q, inp.k)
    gr, gidx = r.cpu().numpy(), idx.cpu().numpy()
    assert score_err(gr, ora_r) <= SCORE_TOL
    check_selection(shape, shape.N, gidx, gr, ora_r, oracle_mod.topk(od, ora_r))
    out = gpu_prefill(shape, inp, idx_in=gidx)
    assert out["status"] == 0
    ref = oracle_mod.prefill(od, inp.q, inp.k, inp.v, inp.wq, inp.wk, idx_in=gidx)["o"]
    assert row_rel_err(out["o"], ref) <= OUT_TOL[shape.dtype]


# Logits that grow (or shrink) by tens of binary orders along the keys: later window tiles (ramp up) or
# the kept prefix after the window part (ramp down) exceed each row's reference maximum by far more than
# the lazy-rescale threshold, so the online softmax moves its reference in mid-row, O and the sums are
# rescaled, and tiles whose probabilities overflow the threshold are recomputed.
LARGE_LOGIT_CASES = {
    "bf16_d64_ramp_up": (Shape(B=1, H=4, Hkv=2, N=1500, d=64, D=64, w=256, C=256, k=128), "up"),
    "bf16_d64_ramp_down": (Shape(B=1, H=4, Hkv=2, N=1500, d=64, D=64, w=256, C=256, k=128), "down"),
    "bf16_d128_ramp_up": (Shape(B=1, H=4, Hkv=1, N=1500, d=128, D=128, w=256, C=256, k=128), "up"),
    "bf16_d128_ramp_down": (Shape(B=1, H=4, Hkv=1, N=1500, d=128, D=128, w=256, C=256, k=128), "down"),
}


@pytest.mark.parametrize("name", list(LARGE_LOGIT_CASES))
def test_prefill_parity_large_logits(lib, oracle_mod, name):
    from linear_attention_still_b200.synth import round_to_bf16_
    shape, ramp = LARGE_LOGIT_CASES[name]
    inp = make_inputs(shape)
    pos = np.arange(shape.N, dtype=np.float32) / shape.N
    f = 1.0 + 5.0 * pos if ramp == "up" else 6.0 - 5.0 * pos
    inp.k *= f[None, None, :, None]
    inp.q *= np.float32(3.0)
    round_to_bf16_(inp.k)
    round_to_bf16_(inp.q)
    out = gpu_prefill(shape, inp)
    assert out["status"] == 0
    d = odims(shape)
    _, ora_r = oracle_mod.saliency(d, inp.q, inp.k)
    assert score_err(out["r"], ora_r) <= SCORE_TOL
    check_selection(shape, shape.N, out["idx"], out["r"], ora_r, oracle_mod.topk(d, ora_r))
    ref = oracle_mod.prefill(d, inp.q, inp.k, inp.v, inp.wq, inp.wk, idx_in=out["idx"])["o"]
    err = row_rel_err(out["o"], ref)
    assert err <= OUT_TOL[shape.dtype], err
