"""The persistent head-dim-64 merge (merge_ring.cu) through the C ABI.

* Parity with the fp64 oracle when the grid is capped to a few CTAs, so that every CTA walks many
  work items: the TMEM slot ring, the tile/parity counters and the double-buffered query tiles then
  cross item boundaries (with the default grid, small problems give every CTA one item).
* The results do not depend on the grid: each work item runs the same arithmetic whichever CTA
  takes it, so outputs, scores and the selection are bit-identical across grid caps.
* A bounded wait that runs out: the test hook makes the first CTA load no key/value tile; the call
  reports STILL_ERR_TIMEOUT through the device status word, and the next normal call on the same
  context matches the oracle again."""
import numpy as np
import pytest
import torch

from linear_attention_still_b200.synth import Shape, make_inputs

pytestmark = pytest.mark.gpu

from tests._gpu import OUT_TOL, SCORE_TOL, check_selection, gpu_prefill, odims, row_rel_err, score_err  # noqa: E402

STILL_ERR_TIMEOUT = 6

CASES = {
    # two heads per CTA, D = 64, one-chunk window: every item type (diagonal, band, ragged kept tile)
    "pair_D64_m1": Shape(B=2, H=8, Hkv=2, N=1000, d=64, D=64, w=128, C=128, k=16),
    # one head per CTA (odd group), D = 128 (Y spans two ring slots), two-chunk window, ragged tail
    "single_D128_m2": Shape(B=1, H=6, Hkv=2, N=1100, d=64, D=128, w=256, C=128, k=24),
    # k = 0: prefix items have no key tile (the prologue's fold alone), window items still do
    "pair_keep_none": Shape(B=1, H=4, Hkv=1, N=777, d=64, D=64, w=256, C=256, k=0),
    # k = C: every token of a decided chunk is kept (exact causal softmax)
    "pair_keep_all": Shape(B=1, H=4, Hkv=2, N=650, d=64, D=128, w=128, C=128, k=128),
}


@pytest.fixture(scope="module")
def lib():
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    assert torch.cuda.is_available()
    yield still
    still.still_debug_merge(False, 0)


def _check_oracle(oracle_mod, shape, inp, out):
    d = odims(shape)
    _, ora_r = oracle_mod.saliency(d, inp.q, inp.k)
    if shape.k > 0:
        assert score_err(out["r"], ora_r) <= SCORE_TOL
        if shape.T > 0:
            check_selection(shape, shape.N, out["idx"], out["r"], ora_r, oracle_mod.topk(d, ora_r))
    ref = oracle_mod.prefill(d, inp.q, inp.k, inp.v, inp.wq, inp.wk,
                             idx_in=out["idx"] if shape.k > 0 and shape.T > 0 else None)["o"]
    err = row_rel_err(out["o"], ref)
    assert err <= OUT_TOL[shape.dtype], err


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("ctas", [1, 3])
def test_persistent_items_match_oracle(lib, oracle_mod, name, ctas):
    shape = CASES[name]
    inp = make_inputs(shape)
    lib.still_debug_merge(False, ctas)
    try:
        out = gpu_prefill(shape, inp)
    finally:
        lib.still_debug_merge(False, 0)
    assert out["status"] == 0
    _check_oracle(oracle_mod, shape, inp, out)


@pytest.mark.parametrize("name", ["pair_D64_m1", "single_D128_m2"])
def test_results_do_not_depend_on_the_grid(lib, name):
    shape = CASES[name]
    inp = make_inputs(shape)
    outs = []
    for ctas in (0, 1, 7):
        lib.still_debug_merge(False, ctas)
        try:
            outs.append(gpu_prefill(shape, inp))
        finally:
            lib.still_debug_merge(False, 0)
        assert outs[-1]["status"] == 0
    for o in outs[1:]:
        for key in ("o", "r", "idx"):
            np.testing.assert_array_equal(o[key], outs[0][key], err_msg=key)


def test_bounded_wait_runs_out_and_context_recovers(lib, oracle_mod):
    shape = CASES["pair_D64_m1"]
    inp = make_inputs(shape)
    lib.still_debug_merge(True, 1)
    try:
        stalled = gpu_prefill(shape, inp)
    finally:
        lib.still_debug_merge(False, 0)
    assert stalled["status"] == STILL_ERR_TIMEOUT
    assert lib.still_get_device_status() == 0  # the status word was read and cleared
    again = gpu_prefill(shape, inp)
    assert again["status"] == 0
    _check_oracle(oracle_mod, shape, inp, again)
