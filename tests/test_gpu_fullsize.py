"""Full-size parity: the prefill at the efficiency workloads' sizes, in the launch configuration the
benchmark times, checked against the fp64 oracle on whole (batch, KV group) slices -- every score
of the slice, every chunk's selection, and sampled output rows covering the first, middle and last
chunks and the ragged tail.  Plus the chunk-delayed decode at a 64K context."""
import numpy as np
import pytest
import torch

from linear_attention_still_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

from tests._gpu import OUT_TOL, SCORE_TOL, check_selection, dev, gpu_prefill, odims, pick_rows, row_rel_err, \
    score_err  # noqa: E402


@pytest.fixture(scope="module")
def lib():
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    return still


def _slice(inp, shape, b, g):
    G = shape.G
    return (inp.q[b:b + 1, g * G:(g + 1) * G], inp.k[b:b + 1, g:g + 1], inp.v[b:b + 1, g:g + 1],
            inp.wq[g * G:(g + 1) * G], inp.wk[g:g + 1])


@pytest.mark.parametrize("name", ["llama32_1b_layer_n16k", "llama31_8b_layer_b4_n16k", "llama31_8b_layer_n64k"])
def test_full_size_prefill_sampled(lib, oracle_mod, name):
    shape = WORKLOADS[name]
    inp = make_inputs(shape)
    out = gpu_prefill(shape, inp)
    assert out["status"] == 0
    assert np.isfinite(out["o"]).all()
    sl = shape.replace(B=1, H=shape.G, Hkv=1)
    d = odims(sl)
    for b, g in [(0, 0), (shape.B - 1, shape.Hkv - 1)]:
        q, k, v, wq, wk = _slice(inp, shape, b, g)
        _, ora_r = oracle_mod.saliency(d, q, k)
        gr = out["r"][b:b + 1, g:g + 1]
        assert score_err(gr, ora_r) <= SCORE_TOL
        gidx = out["idx"][b:b + 1, g:g + 1]
        check_selection(sl, shape.N, gidx, gr, ora_r, oracle_mod.topk(d, ora_r))
        rows = pick_rows(sl, shape.N, 48, seed=b * 131 + g, b=0)
        ref = oracle_mod.prefill(d, q, k, v, wq, wk, idx_in=gidx, rows=rows)["o"]
        got = out["o"][b:b + 1, g * shape.G:(g + 1) * shape.G]
        err = row_rel_err(got[rows[:, 0], rows[:, 1], rows[:, 2]], ref[rows[:, 0], rows[:, 1], rows[:, 2]])
        assert err <= OUT_TOL[shape.dtype], (b, g, err)


def test_decode_at_64k_context(lib, oracle_mod):
    """One sequence of the 8B decode workload: 64K-token prefill into the state, then decode steps
    across a chunk boundary (the step that closes a chunk selects and folds chunk t-m)."""
    base = WORKLOADS["llama31_8b_decode_b16_ctx64k"]
    steps = 1030
    shape = base.replace(B=1, decode_steps=steps)
    N0 = shape.N
    inp = make_inputs(shape)
    cap = N0 + steps
    d = lib.dims_of(shape, N=N0)
    state = torch.zeros(lib.still_decode_state_bytes(d, cap), dtype=torch.uint8, device="cuda")
    lib.still_decode_init(d, cap, state)
    out = gpu_prefill(shape, inp, N=N0, state=state, capacity=cap)
    assert out["status"] == 0
    q, k, v = (dev(getattr(inp, n)[:, :, N0:], shape) for n in ("q", "k", "v"))
    wq, wk = dev(inp.wq, shape), dev(inp.wk, shape)
    check = {0, 1, 511, 1022, 1023, 1024, 1029}  # position N0+1023 closes chunk 64
    got = {}
    o_t = torch.empty(1, shape.H, shape.d, dtype=torch.bfloat16, device="cuda")
    for s_ in range(steps):
        lib.still_decode_step(d, state, cap, N0 + s_, wq, wk, q[:, :, s_].contiguous(), k[:, :, s_].contiguous(),
                              v[:, :, s_].contiguous(), o_t)
        if s_ in check:
            got[s_] = o_t.float().cpu().numpy()
    assert lib.still_get_device_status() == 0
    # oracle: rows N0+s of the prefill of N0+steps tokens, per KV group slice, with the GPU's selection
    full = shape.replace(N=cap, decode_steps=0)
    gp = gpu_prefill(full, inp)  # the GPU prefill of all tokens provides the selection to replay
    sl = full.replace(B=1, H=full.G, Hkv=1)
    dd = odims(sl)
    for g in [0, full.Hkv - 1]:
        qs, ks, vs, wqs, wks = _slice(inp, full, 0, g)
        rows = np.array([(0, h, N0 + s_) for s_ in sorted(check) for h in range(full.G)], dtype=np.int32)
        ref = oracle_mod.prefill(dd, qs, ks, vs, wqs, wks, idx_in=gp["idx"][:1, g:g + 1], rows=rows)["o"]
        for s_ in sorted(check):
            e = row_rel_err(got[s_][0, g * full.G:(g + 1) * full.G], ref[0, :, N0 + s_])
            assert e <= OUT_TOL["bf16"], (g, s_, e)
