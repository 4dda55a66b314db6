"""GPU parity of the chunk-granular delayed decode: prefill(N0) -> T decode steps reproduces rows
N0..N0+T-1 of the oracle's prefill of N0+T tokens, including the steps that close a chunk."""
import numpy as np
import pytest
import torch

from linear_attention_still_b200.synth import WORKLOADS, Shape, make_inputs

pytestmark = pytest.mark.gpu

from tests._gpu import OUT_TOL, dev, gpu_prefill, odims, row_rel_err  # noqa: E402

CASES = {
    # name: (shape with N = prefill length, decode steps)
    "f32_b1_h2": (WORKLOADS["still_f32_b1_h2_n512"].replace(N=300), 100),
    "bf16_gqa": (Shape(B=2, H=8, Hkv=2, N=520, d=64, D=64, w=128, C=128, k=16), 260),
    "bf16_d128_two_chunk_window": (Shape(B=1, H=4, Hkv=1, N=390, d=128, D=128, w=256, C=128, k=24), 140),
    "f32_no_window": (Shape(B=1, H=2, Hkv=1, N=100, d=64, D=32, w=0, C=64, k=0, dtype="f32"), 60),
    "bf16_keep_none": (Shape(B=1, H=4, Hkv=2, N=250, d=64, D=64, w=128, C=128, k=0), 20),
    "bf16_from_empty": (Shape(B=1, H=4, Hkv=2, N=0, d=64, D=64, w=128, C=128, k=16), 300),
    # one case per instantiation of the split-K attention kernels (tensor-core bf16, packed SIMT
    # fp32), plus the general-group fallback
    "f32_d128_g8": (Shape(B=1, H=8, Hkv=1, N=300, d=128, D=64, w=128, C=64, k=8, dtype="f32"), 100),
    "bf16_d128_mha": (Shape(B=2, H=2, Hkv=2, N=260, d=128, D=128, w=128, C=128, k=16), 140),
    "bf16_d128_g2": (Shape(B=1, H=4, Hkv=2, N=200, d=128, D=128, w=128, C=64, k=12), 80),
    "f32_d64_mha": (Shape(B=1, H=2, Hkv=2, N=200, d=64, D=64, w=64, C=64, k=8, dtype="f32"), 80),
    "bf16_d64_g8": (Shape(B=1, H=16, Hkv=2, N=200, d=64, D=64, w=128, C=64, k=8), 80),
    "bf16_d128_g8": (Shape(B=1, H=8, Hkv=1, N=300, d=128, D=64, w=128, C=64, k=8), 100),
    "bf16_d64_mha": (Shape(B=2, H=2, Hkv=2, N=200, d=64, D=64, w=64, C=64, k=8), 80),
    "f32_g8_D256": (Shape(B=1, H=8, Hkv=1, N=150, d=64, D=256, w=64, C=64, k=8, dtype="f32"), 60),
    "bf16_no_window": (Shape(B=1, H=4, Hkv=2, N=100, d=64, D=64, w=0, C=64, k=0), 60),
    # w = 0 prefill on the tensor-core path (C a multiple of 128), then decode across a chunk boundary
    "bf16_no_window_tc": (Shape(B=1, H=4, Hkv=2, N=300, d=64, D=64, w=0, C=128, k=0), 100),
    "bf16_g16_fallback": (Shape(B=1, H=16, Hkv=1, N=200, d=64, D=64, w=64, C=64, k=8), 80),
    "f32_d96_fallback": (Shape(B=1, H=4, Hkv=2, N=150, d=96, D=64, w=64, C=64, k=8, dtype="f32"), 60),
}


@pytest.fixture(scope="module")
def lib():
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    return still


def run_decode(lib, shape, T, inp):
    N0 = shape.N
    cap = N0 + T
    d = lib.dims_of(shape, N=N0)
    state = torch.zeros(lib.still_decode_state_bytes(d, cap), dtype=torch.uint8, device="cuda")
    lib.still_decode_init(d, cap, state)
    if N0 > 0:
        out = gpu_prefill(shape, inp, N=N0, state=state, capacity=cap)
        assert out["status"] == 0
    q, k, v = (dev(getattr(inp, n), shape) for n in ("q", "k", "v"))
    wq, wk = dev(inp.wq, shape), dev(inp.wk, shape)
    outs = []
    o_t = torch.empty(shape.B, shape.H, shape.d, dtype=q.dtype, device="cuda")
    for p in range(N0, cap):
        lib.still_decode_step(d, state, cap, p, wq, wk, q[:, :, p].contiguous(), k[:, :, p].contiguous(),
                              v[:, :, p].contiguous(), o_t)
        outs.append(o_t.float().cpu().numpy().copy())
    assert lib.still_get_device_status() == 0
    return np.stack(outs, axis=2), state  # [B,H,T,d]


@pytest.mark.parametrize("name", list(CASES))
def test_decode_matches_prefill_rows(lib, oracle_mod, name):
    shape, T = CASES[name]
    full = shape.replace(N=shape.N + T)
    inp = make_inputs(shape.replace(decode_steps=T))
    got, _ = run_decode(lib, shape, T, inp)
    gp = gpu_prefill(full, inp)
    idx = gp["idx"] if full.k > 0 and full.T > 0 else None
    ref = oracle_mod.prefill(odims(full), inp.q, inp.k, inp.v, inp.wq, inp.wk, idx_in=idx)["o"]
    tol = OUT_TOL[shape.dtype]
    assert row_rel_err(got, ref[:, :, shape.N:]) <= tol
    assert row_rel_err(got, gp["o"][:, :, shape.N:]) <= tol


def test_decode_from_empty_matches_oracle_state_machine(lib, oracle_mod):
    shape, T = Shape(B=1, H=2, Hkv=1, N=0, d=64, D=64, w=64, C=64, k=8, dtype="f32"), 200
    inp = make_inputs(shape.replace(decode_steps=T))
    got, _ = run_decode(lib, shape, T, inp)
    dec = oracle_mod.Decoder(odims(shape.replace(N=T)), inp.wq, inp.wk)
    for p in range(T):
        o, _ = dec.step(inp.q[:, :, p], inp.k[:, :, p], inp.v[:, :, p])
        assert row_rel_err(got[:, :, p], o) <= OUT_TOL["f32"], p


def test_decode_position_mismatch_is_reported(lib):
    shape = Shape(B=1, H=2, Hkv=1, N=0, d=64, D=64, w=64, C=64, k=8)
    d = lib.dims_of(shape)
    cap = 64
    state = torch.zeros(lib.still_decode_state_bytes(d, cap), dtype=torch.uint8, device="cuda")
    lib.still_decode_init(d, cap, state)
    x = torch.zeros(shape.B, shape.H, shape.d, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(shape.B, shape.Hkv, shape.d, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(shape.H, shape.d, shape.D, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(x)
    lib.still_decode_step(d, state, cap, 3, w, w[:1], x, kv, kv, o)  # state is at 0
    assert lib.still_get_device_status() == 5


def test_bf16_decode_scores_and_chunk_close_selection(lib, oracle_mod):
    """bf16 decode on the tensor-core path, checked directly rather than through its outputs: the group
    saliency score each decode step stores for its token (ring scores) against the oracle's
    (<= 1e-3), and the rows kept by the chunk closes that happen during decode against the top-k of
    the GPU's own scores (bit-exact) and the oracle's selection (differences only between oracle
    near-ties)."""
    from tests._gpu import SCORE_TOL, check_selection, score_err
    shape, T = CASES["bf16_gqa"]
    N0, C, k, m = shape.N, shape.C, shape.k, shape.w // shape.C
    cap = N0 + T
    full = shape.replace(N=cap)
    inp = make_inputs(shape.replace(decode_steps=T))
    d = lib.dims_of(shape, N=N0)
    L = lib.still_decode_state_layout(d, cap)
    state = torch.zeros(lib.still_decode_state_bytes(d, cap), dtype=torch.uint8, device="cuda")
    lib.still_decode_init(d, cap, state)
    out = gpu_prefill(shape, inp, N=N0, state=state, capacity=cap)
    assert out["status"] == 0
    BK = shape.B * shape.Hkv
    ring_r = state[L["ring_r"]: L["ring_r"] + BK * L["ring_rows"] * 4].view(torch.float32).view(BK, L["ring_rows"])

    def row(j):
        return ((j // C) % (m + 1)) * C + j % C

    r_gpu = np.full((shape.B, shape.Hkv, cap), np.nan)
    r_gpu[:, :, :N0] = out["r"]
    q, kk, v = (dev(getattr(inp, n), shape) for n in ("q", "k", "v"))
    wq, wk = dev(inp.wq, shape), dev(inp.wk, shape)
    o_t = torch.empty(shape.B, shape.H, shape.d, dtype=q.dtype, device="cuda")
    closes = []
    for p in range(N0, cap):
        lib.still_decode_step(d, state, cap, p, wq, wk, q[:, :, p].contiguous(), kk[:, :, p].contiguous(),
                              v[:, :, p].contiguous(), o_t)
        r_gpu[:, :, p] = ring_r[:, row(p)].cpu().numpy().reshape(shape.B, shape.Hkv)
        if p % C == C - 1 and p // C - m >= 0:
            closes.append(p // C - m)  # this step closed chunk t - m
    assert lib.still_get_device_status() == 0
    assert closes, "the case must close a chunk during decode"
    # scores of the decode tokens against the oracle's saliency of the whole sequence
    _, r_ora = oracle_mod.saliency(odims(full), inp.q, inp.k)
    assert score_err(r_gpu[:, :, N0:], r_ora[:, :, N0:]) <= SCORE_TOL
    # kept rows of the chunks closed during decode, mapped back to positions by their keys
    khat = state[L["khat"]: L["khat"] + BK * L["cap_chunks"] * k * shape.d * 2].view(torch.bfloat16)
    khat = khat.view(shape.B, shape.Hkv, L["cap_chunks"] * k, shape.d).float().cpu().numpy()
    kin = kk.float().cpu().numpy()
    for c in closes:
        lo = c * C
        got = np.zeros((shape.B, shape.Hkv, 1, k), dtype=np.int32)
        for b in range(shape.B):
            for g in range(shape.Hkv):
                for e in range(k):
                    hit = np.nonzero((kin[b, g, lo:lo + C] == khat[b, g, c * k + e]).all(axis=-1))[0]
                    assert hit.size == 1, (c, b, g, e)
                    got[b, g, 0, e] = lo + hit[0]
        sub = full.replace(N=C)  # one chunk: check_selection's top-k of this chunk's scores
        gpu_r = r_gpu[:, :, lo:lo + C]
        ora_r = r_ora[:, :, lo:lo + C]
        ora_idx = oracle_mod.topk(odims(sub), ora_r)
        check_selection(sub, C, got - lo, gpu_r, ora_r, ora_idx)
