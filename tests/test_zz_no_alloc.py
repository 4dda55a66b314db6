"""still_hybrid_prefill_static: the prefill for callers that cannot allocate device memory (for
example a serving loop that must keep its memory footprint fixed, or a host thread that may not
call cudaMalloc while other work is in flight).  Its scratch is a fixed array inside the library
instead of a caller workspace.

It runs the same kernels on the same inputs as still_hybrid_prefill, so its output, selection and
exported decode state must be bit-identical to the regular entry point's, on repeated calls and with
the scratch left dirty by earlier calls of other shapes; after one warm-up call, further calls must
leave the device's free memory and torch's allocator untouched; shapes whose scratch would not fit
are refused before any work.  (The file name puts it last in collection, after every other GPU
test; it also passes alone in a fresh process.)"""
import ctypes as ct
import os
import re

import numpy as np
import pytest

from linear_attention_still_b200.synth import WORKLOADS, Shape, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SHAPES = {
    "bf16_gqa_ragged": Shape(B=2, H=8, Hkv=2, N=1000, d=64, D=64, w=128, C=128, k=16),
    "bf16_d128_two_chunk_window": Shape(B=1, H=4, Hkv=1, N=1300, d=128, D=128, w=256, C=128, k=32),
    "f32_gqa_d128_D64": Shape(B=1, H=4, Hkv=2, N=520, d=128, D=64, w=128, C=64, k=8, dtype="f32"),
}


@pytest.fixture(scope="module")
def lib():
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    return still


def test_static_limit_matches_the_header(lib):
    text = open(os.path.join(ROOT, "include", "still.h")).read()
    m = re.search(r"#define\s+STILL_STATIC_WORKSPACE_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "STILL_STATIC_WORKSPACE_BYTES not found in include/still.h"
    assert int(m.group(1)) << int(m.group(2)) == lib.STATIC_WORKSPACE_BYTES


def test_static_prefill_refuses_shapes_beyond_its_scratch(lib):
    big = WORKLOADS["llama31_8b_layer_b4_n16k"]
    d = lib.dims_of(big)
    assert lib.still_prefill_workspace_bytes(d) > lib.STATIC_WORKSPACE_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes before any work
    f = lib._lib.still_hybrid_prefill_static
    assert f(ct.byref(d), fake, fake, fake, fake, fake, fake, None, None, 0, None) == 3  # STILL_ERR_WORKSPACE
    bad = lib.dims_of(big.replace(w=100))  # not a whole number of chunks: same error as the regular call
    assert f(ct.byref(bad), fake, fake, fake, fake, fake, fake, None, None, 0, None) == 1
    # argument errors come before the size refusal, as in the regular entry point
    assert f(ct.byref(d), None, fake, fake, fake, fake, fake, None, None, 0, None) == 1
    assert f(ct.byref(d), fake + 8, fake, fake, fake, fake, fake, None, None, 0, None) == 1
    assert f(ct.byref(d), fake, fake, fake, fake, fake, fake, None, fake, big.N - 1, None) == 1


def _upload(lib, shape):
    from tests._gpu import dev
    inp = make_inputs(shape)
    return [dev(getattr(inp, n), shape) for n in ("q", "k", "v", "wq", "wk")]


@pytest.mark.gpu
def test_static_prefill_matches_workspace_prefill(lib):
    import torch
    for name, shape in SHAPES.items():
        d = lib.dims_of(shape)
        assert lib.still_prefill_workspace_bytes(d) <= lib.STATIC_WORKSPACE_BYTES
        q, k, v, wq, wk = _upload(lib, shape)
        ws = torch.empty(lib.still_prefill_workspace_bytes(d), dtype=torch.uint8, device="cuda")
        ref = torch.full_like(q, float("nan"))
        lib.still_hybrid_prefill(d, q, k, v, wq, wk, ref, workspace=ws)
        assert lib.still_get_device_status() == 0
        want = ref.cpu()
        for call in range(2):  # two calls in a row on the same (dirty) scratch
            o = torch.full_like(q, float("nan"))
            lib.still_hybrid_prefill_static(d, q, k, v, wq, wk, o)
            assert lib.still_get_device_status() == 0
            assert torch.equal(o.cpu(), want), (name, call)


@pytest.mark.gpu
def test_static_prefill_exports_the_same_decode_state(lib):
    import torch
    shape = SHAPES["bf16_gqa_ragged"]
    d = lib.dims_of(shape)
    cap = shape.N + 64
    q, k, v, wq, wk = _upload(lib, shape)
    nbytes = lib.still_decode_state_bytes(d, cap)
    states = []
    for static in (False, True, True):
        st = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        lib.still_decode_init(d, cap, st)
        o = torch.empty_like(q)
        if static:
            lib.still_hybrid_prefill_static(d, q, k, v, wq, wk, o, state=st, state_capacity=cap)
        else:
            ws = torch.empty(lib.still_prefill_workspace_bytes(d), dtype=torch.uint8, device="cuda")
            lib.still_hybrid_prefill(d, q, k, v, wq, wk, o, workspace=ws, state=st, state_capacity=cap)
        assert lib.still_get_device_status() == 0
        states.append((st.cpu(), o.cpu()))
    for st, o in states[1:]:
        assert torch.equal(st, states[0][0])
        assert torch.equal(o, states[0][1])


@pytest.mark.gpu
def test_static_prefill_allocates_nothing_after_warm_up(lib):
    import torch
    shape = SHAPES["bf16_gqa_ragged"]
    d = lib.dims_of(shape)
    q, k, v, wq, wk = _upload(lib, shape)
    o = torch.empty_like(q)
    lib.still_hybrid_prefill_static(d, q, k, v, wq, wk, o)  # warm-up: may load the module holding the array
    torch.cuda.synchronize()
    before = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
    for _ in range(2):
        lib.still_hybrid_prefill_static(d, q, k, v, wq, wk, o)
    torch.cuda.synchronize()
    assert lib.still_get_device_status() == 0
    after = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
    assert after == before
