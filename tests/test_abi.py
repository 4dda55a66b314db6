"""CPU checks of the C-ABI library: it loads, exports every entry point include/still.h declares,
and rejects bad arguments on the host before launching anything (no GPU needed)."""
import ctypes as ct
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    return still


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"STILL_API\s+[\w\s\*]+?\b(still_\w+)\s*\(", txt)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert len(declared) >= 12
    so = ct.CDLL(lib.library_path())
    for name in declared:
        assert hasattr(so, name), name
    assert set(declared) == set(lib.EXPORTS)


def test_status_strings(lib):
    for code in range(7):
        assert lib.status_string(code)
    assert lib.status_string(99) == "unknown status"


def _dims(lib, **kw):
    base = dict(B=1, H=4, Hkv=2, N=300, d=64, D=64, w=128, C=64, k=8, dtype="bf16")
    base.update(kw)
    return lib.make_dims(**base)


FAKE = 1 << 20  # an aligned address that is never dereferenced: validation fails first


@pytest.mark.parametrize("kw,code", [
    (dict(w=100), 1),          # window not a whole number of chunks
    (dict(w=0, k=4), 1),       # no window but tokens kept
    (dict(k=65), 1),           # k > C
    (dict(H=6, Hkv=4), 1),     # H % Hkv
    (dict(d=12), 1),           # head dim not a multiple of 8
    (dict(D=0), 1),
    (dict(d=512), 2),          # beyond the supported head dim
    (dict(H=64, Hkv=1), 2),    # group larger than 32
    (dict(N=-1), 1),
    (dict(dtype=7), 1),
])
def test_prefill_rejects_bad_dims(lib, kw, code):
    d = _dims(lib, **kw)
    assert lib._lib.still_hybrid_prefill(ct.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                                         None, 0, None) == code
    assert lib.still_prefill_workspace_bytes(d) == 0


def test_prefill_rejects_bad_pointers_and_workspace(lib):
    d = _dims(lib)
    need = lib.still_prefill_workspace_bytes(d)
    assert need > 0
    L = lib.still_prefill_workspace_layout(d)
    assert L["total"] == need and L["r"] == 0
    assert all(L[a] < L[b] for a, b in zip(("r", "idx", "khat", "vhat", "S", "z", "phik"),
                                             ("idx", "khat", "vhat", "S", "z", "phik", "total")))
    f = lib._lib.still_hybrid_prefill
    assert f(ct.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need, None, 0, None) == 1
    assert f(ct.byref(d), FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need, None, 0, None) == 1
    assert f(ct.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need - 1, None, 0, None) == 3
    assert f(ct.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need, FAKE, 299, None) == 1
    assert f(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need, None, 0, None) == 1


def test_step_entry_points_reject(lib):
    d = _dims(lib, w=0, k=0)
    assert lib._lib.still_saliency(ct.byref(d), FAKE, FAKE, FAKE, None, None) == 1  # needs a window
    d = _dims(lib)
    assert lib._lib.still_saliency(ct.byref(d), None, FAKE, FAKE, None, None) == 1
    assert lib._lib.still_select_topk(ct.byref(d), FAKE + 8, FAKE, None) == 1
    assert lib._lib.still_diagonal_score(ct.byref(d), FAKE, None, FAKE, None) == 1
    assert lib._lib.still_diagonal_score(ct.byref(d), FAKE, FAKE, FAKE + 4, None) == 1
    assert lib._lib.still_npmap(1, 2, 10, 12, 64, 1, FAKE, FAKE, FAKE, None) == 1
    assert lib._lib.still_npmap(1, 2, 10, 64, 512, 1, FAKE, FAKE, FAKE, None) == 2


def test_backward_rejects(lib):
    f = lib._lib.still_hybrid_backward
    d0 = _dims(lib, w=0, k=0)
    assert lib.still_backward_workspace_bytes(d0) > 0                    # no window: covered (sized, no call)
    d = _dims(lib)
    need = lib.still_backward_workspace_bytes(d)
    assert need > 0
    args = [FAKE] * 13
    args[5] = None                                                       # selection missing (k > 0)
    assert f(ct.byref(d), *args, need, None) == 1
    assert f(ct.byref(d), *([FAKE] * 13), need - 1, None) == 3           # workspace too small
    args = [FAKE] * 13
    args[6] = FAKE + 4                                                   # misaligned dO
    assert f(ct.byref(d), *args, need, None) == 1
    # the form that takes the forward's output and normaliser refuses before any launch as well
    fs = lib._lib.still_hybrid_backward_saved
    for i, bad in ((7, None), (8, None), (8, FAKE + 4), (5, None)):       # o, lse, misaligned lse, idx
        args = [FAKE] * 15
        args[i] = bad
        assert fs(ct.byref(d), *args, need, None) == 1, i
    assert fs(ct.byref(d), *([FAKE] * 15), need - 1, None) == 3


def test_decode_rejects(lib):
    d = _dims(lib)
    assert lib.still_decode_state_bytes(d, 4096) > 0
    f = lib._lib.still_decode_step
    assert f(ct.byref(d), FAKE, 100, 100, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1   # pos == capacity
    assert f(ct.byref(d), FAKE, 100, -1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(ct.byref(d), None, 100, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert lib._lib.still_decode_init(ct.byref(d), -1, FAKE, None) == 1


def test_decode_state_size_grows_with_capacity(lib):
    d = _dims(lib)
    a, b = lib.still_decode_state_bytes(d, 1024), lib.still_decode_state_bytes(d, 8192)
    assert b > a > 0


def test_binding_fails_loudly_without_the_library(tmp_path):
    """No fallback: a package copy without libstill.so refuses to import its binding."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "linear_attention_still_b200")
    dst = tmp_path / "linear_attention_still_b200"
    dst.mkdir()
    for f in ("__init__.py", "still.py", "synth.py"):
        shutil.copy(os.path.join(pkg, f), dst / f)
    r = subprocess.run([sys.executable, "-c", "import linear_attention_still_b200.still"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libstill.so is not built" in r.stderr


@pytest.mark.parametrize("kw", [dict(), dict(dtype="f32"), dict(d=128, D=128, w=256, C=128, k=32, N=1300),
                                dict(N=50), dict(w=0, k=0), dict(N=1)])
def test_workspace_segments_hold_the_documented_tensors(lib, kw):
    """Every segment of still_prefill_workspace_layout is 256-byte aligned, segments follow each
    other without overlap, and each is at least as large as the tensor the header documents for
    it (sizes restated here from the header's shapes)."""
    d = _dims(lib, **kw)
    L = lib.still_prefill_workspace_layout(d)
    B, H, Hkv, N, hd, D, C, k = d.B, d.H, d.Hkv, d.N, d.d, d.D, d.C, d.k
    T = N // C
    es = 2 if d.dtype == 1 else 4
    need = {"r": B * Hkv * N * 4, "idx": B * Hkv * T * k * 4, "khat": B * Hkv * T * k * hd * es,
            "vhat": B * Hkv * T * k * hd * es, "S": B * Hkv * (T + 1) * D * hd * 4,
            "z": B * Hkv * (T + 1) * D * 4}
    order = ["r", "idx", "khat", "vhat", "S", "z", "phik", "sig", "lse", "fix", "wqt", "wkt", "st", "total"]
    for a, b in zip(order, order[1:]):
        assert L[a] % 256 == 0 and L[a] <= L[b], (a, b)
        if a in need:
            assert L[b] - L[a] >= need[a], a
    if d.dtype == 1:  # bf16 path: per-head scores and the tensor-core operands
        assert L["lse"] - L["sig"] >= B * H * N * 4
        assert L["wqt"] - L["fix"] >= 256 + B * H * N * 4
        assert L["wkt"] - L["wqt"] >= H * D * hd * 2
        assert L["total"] - L["st"] >= B * Hkv * (T + 1) * hd * D * 2
    assert L["total"] == lib.still_prefill_workspace_bytes(d)
    bw = lib.still_backward_workspace_bytes(d)
    if d.w > 0:
        # phik, S, z, A, D, dYq, R, r, dYk, Ms, 1/Z (fp32)
        floats = (B * Hkv * N * D + 2 * B * Hkv * (T + 1) * (D * hd + D) + B * H * N * (2 * D + 3)
                  + B * Hkv * N * D)
        assert bw >= floats * 4


def test_binding_refuses_host_tensors_before_calling_the_library(lib):
    """The binding hands the library bare addresses, so it refuses tensors that are not on the GPU
    (a host address read by a kernel would fault) -- before any library call, so no GPU is needed."""
    import torch
    d = _dims(lib)
    host = torch.zeros(1, 4, 300, 64, dtype=torch.bfloat16)
    r = torch.zeros(1, 2, 300)
    with pytest.raises(ValueError, match="q: expected a CUDA tensor"):
        lib.still_saliency(d, host, FAKE, r)
    with pytest.raises(ValueError, match="r_kv: expected a CUDA tensor"):
        lib.still_diagonal_score(d, FAKE, FAKE, r)
    with pytest.raises(ValueError, match="workspace: expected a CUDA tensor"):
        lib.still_hybrid_prefill(d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, workspace=torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="state: expected a CUDA tensor"):
        lib.still_decode_step(d, torch.zeros(16, dtype=torch.uint8), 64, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    with pytest.raises(ValueError, match="o_t: expected a CUDA tensor"):
        lib.still_decode_step(d, FAKE, 64, 0, FAKE, FAKE, FAKE, FAKE, FAKE, torch.zeros(4, 64))
    with pytest.raises(ValueError, match="dwk: expected a CUDA tensor"):
        lib.still_hybrid_backward(d, *([FAKE] * 11), torch.zeros(2, 64, 64), workspace=FAKE, workspace_bytes=1 << 30)
    # raw addresses (and a raw stream handle) pass through unchanged: the library's own validation answers
    with pytest.raises(lib.StillError, match="INVALID_ARG"):
        lib.still_saliency(lib.make_dims(B=1, H=4, Hkv=2, N=300, d=64, D=64, w=0, C=64, k=0), FAKE, FAKE, FAKE,
                           stream=0)
