"""Randomised check of the host-side dims validation against the rules include/still.h states
(restated here from the header, not from the implementation): for any dims the size queries
return 0 exactly when a rule is broken, and an entry point given such dims returns
STILL_ERR_INVALID_ARG or STILL_ERR_UNSUPPORTED as the header assigns them, before touching any
pointer; for valid dims the workspace segments hold the documented tensors.  No GPU needed: no
call here gets past validation."""
import ctypes as ct
import math

import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

FAKE = 1 << 20  # never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    return still


def header_status(B, H, Hkv, N, d, D, w, C, k, scale, dtype):
    """0 (valid), 1 (STILL_ERR_INVALID_ARG) or 2 (STILL_ERR_UNSUPPORTED) by the header's rules."""
    if B < 0 or N < 0 or H < 1 or Hkv < 1 or C < 1 or k < 0 or w < 0:
        return 1
    if H % Hkv or k > C or w % C or (w == 0 and k != 0):
        return 1
    if dtype not in (0, 1):
        return 1
    if d < 8 or d % 8 or D < 8 or D % 8:
        return 1
    if not math.isfinite(scale) or scale < 0:
        return 1
    if d > 256 or D > 256 or H // Hkv > 32 or C > 16384 or B * H > 65535 or N > 1 << 26:
        return 2
    return 0


@st.composite
def dims_st(draw):
    """Valid dims, then (half the time) one rule broken or one limit passed."""
    Hkv = draw(st.sampled_from([1, 2, 4, 8]))
    C = draw(st.sampled_from([16, 64, 128, 512, 1024]))
    m = draw(st.integers(0, 3))
    p = {"B": draw(st.integers(1, 8)), "Hkv": Hkv, "H": Hkv * draw(st.sampled_from([1, 2, 4, 8, 32])),
         "N": draw(st.integers(0, 5000)), "d": draw(st.sampled_from([8, 16, 64, 96, 128, 256])),
         "D": draw(st.sampled_from([8, 32, 64, 128, 256])), "C": C, "w": m * C,
         "k": draw(st.integers(0, C)) if m > 0 else 0, "scale": draw(st.sampled_from([0.0, 0.125, 1.0])),
         "dtype": draw(st.sampled_from([0, 1]))}
    breaks = {
        "B": -1, "N": -1, "H": 0, "Hkv": 0, "C": 0, "k": -1, "w": -C,
        "H%Hkv": None, "k>C": None, "w%C": None, "w0k": None, "dtype": 2, "d": 12, "D": 4, "scale": None,
        "d>256": 264, "D>256": 512, "G>32": None, "C>16384": 16400, "B*H": None, "N>2^26": (1 << 26) + 1,
    }
    which = draw(st.sampled_from([None] * len(breaks) + sorted(breaks)))
    if which in ("B", "N", "H", "Hkv", "C", "k", "w", "dtype", "d", "D", "d>256", "D>256", "C>16384", "N>2^26"):
        key = {"d>256": "d", "D>256": "D", "C>16384": "C", "N>2^26": "N"}.get(which, which)
        p[key] = breaks[which]
        if which == "C>16384":
            p["w"] = p["C"] * max(1, m) if p["w"] else 0
    elif which == "H%Hkv":
        p["Hkv"], p["H"] = 3, 8
    elif which == "k>C":
        p["w"], p["k"] = max(1, m) * C, C + 1
    elif which == "w%C":
        p["w"] = max(1, m) * C + 1
    elif which == "w0k":
        p["w"], p["k"] = 0, 1
    elif which == "scale":
        p["scale"] = draw(st.sampled_from([-1.0, math.inf, math.nan]))
    elif which == "G>32":
        p["H"] = p["Hkv"] * 64
    elif which == "B*H":
        p["H"], p["Hkv"], p["B"] = 32, 8, 2048 + 1
    return p


@settings(max_examples=400, deadline=None)
@given(dims_st())
def test_validation_follows_the_header(lib, p):
    args = (p["B"], p["H"], p["Hkv"], p["N"], p["d"], p["D"], p["w"], p["C"], p["k"], p["scale"], p["dtype"])
    want = header_status(*args)
    d = lib.still_dims(*args)
    ws = lib.still_prefill_workspace_bytes(d)
    if want:
        assert ws == 0
        assert lib.still_backward_workspace_bytes(d) == 0
        got = lib._lib.still_hybrid_prefill(ct.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                                            None, 0, None)
        assert got == want, (args, got)
        return
    if p["B"] * p["N"] > 0:
        assert ws > 0
    L = lib.still_prefill_workspace_layout(d)
    B, H, Hkv, N, hd, D, C, k = d.B, d.H, d.Hkv, d.N, d.d, d.D, d.C, d.k
    T = N // C
    es = 2 if d.dtype == 1 else 4
    need = {"r": B * Hkv * N * 4, "idx": B * Hkv * T * k * 4, "khat": B * Hkv * T * k * hd * es,
            "vhat": B * Hkv * T * k * hd * es, "S": B * Hkv * (T + 1) * D * hd * 4, "z": B * Hkv * (T + 1) * D * 4}
    order = ["r", "idx", "khat", "vhat", "S", "z", "phik", "sig", "lse", "fix", "wqt", "wkt", "st", "total"]
    for a, b in zip(order, order[1:]):
        assert L[a] % 256 == 0 and L[a] <= L[b], (args, a)
        if a in need:
            assert L[b] - L[a] >= need[a], (args, a)
    assert L["total"] == ws
