"""Helpers of the GPU parity tests: upload seeded inputs, run the C-ABI entry points, read the
intermediate results out of the workspace, and compare against the fp64 oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

from linear_attention_still_b200 import still
from linear_attention_still_b200.synth import Shape

# Tolerances: outputs row-normwise relative error (1e-4 fp32, 2e-2 bf16), scores |r - r*| / max(|r*|, 1) <= 1e-3.
OUT_TOL = {"f32": 1e-4, "bf16": 2e-2}
SCORE_TOL = 1e-3


def tdtype(shape: Shape):
    return torch.bfloat16 if shape.dtype == "bf16" else torch.float32


def dev(a, shape: Shape):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(tdtype(shape))


def odims(shape: Shape, N: int | None = None, **over):
    import oracle
    return oracle.Dims.of(shape.replace(N=shape.N if N is None else N), **over)


def ws_view(ws, L, name, dtype, shape):
    n = int(np.prod(shape))
    esz = torch.tensor([], dtype=dtype).element_size()
    return ws[L[name]: L[name] + n * esz].view(dtype).view(*shape)


def gpu_prefill(shape: Shape, inp, N: int | None = None, idx_in=None, state=None, capacity: int = 0):
    N = shape.N if N is None else N
    d = still.dims_of(shape, N)
    q, k, v = (dev(getattr(inp, n)[:, :, :N], shape) for n in ("q", "k", "v"))
    wq, wk = dev(inp.wq, shape), dev(inp.wk, shape)
    o = torch.full_like(q, float("nan"))
    ws = torch.zeros(max(still.still_prefill_workspace_bytes(d), 256), dtype=torch.uint8, device="cuda")
    ii = None if idx_in is None else torch.from_numpy(np.ascontiguousarray(idx_in, dtype=np.int32)).cuda()
    still.still_hybrid_prefill(d, q, k, v, wq, wk, o, idx_in=ii, workspace=ws, state=state, state_capacity=capacity)
    status = still.still_get_device_status()
    L = still.still_prefill_workspace_layout(d)
    B, Hkv, T = shape.B, shape.Hkv, N // shape.C
    out = {
        "o": o.float().cpu().numpy(),
        "r": ws_view(ws, L, "r", torch.float32, (B, Hkv, N)).cpu().numpy(),
        "idx": ws_view(ws, L, "idx", torch.int32, (B, Hkv, T, shape.k)).cpu().numpy(),
        "S": ws_view(ws, L, "S", torch.float32, (B, Hkv, T + 1, shape.D, shape.d)).cpu().numpy(),
        "z": ws_view(ws, L, "z", torch.float32, (B, Hkv, T + 1, shape.D)).cpu().numpy(),
        "status": status,
    }
    return out


def row_rel_err(o, ref) -> float:
    o = np.asarray(o, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(o).all(), "non-finite GPU output"
    num = np.abs(o - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return float((num / np.maximum(den, 1e-30)).max()) if num.size else 0.0


def score_err(r, ref) -> float:
    r = np.asarray(r, np.float64)
    ref = np.asarray(ref, np.float64)
    both_inf = np.isinf(r) & np.isinf(ref) & (np.sign(r) == np.sign(ref))
    with np.errstate(invalid="ignore"):   # inf - inf on the both_inf entries, masked below
        err = np.where(both_inf, 0.0, np.abs(r - ref) / np.maximum(np.abs(ref), 1.0))
    err = np.where(np.isnan(err), np.inf, err)
    return float(err.max()) if err.size else 0.0


def check_selection(shape: Shape, N: int, gpu_idx, gpu_r, ora_r, ora_idx, tol=SCORE_TOL):
    """GPU selection is bit-exact given its own scores, and differs from the oracle's selection only
    between tokens whose oracle scores are within the score tolerance."""
    import oracle
    d = odims(shape, N)
    again = oracle.topk(d, np.asarray(gpu_r, np.float32).astype(np.float64))
    np.testing.assert_array_equal(gpu_idx, again)
    B, Hkv, T, k = gpu_idx.shape
    swaps = 0
    for b in range(B):
        for g in range(Hkv):
            for c in range(T):
                A, O = set(gpu_idx[b, g, c].tolist()), set(ora_idx[b, g, c].tolist())
                for a in A - O:
                    for o_ in O - A:
                        ra, ro = ora_r[b, g, a], ora_r[b, g, o_]
                        assert abs(ra - ro) <= 2 * tol * max(1.0, abs(ro)), (b, g, c, a, o_, ra, ro)
                swaps += len(A - O)
    return swaps


def pick_rows(shape: Shape, N: int, n: int, seed: int = 0, b: int | None = None):
    """Sample (b, h, i) rows covering the first, middle and last chunks and the ragged tail."""
    rng = np.random.default_rng(seed)
    rows = set()
    last = N - 1
    for i in (0, 1, min(shape.C - 1, last), min(shape.C, last), N // 2, last):
        rows.add((0 if b is None else b, int(rng.integers(shape.H)), i))
    while len(rows) < n:
        rows.add((int(rng.integers(shape.B)) if b is None else b, int(rng.integers(shape.H)),
                  int(rng.integers(N))))
    return np.array(sorted(rows), dtype=np.int32)


def nan_to_num_inf(x):
    return np.where(np.isposinf(x), math.inf, x)
