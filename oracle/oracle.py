"""ctypes front end of the C fp64 oracle (still_oracle.c).

TEST INFRASTRUCTURE: see the package docstring for who may call this.
Arrays are passed as contiguous float64 / int32 numpy arrays; every function
returns numpy arrays.  The C side computes each quantity directly from its
definition (page citations are in still_oracle.c).
"""
from __future__ import annotations

import ctypes as ct
import dataclasses
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "still_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libstill_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile still_oracle.c with gcc (plain -O2, IEEE math) if stale."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _ODims(ct.Structure):
    _fields_ = [(n, ct.c_int) for n in ("B", "H", "Hkv", "N", "d", "D", "w", "C", "k")] + [("scale", ct.c_double)]


@dataclasses.dataclass
class Dims:
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    D: int
    w: int
    C: int
    k: int
    scale: float | None = None   # None: 1/sqrt(d)

    @classmethod
    def of(cls, shape, **over) -> "Dims":
        kw = {f: getattr(shape, f) for f in ("B", "H", "Hkv", "N", "d", "D", "w", "C", "k")}
        kw.update(over)
        return cls(**kw)

    def c(self) -> _ODims:
        sc = self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)
        return _ODims(self.B, self.H, self.Hkv, self.N, self.d, self.D, self.w, self.C, self.k, sc)

    @property
    def T(self) -> int:
        return self.N // self.C


def _load():
    global _lib
    if _lib is None:
        lib = ct.CDLL(build())
        P = ct.c_void_p
        lib.od_saliency.argtypes = [ct.POINTER(_ODims), P, P, P, P, ct.c_int]
        lib.od_topk.argtypes = [ct.POINTER(_ODims), P, P]
        lib.od_diagonal_score.argtypes = [ct.POINTER(_ODims), P, P, P]
        lib.od_npmap.argtypes = [ct.c_int, ct.c_int, ct.c_int, P, P, P]
        lib.od_prefill.argtypes = [ct.POINTER(_ODims), P, P, P, P, P, P, P, P, P, P, ct.c_long, ct.c_int]
        lib.od_prefill_given_phik.argtypes = [ct.POINTER(_ODims), P, P, P, P, P, P, P, P, P, P, ct.c_long,
                                              ct.c_int]
        lib.od_linear_state.argtypes = [ct.POINTER(_ODims), P, P, P, P, ct.c_int, ct.c_int, ct.c_int, P, P]
        lib.od_decode_new.argtypes = [ct.POINTER(_ODims), P, P]
        lib.od_decode_new.restype = ct.c_void_p
        lib.od_decode_free.argtypes = [P]
        lib.od_decode_step.argtypes = [P, P, P, P, P, P]
        lib.od_decode_pos.argtypes = [P]
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ct.c_void_p)


def _nthreads(n):
    if n:
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def saliency(dims: Dims, q, k, nthreads: int | None = None):
    """Returns (sigma [B,H,N], r [B,Hkv,N]) in float64."""
    lib = _load()
    q, k = _f64(q), _f64(k)
    sigma = np.empty((dims.B, dims.H, dims.N))
    r = np.empty((dims.B, dims.Hkv, dims.N))
    _check(lib.od_saliency(ct.byref(dims.c()), _p(q), _p(k), _p(sigma), _p(r), _nthreads(nthreads)), "saliency")
    return sigma, r


def diagonal_score(dims: Dims, q, k) -> np.ndarray:
    """Diagonal-only router score r [B,Hkv,N] (float64): group mean of tau <q_hi, k_gi>."""
    lib = _load()
    q, k = _f64(q), _f64(k)
    r = np.empty((dims.B, dims.Hkv, dims.N))
    _check(lib.od_diagonal_score(ct.byref(dims.c()), _p(q), _p(k), _p(r)), "diagonal_score")
    return r


def topk(dims: Dims, r) -> np.ndarray:
    """r [B,Hkv,N] (float64; pass fp32 values upcast for bit-exact checks) -> idx [B,Hkv,T,k] int32."""
    lib = _load()
    r = _f64(r)
    idx = np.empty((dims.B, dims.Hkv, dims.T, dims.k), dtype=np.int32)
    _check(lib.od_topk(ct.byref(dims.c()), _p(r), _p(idx)), "topk")
    return idx


def npmap(x, W) -> np.ndarray:
    """x [n,d], W [d,D] -> phi [n,D]."""
    lib = _load()
    x, W = _f64(x), _f64(W)
    n, d = x.shape
    D = W.shape[1]
    phi = np.empty((n, D))
    _check(lib.od_npmap(n, d, D, _p(x), _p(W), _p(phi)), "npmap")
    return phi


def prefill(dims: Dims, q, k, v, wq, wk, idx_in=None, rows=None, nthreads: int | None = None, phik=None):
    """Full forward.  Returns dict(o=[B,H,N,d] (NaN where not computed), r, idx).

    idx_in [B,Hkv,T,k] injects the selection; rows [n,3] of (b,h,i) limits the
    output rows computed; phik [B,Hkv,N,D] (as npmap computes it for every key
    with its group's Wk) is used instead of computing phi(k) again (wk is then
    not read)."""
    lib = _load()
    q, k, v, wq = map(_f64, (q, k, v, wq))
    o = np.full((dims.B, dims.H, dims.N, dims.d), np.nan)
    r = np.full((dims.B, dims.Hkv, dims.N), np.nan)
    idx = np.zeros((dims.B, dims.Hkv, dims.T, dims.k), dtype=np.int32)
    ii = None if idx_in is None else _i32(idx_in)
    rr = None if rows is None else _i32(rows)
    nrows = 0 if rr is None else rr.shape[0]
    if phik is None:
        wk = _f64(wk)
        rc = lib.od_prefill(ct.byref(dims.c()), _p(q), _p(k), _p(v), _p(wq), _p(wk), _p(ii), _p(o), _p(r),
                            _p(idx), _p(rr), nrows, _nthreads(nthreads))
    else:
        phik = _f64(phik)
        if phik.shape != (dims.B, dims.Hkv, dims.N, dims.D):
            raise ValueError(f"phik has shape {phik.shape}, expected {(dims.B, dims.Hkv, dims.N, dims.D)}")
        rc = lib.od_prefill_given_phik(ct.byref(dims.c()), _p(q), _p(k), _p(v), _p(wq), _p(phik), _p(ii), _p(o),
                                       _p(r), _p(idx), _p(rr), nrows, _nthreads(nthreads))
    _check(rc, "prefill")
    return {"o": o, "r": r, "idx": idx}


def linear_state(dims: Dims, k, v, wk, idx, b: int, g: int, t: int):
    """(S_t [D,d], z_t [D]) seen by query chunk t of (b, g)."""
    lib = _load()
    k, v, wk = map(_f64, (k, v, wk))
    idx = _i32(idx)
    S = np.empty((dims.D, dims.d))
    z = np.empty((dims.D,))
    _check(lib.od_linear_state(ct.byref(dims.c()), _p(k), _p(v), _p(wk), _p(idx), b, g, t, _p(S), _p(z)),
           "linear_state")
    return S, z


class Decoder:
    """Incremental chunk-delayed decode state machine (dims.N = capacity)."""

    def __init__(self, dims: Dims, wq, wk):
        self._lib = _load()
        self.dims = dims
        self._wq, self._wk = _f64(wq), _f64(wk)
        self._h = self._lib.od_decode_new(ct.byref(dims.c()), _p(self._wq), _p(self._wk))
        if not self._h:
            raise RuntimeError("oracle decode state allocation failed")

    def step(self, q_t, k_t, v_t):
        """q_t [B,H,d], k_t/v_t [B,Hkv,d] -> (o_t [B,H,d], r_t [B,Hkv])."""
        q_t, k_t, v_t = map(_f64, (q_t, k_t, v_t))
        o = np.empty((self.dims.B, self.dims.H, self.dims.d))
        r = np.empty((self.dims.B, self.dims.Hkv))
        _check(self._lib.od_decode_step(self._h, _p(q_t), _p(k_t), _p(v_t), _p(o), _p(r)), "decode_step")
        return o, r

    @property
    def pos(self) -> int:
        return self._lib.od_decode_pos(self._h)

    def close(self):
        if self._h:
            self._lib.od_decode_free(self._h)
            self._h = None

    def __del__(self):
        self.close()
