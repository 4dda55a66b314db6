"""Python binding of libstill.so (include/still.h): argument marshalling only.

Each function has the name of its C entry point and takes device tensors (or
raw device addresses as ints); it passes their addresses, the sizes and the
current CUDA stream to the library and raises StillError on a non-OK status.
Every step of the computation runs in the library's kernels; there is no
fallback.  If libstill.so is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes as ct
import math
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libstill.so")

STILL_F32, STILL_BF16 = 0, 1
STATUS = {0: "STILL_OK", 1: "STILL_ERR_INVALID_ARG", 2: "STILL_ERR_UNSUPPORTED", 3: "STILL_ERR_WORKSPACE",
          4: "STILL_ERR_CUDA", 5: "STILL_ERR_DEVICE_CHECK", 6: "STILL_ERR_TIMEOUT"}

EXPORTS = ("still_status_string", "still_saliency", "still_select_topk", "still_npmap",
           "still_prefill_workspace_bytes", "still_prefill_workspace_layout", "still_hybrid_prefill",
           "still_decode_state_bytes", "still_decode_init", "still_decode_step", "still_get_device_status",
           "still_launch_count", "still_timing_enable", "still_timing_read", "still_debug_merge",
           "still_hybrid_prefill_static", "still_diagonal_score", "still_backward_workspace_bytes",
           "still_hybrid_backward", "still_hybrid_backward_saved", "still_decode_state_layout")


class StillError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} -> {STATUS.get(status, status)} ({status_string(status)})")


class still_dims(ct.Structure):
    _fields_ = [(n, ct.c_int) for n in ("B", "H", "Hkv", "N", "d", "D", "w", "C", "k")] + \
               [("scale", ct.c_float), ("dtype", ct.c_int)]


class still_state_layout(ct.Structure):
    _fields_ = [(n, ct.c_size_t) for n in ("header", "khat", "vhat", "S", "z", "ring_k", "ring_v", "ring_r", "total")] + \
               [("ring_rows", ct.c_int), ("cap_chunks", ct.c_int)]


class still_ws_layout(ct.Structure):
    _fields_ = [(n, ct.c_size_t) for n in ("r", "idx", "khat", "vhat", "S", "z", "phik", "sig", "lse", "fix", "wqt", "wkt", "st", "total")]


if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libstill.so is not built ({_LIB_PATH}); run linear_attention_still_b200._build")

_lib = ct.CDLL(_LIB_PATH)
_P = ct.c_void_p
_D = ct.POINTER(still_dims)
_SIG = {
    "still_status_string": ([ct.c_int], ct.c_char_p),
    "still_saliency": ([_D, _P, _P, _P, _P, _P], ct.c_int),
    "still_select_topk": ([_D, _P, _P, _P], ct.c_int),
    "still_diagonal_score": ([_D, _P, _P, _P, _P], ct.c_int),
    "still_npmap": ([ct.c_int, ct.c_int, ct.c_int, ct.c_int, ct.c_int, ct.c_int, _P, _P, _P, _P], ct.c_int),
    "still_prefill_workspace_bytes": ([_D], ct.c_size_t),
    "still_prefill_workspace_layout": ([_D, ct.POINTER(still_ws_layout)], ct.c_int),
    "still_hybrid_prefill": ([_D, _P, _P, _P, _P, _P, _P, _P, _P, ct.c_size_t, _P, ct.c_int, _P], ct.c_int),
    "still_hybrid_prefill_static": ([_D, _P, _P, _P, _P, _P, _P, _P, _P, ct.c_int, _P], ct.c_int),
    "still_backward_workspace_bytes": ([_D], ct.c_size_t),
    "still_hybrid_backward": ([_D] + [_P] * 13 + [ct.c_size_t, _P], ct.c_int),
    "still_hybrid_backward_saved": ([_D] + [_P] * 15 + [ct.c_size_t, _P], ct.c_int),
    "still_decode_state_bytes": ([_D, ct.c_int], ct.c_size_t),
    "still_decode_init": ([_D, ct.c_int, _P, _P], ct.c_int),
    "still_decode_state_layout": ([_D, ct.c_int, ct.POINTER(still_state_layout)], ct.c_int),
    "still_decode_step": ([_D, _P, ct.c_int, ct.c_int, _P, _P, _P, _P, _P, _P, _P], ct.c_int),
    "still_get_device_status": ([_P], ct.c_int),
    "still_launch_count": ([], ct.c_uint64),
    "still_timing_enable": ([ct.c_int], ct.c_int),
    "still_debug_merge": ([ct.c_int, ct.c_int], None),
    "still_timing_read": ([ct.POINTER(ct.c_double), ct.POINTER(ct.c_int), ct.c_int], ct.c_int),
}
for _name, (_args, _res) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def library_path() -> str:
    return _LIB_PATH


def make_dims(B, H, Hkv, N, d, D, w, C, k, dtype="bf16", scale=0.0) -> still_dims:
    dt = {"bf16": STILL_BF16, "f32": STILL_F32}[dtype] if isinstance(dtype, str) else int(dtype)
    return still_dims(B, H, Hkv, N, d, D, w, C, k, float(scale), dt)


def dims_of(shape, N: int | None = None) -> still_dims:
    """still_dims of a synth.Shape (N overridable)."""
    return make_dims(shape.B, shape.H, shape.Hkv, shape.N if N is None else N, shape.d, shape.D, shape.w,
                     shape.C, shape.k, shape.dtype)


def _ptr(x):
    """Address of a host-or-device operand (a tensor or a raw address)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _dptr(x, name: str = "operand"):
    """Address of a device operand.  A raw int is passed as given; a tensor must be a contiguous CUDA
    tensor on the current device -- the library takes no strides, and a host address or another
    device's memory handed to a kernel would be read as if it were this device's."""
    if x is None or isinstance(x, int):
        return x
    import torch
    if not x.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor, got one on {x.device}")
    if x.get_device() != torch.cuda.current_device():
        raise ValueError(f"{name}: tensor on cuda:{x.get_device()}, current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if not x.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor (the library takes no strides)")
    return x.data_ptr()


def _dargs(**operands) -> list:
    """_dptr of each keyword argument, in the order given."""
    return [_dptr(x, name) for name, x in operands.items()]


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ok(fn: str, st: int):
    if st != 0:
        raise StillError(fn, st)


def status_string(status: int) -> str:
    return _lib.still_status_string(int(status)).decode()


def still_saliency(dims, q, k, r_kv, r_q=None, stream=None):
    _ok("still_saliency", _lib.still_saliency(ct.byref(dims), *_dargs(q=q, k=k, r_kv=r_kv, r_q=r_q), _stream(stream)))


def still_select_topk(dims, r_kv, idx, stream=None):
    _ok("still_select_topk", _lib.still_select_topk(ct.byref(dims), *_dargs(r_kv=r_kv, idx=idx), _stream(stream)))


def still_diagonal_score(dims, q, k, r_kv, stream=None):
    _ok("still_diagonal_score",
        _lib.still_diagonal_score(ct.byref(dims), *_dargs(q=q, k=k, r_kv=r_kv), _stream(stream)))


def still_npmap(B, Hx, N, d, D, dtype, x, W, phi, stream=None):
    dt = {"bf16": STILL_BF16, "f32": STILL_F32}[dtype] if isinstance(dtype, str) else int(dtype)
    _ok("still_npmap", _lib.still_npmap(B, Hx, N, d, D, dt, *_dargs(x=x, W=W, phi=phi), _stream(stream)))


def still_prefill_workspace_bytes(dims) -> int:
    return int(_lib.still_prefill_workspace_bytes(ct.byref(dims)))


def still_prefill_workspace_layout(dims) -> dict:
    out = still_ws_layout()
    _ok("still_prefill_workspace_layout", _lib.still_prefill_workspace_layout(ct.byref(dims), ct.byref(out)))
    return {n: int(getattr(out, n)) for n, _ in still_ws_layout._fields_}


def still_hybrid_prefill(dims, q, k, v, wq, wk, o, idx_in=None, workspace=None, workspace_bytes=None, state=None,
                         state_capacity=0, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    a = _dargs(q=q, k=k, v=v, wq=wq, wk=wk, o=o, idx_in=idx_in, workspace=workspace, state=state)
    _ok("still_hybrid_prefill",
        _lib.still_hybrid_prefill(ct.byref(dims), *a[:8], int(workspace_bytes), a[8], int(state_capacity),
                                  _stream(stream)))


STATIC_WORKSPACE_BYTES = 64 << 20  # STILL_STATIC_WORKSPACE_BYTES


def still_hybrid_prefill_static(dims, q, k, v, wq, wk, o, idx_in=None, state=None, state_capacity=0, stream=None):
    """still_hybrid_prefill with the library's fixed device scratch (allocates nothing)."""
    a = _dargs(q=q, k=k, v=v, wq=wq, wk=wk, o=o, idx_in=idx_in, state=state)
    _ok("still_hybrid_prefill_static",
        _lib.still_hybrid_prefill_static(ct.byref(dims), *a, int(state_capacity), _stream(stream)))


def still_backward_workspace_bytes(dims) -> int:
    return int(_lib.still_backward_workspace_bytes(ct.byref(dims)))


def still_hybrid_backward(dims, q, k, v, wq, wk, idx, do, dq, dk, dv, dwq, dwk, workspace=None, workspace_bytes=None,
                          stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    a = _dargs(q=q, k=k, v=v, wq=wq, wk=wk, idx=idx, do=do, dq=dq, dk=dk, dv=dv, dwq=dwq, dwk=dwk,
               workspace=workspace)
    _ok("still_hybrid_backward",
        _lib.still_hybrid_backward(ct.byref(dims), *a, int(workspace_bytes), _stream(stream)))


def still_hybrid_backward_saved(dims, q, k, v, wq, wk, idx, do, o, lse, dq, dk, dv, dwq, dwk, workspace=None,
                                workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    a = _dargs(q=q, k=k, v=v, wq=wq, wk=wk, idx=idx, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv, dwq=dwq, dwk=dwk,
               workspace=workspace)
    _ok("still_hybrid_backward_saved",
        _lib.still_hybrid_backward_saved(ct.byref(dims), *a, int(workspace_bytes), _stream(stream)))


def still_decode_state_bytes(dims, capacity: int) -> int:
    return int(_lib.still_decode_state_bytes(ct.byref(dims), int(capacity)))


def still_decode_state_layout(dims, capacity) -> dict:
    out = still_state_layout()
    _ok("still_decode_state_layout", _lib.still_decode_state_layout(ct.byref(dims), int(capacity), ct.byref(out)))
    return {n: int(getattr(out, n)) for n, _ in still_state_layout._fields_}


def still_decode_init(dims, capacity, state, stream=None):
    _ok("still_decode_init", _lib.still_decode_init(ct.byref(dims), int(capacity), *_dargs(state=state),
                                                    _stream(stream)))


def still_decode_step(dims, state, capacity, pos, wq, wk, q_t, k_t, v_t, o_t, stream=None):
    (st,) = _dargs(state=state)
    _ok("still_decode_step",
        _lib.still_decode_step(ct.byref(dims), st, int(capacity), int(pos),
                               *_dargs(wq=wq, wk=wk, q_t=q_t, k_t=k_t, v_t=v_t, o_t=o_t), _stream(stream)))


def still_get_device_status(stream=None) -> int:
    """Synchronises the stream; returns the (cleared) device status code."""
    return int(_lib.still_get_device_status(_stream(stream)))


def still_launch_count() -> int:
    return int(_lib.still_launch_count())


def still_debug_merge(stall: bool = False, max_ctas: int = 0):
    """Test hooks of the head-dim-64 tensor-core merge: `stall` makes the first CTA of each later
    launch load no key/value tile (its bounded wait runs out: STILL_ERR_TIMEOUT); `max_ctas` > 0 caps
    the persistent grid.  Defaults restore normal operation."""
    _lib.still_debug_merge(1 if stall else 0, int(max_ctas))


TIMING_CLASSES = ("saliency", "topk_gather", "npmap", "linear_state", "merge", "state_export", "merge_prefix",
                  "decode_append", "decode_attn", "decode_combine", "decode_close", "bwd_dq", "bwd_dkv",
                  "bwd_linear")


def still_timing_enable(on: bool = True):
    _ok("still_timing_enable", _lib.still_timing_enable(1 if on else 0))


def still_timing_read() -> dict:
    """{class: (milliseconds, launches)} of the kernels timed since the last read."""
    n = len(TIMING_CLASSES)
    ms = (ct.c_double * n)()
    cnt = (ct.c_int * n)()
    _ok("still_timing_read", _lib.still_timing_read(ms, cnt, n))
    return {name: (ms[i], cnt[i]) for i, name in enumerate(TIMING_CLASSES)}


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
