"""Seeded synthetic inputs for the STILL hybrid-attention layer.

This module only draws numbers and rounds them to the storage dtype; it holds
none of the method's arithmetic.  Both the CUDA path (tests, bench) and the CPU
oracle are fed from here, so the two sides always see bit-identical inputs.

Value distribution (STILL: Selecting Tokens for Intra-Layer Hybrid Attention
to Linearize LLMs, "Efficiency" results: Llama-3.2-1B / Llama-3.1-8B layers at
16K-64K context; the pages print no input recipe, so this one is a reading):

* every token-head vector of Q, K and V is drawn N(0, I_d) and multiplied by a
  per-(batch, head, token) factor lambda ~ LogNormal(0, 0.5);
* a few "heavy" token positions (1 % of N, or 4 for the small fp32 case) are
  drawn without replacement from [1, N) per batch item; their Q, K and V rows
  are scaled by 4 in every head;
* the NP-Map weights Wq [H, d, D] and Wk [Hkv, d, D] are N(0, 1/d);
* everything is drawn in fp32 from numpy PCG64 streams: SeedSequence(seed)
  spawns B+1 children; child 0 draws Wq then Wk, child 1+b draws batch item
  b's Q, K, V, lambda_q, lambda_k, lambda_v and heavy positions in that order
  (so one batch item can be regenerated alone); then everything is rounded
  to the workload dtype (bf16 by round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["Shape", "WORKLOADS", "Inputs", "make_inputs", "round_to_bf16", "round_to_bf16_", "bf16_bits_to_f32"]


@dataclasses.dataclass(frozen=True)
class Shape:
    """One STILL layer problem: Q [B,H,N,d], K/V [B,Hkv,N,d], window w = m*C,
    chunk C, k tokens kept per chunk, NP-Map feature width D."""

    B: int
    H: int
    Hkv: int
    N: int
    d: int
    D: int
    w: int
    C: int
    k: int
    dtype: str = "bf16"          # "f32" or "bf16": storage and I/O type
    heavy: int | None = None     # planted heavy tokens per batch item (None: 1% of N)
    decode_steps: int = 0        # tokens generated after a prefill of N (decode workloads)
    seed: int = 0

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def T(self) -> int:          # full chunks
        return self.N // self.C

    @property
    def n_heavy(self) -> int:
        return self.heavy if self.heavy is not None else (self.N + self.decode_steps) // 100

    def replace(self, **kw) -> "Shape":
        return dataclasses.replace(self, **kw)


# Workloads named by what they are.  The first one is small enough for the
# oracle to finish in seconds; the others follow the pages' efficiency settings.
WORKLOADS = {
    "still_f32_b1_h2_n512": Shape(B=1, H=2, Hkv=2, N=512, d=64, D=64, w=64, C=64, k=8,
                                  dtype="f32", heavy=4),
    # the same layer decoding 128 tokens after its 512-token prefill (a chunk close every 64)
    "still_f32_decode_b1_ctx512": Shape(B=1, H=2, Hkv=2, N=512, d=64, D=64, w=64, C=64, k=8,
                                        dtype="f32", heavy=4, decode_steps=128),
    "llama32_1b_layer_n16k": Shape(B=1, H=32, Hkv=8, N=16384, d=64, D=64, w=512, C=512, k=64),
    # the same layer with no softmax window (w = 0, k = 0): pure chunked linear attention with NP-Map
    "llama32_1b_linear_n16k": Shape(B=1, H=32, Hkv=8, N=16384, d=64, D=64, w=0, C=512, k=0),
    "llama31_8b_layer_b4_n16k": Shape(B=4, H=32, Hkv=8, N=16384, d=128, D=128, w=1024, C=1024, k=128),
    "llama31_8b_layer_n64k": Shape(B=1, H=32, Hkv=8, N=65536, d=128, D=128, w=1024, C=1024, k=128),
    "llama31_8b_decode_b16_ctx64k": Shape(B=16, H=32, Hkv=8, N=65536, d=128, D=128, w=1024, C=1024,
                                          k=128, decode_steps=1024),
    # the same decode at batch 4: small enough (about 5 GB on the device) for multi-pass profiling
    "llama31_8b_decode_b4_ctx64k": Shape(B=4, H=32, Hkv=8, N=65536, d=128, D=128, w=1024, C=1024,
                                         k=128, decode_steps=1024),
}


def round_to_bf16(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round fp32 -> bf16 (round to nearest, ties to even).

    Returns (values as fp32, raw bf16 bit patterns as uint16).  Inputs are
    finite by construction."""
    vals = np.array(x, dtype=np.float32, copy=True)
    round_to_bf16_(vals)
    return vals, (vals.view(np.uint32) >> 16).astype(np.uint16)


def round_to_bf16_(x: np.ndarray) -> np.ndarray:
    """In-place variant: x (contiguous fp32) is replaced by its bf16-rounded values."""
    u = x.view(np.uint32)
    tmp = u >> 16
    tmp &= 1
    tmp += np.uint32(0x7FFF)
    u += tmp
    u &= np.uint32(0xFFFF0000)
    return x


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Inputs:
    shape: Shape
    q: np.ndarray      # [B, H, Ntot, d]  fp32 holding dtype-representable values
    k: np.ndarray      # [B, Hkv, Ntot, d]
    v: np.ndarray      # [B, Hkv, Ntot, d]
    wq: np.ndarray     # [H, d, D]
    wk: np.ndarray     # [Hkv, d, D]
    heavy: np.ndarray  # [B, n_heavy] int64 positions

    def bits(self, name: str) -> np.ndarray:
        """bf16 bit patterns of one tensor (bf16 workloads only)."""
        assert self.shape.dtype == "bf16"
        return round_to_bf16(getattr(self, name))[1]


def make_inputs(shape: Shape, seed: int | None = None, batches=None, threads: int = 1) -> Inputs:
    """Draw the inputs for `shape` (Ntot = N + decode_steps tokens).

    batches: optional list of batch indices to draw (others are skipped); the
    returned arrays then hold only those items, in the given order.
    threads: batch items drawn concurrently (each from its own stream, so the
    values do not depend on it; numpy's generators release the GIL while they
    fill an array)."""
    s = shape
    seed = s.seed if seed is None else seed
    ntot = s.N + s.decode_steps
    bsel = list(range(s.B)) if batches is None else [int(b) for b in batches]
    f32 = np.float32
    children = np.random.SeedSequence(seed).spawn(s.B + 1)
    wrng = np.random.Generator(np.random.PCG64(children[0]))
    wq = wrng.standard_normal((s.H, s.d, s.D), dtype=f32) * f32(1.0 / math.sqrt(s.d))
    wk = wrng.standard_normal((s.Hkv, s.d, s.D), dtype=f32) * f32(1.0 / math.sqrt(s.d))
    nb = len(bsel)
    q = np.empty((nb, s.H, ntot, s.d), dtype=f32)
    k = np.empty((nb, s.Hkv, ntot, s.d), dtype=f32)
    v = np.empty((nb, s.Hkv, ntot, s.d), dtype=f32)
    nh = min(s.n_heavy, max(ntot - 1, 0))
    heavy = np.zeros((nb, nh), dtype=np.int64)

    def draw(n: int, b: int) -> None:
        rng = np.random.Generator(np.random.PCG64(children[1 + b]))
        rng.standard_normal((s.H, ntot, s.d), dtype=f32, out=q[n])
        rng.standard_normal((s.Hkv, ntot, s.d), dtype=f32, out=k[n])
        rng.standard_normal((s.Hkv, ntot, s.d), dtype=f32, out=v[n])
        lq = rng.lognormal(0.0, 0.5, size=(s.H, ntot)).astype(f32)
        lk = rng.lognormal(0.0, 0.5, size=(s.Hkv, ntot)).astype(f32)
        lv = rng.lognormal(0.0, 0.5, size=(s.Hkv, ntot)).astype(f32)
        if nh > 0:
            heavy[n] = rng.choice(np.arange(1, ntot), size=nh, replace=False)
        q[n] *= lq[..., None]
        k[n] *= lk[..., None]
        v[n] *= lv[..., None]
        pos = heavy[n]
        q[n][:, pos, :] *= f32(4.0)
        k[n][:, pos, :] *= f32(4.0)
        v[n][:, pos, :] *= f32(4.0)
        if s.dtype == "bf16":
            for a in (q[n], k[n], v[n]):
                round_to_bf16_(a)

    if s.dtype not in ("bf16", "f32"):
        raise ValueError(f"unknown dtype {s.dtype}")
    if threads > 1 and nb > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(threads, nb)) as ex:
            list(ex.map(lambda nb_: draw(*nb_), enumerate(bsel)))
    else:
        for n, b in enumerate(bsel):
            draw(n, b)
    if s.dtype == "bf16":
        for a in (wq, wk):
            round_to_bf16_(a)
    return Inputs(s, q, k, v, wq, wk, heavy)
