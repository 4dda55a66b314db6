"""Gradient of the STILL layer output -- TEST INFRASTRUCTURE (see the package docstring).

The pages describe the hybrid layer as trained and run with one chunk-parallel implementation
("STILL: Selecting Tokens for Intra-Layer Hybrid Attention to Linearize LLMs", [p1] jsqmd.com
introduction and "Chunk-Wise").  The backward pass is the exact derivative of the forward
definition the oracle computes (same routing sets, NP-Map and shared normaliser), with the
per-chunk selection held fixed: the top-k is a discrete choice with no gradient.  Written out
per query row in fp64 numpy, for small inputs; pinned against central finite differences of the
C forward oracle.

For query row i of head h (group g) with softmax set Soft(i) and linear set Lin(i):
    e_ij = exp(s_ij), s_ij = tau <q_i, k_j>          (j in Soft)
    w_ij = <phi(q_i; Wq_h), phi(k_j; Wk_g)>           (j in Lin)
    Z_i = sum_Soft e_ij + sum_Lin w_ij,  o_i = (sum_Soft e_ij v_j + sum_Lin w_ij v_j) / Z_i
and with g_i = dL/do_i, delta_ij = <g_i, v_j - o_i> / Z_i:
    dL/ds_ij = e_ij delta_ij,  dL/dw_ij = delta_ij,  dL/dv_j += (e_ij or w_ij) g_i / Z_i.
"""
from __future__ import annotations

import math

import numpy as np


def _softmax(y):
    e = np.exp(y - y.max())
    return e / e.sum()


def npmap_forward(x, W):
    """phi(x) = ||x|| f / ||f||, f = softmax(x W) over the features."""
    f = _softmax(x @ W)
    return np.linalg.norm(x) * f / np.linalg.norm(f)


def npmap_backward(x, W, dphi):
    """(dx, dW) of phi(x; W) for an upstream gradient dphi."""
    y = x @ W
    f = _softmax(y)
    nf = np.linalg.norm(f)
    u = f / nf
    n = np.linalg.norm(x)
    dn = float(dphi @ u)                 # phi = n u
    du = n * dphi
    df = (du - u * float(u @ du)) / nf   # u = f / ||f||
    dy = f * (df - float(f @ df))        # f = softmax(y)
    dx = W @ dy + (dn * x / n if n > 0 else 0.0)
    dW = np.outer(x, dy)
    return dx, dW


def routing_sets(i, N, w, C, sel_of_chunk):
    """(Soft(i), Lin(i)) under the chunk-granular delayed selection (chunk c is decided for query
    chunk t iff c <= t - m - 1); w = 0 puts every j <= i in the linear set."""
    if w == 0:
        return [], list(range(i + 1))
    m, t, T = w // C, i // C, N // C
    local = list(range(max(0, (t - m) * C), i + 1))
    soft, lin = [], []
    for c in range(0, min(t - m, T)):
        kept = set(sel_of_chunk(c))
        soft += sorted(kept)
        lin += [j for j in range(c * C, (c + 1) * C) if j not in kept]
    return soft + local, lin


def _round_bf16(x):
    """x rounded to the nearest bf16 (ties to even), returned in fp64."""
    x = np.array(x, dtype=np.float32)
    u = x.view(np.uint32)
    u += ((u >> 16) & 1) + np.uint32(0x7FFF)
    u &= np.uint32(0xFFFF0000)
    return x.astype(np.float64)


def layer_backward(q, k, v, wq, wk, do, idx, w, C, scale=None, d_from_output=None):
    """Gradients (dq, dk, dv, dwq, dwk) of L = sum(do * o) with the selection idx [B,Hkv,T,k] held
    fixed (idx may be None when no chunk is ever decided, or k = 0).

    d_from_output="bf16": the row term D_i = <do_i, o_i> is formed from the row's output rounded to
    bf16, as a backward that takes the forward's stored (bf16) output does; every other step is exact.
    (D_i enters dL/ds_ij and dL/dw_ij through the difference do.v_j - D_i, so the rounding of o reaches
    dq, dk, dWq and dWk but not dv.)"""
    q, k, v, wq, wk, do = (np.asarray(a, np.float64) for a in (q, k, v, wq, wk, do))
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    tau = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dwq, dwk = np.zeros_like(wq), np.zeros_like(wk)
    for b in range(B):
        for g in range(Hkv):
            K, V = k[b, g], v[b, g]
            phik = np.array([npmap_forward(K[j], wk[g]) for j in range(N)])
            dphik = np.zeros_like(phik)

            def sel_of(c, b=b, g=g):
                return [] if idx is None or idx.shape[-1] == 0 else [int(j) for j in idx[b, g, c]]

            for hh in range(G):
                h = g * G + hh
                for i in range(N):
                    soft, lin = routing_sets(i, N, w, C, sel_of)
                    qi, gi = q[b, h, i], do[b, h, i]
                    phiq = npmap_forward(qi, wq[h])
                    s = np.array([tau * (qi @ K[j]) for j in soft])
                    M = s.max() if len(soft) else 0.0
                    e = np.exp(s - M)                                   # e_ij e^-M
                    wl = np.array([phiq @ phik[j] for j in lin]) * math.exp(-M)  # w_ij e^-M
                    Z = e.sum() + wl.sum()
                    if Z <= 0:
                        continue
                    o = (e @ V[soft] if len(soft) else 0.0) + (wl @ V[lin] if len(lin) else 0.0)
                    o = o / Z
                    go = float(gi @ (_round_bf16(o) if d_from_output == "bf16" else o))
                    dphiq = np.zeros_like(phiq)
                    if len(soft):  # every index of a row's sets is distinct
                        p = e / Z
                        ds = p * (V[soft] @ gi - go)       # dL/ds_ij
                        dq[b, h, i] += tau * (ds @ K[soft])
                        dk[b, g, soft] += tau * np.outer(ds, qi)
                        dv[b, g, soft] += np.outer(p, gi)
                    if len(lin):
                        dw = (V[lin] @ gi - go) * math.exp(-M) / Z   # dL/dw_ij
                        dv[b, g, lin] += np.outer(wl / Z, gi)
                        dphiq += dw @ phik[lin]
                        dphik[lin] += np.outer(dw, phiq)
                    dx, dW = npmap_backward(qi, wq[h], dphiq)
                    dq[b, h, i] += dx
                    dwq[h] += dW
            for j in range(N):
                if np.any(dphik[j]):
                    dx, dW = npmap_backward(K[j], wk[g], dphik[j])
                    dk[b, g, j] += dx
                    dwk[g] += dW
    return dq, dk, dv, dwq, dwk
