"""Second, independent oracle in pure numpy/Python for tiny inputs (N <= ~64).

TEST INFRASTRUCTURE.  Written separately from still_oracle.c, straight from the
prose of "STILL: Selecting Tokens for Intra-Layer Hybrid Attention to
Linearize LLMs" ([p1] jsqmd.com sections "Self-Saliency Score", "NP-Map",
"Chunk-Wise"; [p4] atlas.scime.ai "Approach"), with the same readings:
routing sets are built as Python sets and every sum is taken over them.
"""
from __future__ import annotations

import math

import numpy as np


def _softmax(x):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max())
    return e / e.sum()


def sigma(q_i, K, i, w, scale):
    """KL(p' || p) of token i: p over the band [i-w+1, i], p' without i."""
    band = list(range(max(0, i - w + 1), i + 1))
    if len(band) < 2:
        return math.inf
    logits = np.array([scale * float(np.dot(q_i, K[j])) for j in band])
    p = _softmax(logits)
    p_wo = _softmax(logits[:-1])
    return float(np.sum(p_wo * np.log(p_wo / p[:-1])))


def phi(x, W):
    f = _softmax(np.asarray(x, np.float64) @ np.asarray(W, np.float64))
    return np.linalg.norm(x) * f / np.linalg.norm(f)


def layer(q, k, v, wq, wk, w, C, kk, scale=None, idx_in=None):
    """Returns (o [B,H,N,d], r [B,Hkv,N], sel: dict (b,g,c) -> sorted list)."""
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    T = N // C
    m = w // C
    r = np.zeros((B, Hkv, N))
    sel = {}
    for b in range(B):
        for g in range(Hkv):
            if w > 0:
                for i in range(N):
                    r[b, g, i] = np.mean([sigma(q[b, g * G + hh, i], k[b, g], i, w, scale) for hh in range(G)])
            for c in range(T):
                if idx_in is not None:
                    sel[(b, g, c)] = sorted(int(j) for j in idx_in[b, g, c])
                    continue
                members = list(range(c * C, (c + 1) * C))
                ranked = sorted(members, key=lambda j: (-r[b, g, j], j))
                sel[(b, g, c)] = sorted(ranked[:kk])
    o = np.zeros((B, H, N, d))
    for b in range(B):
        for h in range(H):
            g = h // G
            for i in range(N):
                t = i // C
                if w == 0:
                    soft, lin = set(), set(range(i + 1))
                else:
                    soft = set(range(max(0, (t - m) * C), i + 1))
                    lin = set()
                    for c in range(0, t - m):
                        chosen = set(sel[(b, g, c)])
                        soft |= chosen
                        lin |= set(range(c * C, (c + 1) * C)) - chosen
                pq = phi(q[b, h, i], wq[h])
                weights = {}
                for j in soft:
                    weights[j] = math.exp(scale * float(np.dot(q[b, h, i], k[b, g, j])))
                for j in lin:
                    weights[j] = float(np.dot(pq, phi(k[b, g, j], wk[g])))
                den = sum(weights.values())
                o[b, h, i] = sum(wt * v[b, g, j] for j, wt in weights.items()) / den
    return o, r, sel
