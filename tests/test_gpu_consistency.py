"""Local-global consistency of the library's own selection at the bench shape ([p1] "Self-Saliency
Score": a token the window attends to strongly is one later queries attend to as well): on one
(batch, KV group) slice of the Llama-3.2-1B-shaped layer (N = 16384, C = 512, k = 64), the share of
each chunk's kept tokens, as selected on the GPU by still_saliency + still_select_topk, that are also
in the chunk's top-k by the attention mass the token receives from every later query under full
causal softmax attention (fp64 numpy on the same bf16 inputs, averaged over the group's heads).
The oracle's selection on the same slice is scored the same way for comparison; the pages' 84.8 %
is measured on real data and is context only."""
import numpy as np
import pytest
import torch

from linear_attention_still_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def received_mass(q, k, tau, block=512):
    """Column sums of the causal softmax attention matrix (rows = queries), averaged over heads."""
    H, N, _ = q.shape
    recv = np.zeros(N)
    for h in range(H):
        for i0 in range(0, N, block):
            i1 = min(N, i0 + block)
            s = tau * q[h, i0:i1] @ k[:i1].T
            s[np.arange(i1 - i0)[:, None] < np.arange(i1)[None, :] - i0] = -np.inf
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            recv[:i1] += p.sum(axis=0) / H
    return recv


def overlap(sel, recv, C, k):
    out = []
    for c in range(sel.shape[0]):
        seg = recv[c * C:(c + 1) * C]
        top = np.lexsort((np.arange(C), -seg))[:k] + c * C  # mass descending, then position
        out.append(len(set(top.tolist()) & set(sel[c].tolist())) / k)
    return float(np.mean(out))


def test_gpu_selection_overlaps_global_attention_mass_at_bench_shape(oracle_mod):
    from linear_attention_still_b200 import _build
    _build.build()
    from linear_attention_still_b200 import still
    shape = WORKLOADS["llama32_1b_layer_n16k"]
    inp = make_inputs(shape, threads=8)
    q = torch.from_numpy(inp.q).to(torch.bfloat16).cuda()
    k = torch.from_numpy(inp.k).to(torch.bfloat16).cuda()
    d = still.dims_of(shape)
    r = torch.empty(shape.B, shape.Hkv, shape.N, device="cuda")
    rq = torch.empty(shape.B, shape.H, shape.N, device="cuda")
    idx = torch.empty(shape.B, shape.Hkv, shape.T, shape.k, dtype=torch.int32, device="cuda")
    still.still_saliency(d, q, k, r, rq)
    still.still_select_topk(d, r, idx)
    assert still.still_get_device_status() == 0
    sel_gpu = idx.cpu().numpy()[0, 0]
    G = shape.G
    qs = inp.q[0, :G].astype(np.float64)       # the heads of KV group 0
    ks = inp.k[0, 0].astype(np.float64)
    recv = received_mass(qs, ks, 1.0 / np.sqrt(shape.d))
    sl = shape.replace(B=1, H=G, Hkv=1)
    od = oracle_mod.Dims.of(sl)
    _, r_ora = oracle_mod.saliency(od, inp.q[:1, :G], inp.k[:1, :1])
    sel_ora = oracle_mod.topk(od, r_ora)[0, 0]
    ov_gpu = overlap(sel_gpu, recv, shape.C, shape.k)
    ov_ora = overlap(sel_ora, recv, shape.C, shape.k)
    print(f"1B 16K slice (b=0, g=0): overlap with the global top-k: GPU selection {ov_gpu:.3f}, oracle "
          f"selection {ov_ora:.3f}, chance {shape.k / shape.C:.3f}")
    assert ov_gpu > 2 * shape.k / shape.C
    assert abs(ov_gpu - ov_ora) < 0.02  # the GPU picks what the oracle picks, up to near-ties
