"""Local-global consistency of the per-chunk selection (the pages' motivation for routing per chunk:
[p1] "Self-Saliency Score" -- tokens that matter locally also matter globally): on synthetic inputs,
the overlap between each chunk's top-k by the Self-Saliency Score (or by the diagonal-only router)
and its top-k by the attention mass the token receives from every later query under full causal
softmax attention.  CPU only (fp64 oracle scores, numpy attention); prints the overlaps."""
import numpy as np
import pytest

from linear_attention_still_b200.synth import Shape, make_inputs


def _received_mass(q, k, tau):
    """Column sums of the causal softmax attention matrix, averaged over the query heads."""
    N = k.shape[0]
    mask = np.tril(np.ones((N, N), dtype=bool))
    recv = np.zeros(N)
    for h in range(q.shape[0]):
        s = tau * q[h] @ k.T
        s[~mask] = -np.inf
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        recv += p.sum(axis=0) / q.shape[0]
    return recv


def _overlap(sel, recv, C, k):
    out = []
    for c in range(sel.shape[0]):
        seg = recv[c * C:(c + 1) * C]
        top = np.lexsort((np.arange(C), -seg))[:k] + c * C  # mass descending, then position
        out.append(len(set(top.tolist()) & set(sel[c].tolist())) / k)
    return float(np.mean(out))


@pytest.mark.parametrize("N,C,k,w", [(1024, 64, 8, 64), (1024, 128, 16, 256)])
def test_selection_overlaps_global_attention_mass(oracle_mod, N, C, k, w):
    sh = Shape(B=1, H=4, Hkv=1, N=N, d=64, D=64, w=w, C=C, k=k, dtype="f32")
    inp = make_inputs(sh)
    d = oracle_mod.Dims.of(sh)
    recv = _received_mass(inp.q[0].astype(np.float64), inp.k[0, 0].astype(np.float64), 1 / np.sqrt(sh.d))
    _, r_sal = oracle_mod.saliency(d, inp.q, inp.k)
    r_diag = oracle_mod.diagonal_score(d, inp.q, inp.k)
    ov_sal = _overlap(oracle_mod.topk(d, r_sal)[0, 0], recv, C, k)
    ov_diag = _overlap(oracle_mod.topk(d, r_diag)[0, 0], recv, C, k)
    print(f"N={N} C={C} k={k} w={w}: overlap with the global top-k: saliency {ov_sal:.3f}, "
          f"diagonal router {ov_diag:.3f}, chance {k / C:.3f}")
    # both routers pick far more of the globally attended tokens than a random choice would
    assert ov_sal > 2 * k / C and ov_diag > 2 * k / C
