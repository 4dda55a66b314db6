"""The FMA-pipe exp2 used for part of the softmax exponentials (exp2_poly2 in tc_ptx.cuh): its relative
error against 2^x is checked on the GPU over the range the softmax feeds it (x <= 8, clamped at -127)."""
import os
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "linear_attention_still_b200",
                    "csrc")

CUDA_SRC = r'''
#include <torch/extension.h>
#include "tc_ptx.cuh"
__global__ void exp2_pairs(const float *x, float *y, int n) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (2 * i + 1 < n) {
        float2 r = still::tc::exp2_poly2(make_float2(x[2 * i], x[2 * i + 1]));
        y[2 * i] = r.x;
        y[2 * i + 1] = r.y;
    }
}
__global__ void packed_ops(const float *a, float *out) {
    // out: ffma2 (2), fadd2 (2), fmax3 (1)
    float2 f = still::tc::ffma2(make_float2(a[0], a[1]), make_float2(a[2], a[3]), make_float2(a[4], a[5]));
    float2 g = still::tc::fadd2(make_float2(a[0], a[1]), make_float2(a[2], a[3]));
    out[0] = f.x; out[1] = f.y; out[2] = g.x; out[3] = g.y;
    out[4] = still::tc::fmax3(a[0], a[6], a[7]);
}
torch::Tensor packed(torch::Tensor a) {
    auto out = torch::zeros({5}, a.options());
    packed_ops<<<1, 1>>>(a.data_ptr<float>(), out.data_ptr<float>());
    return out;
}
torch::Tensor run(torch::Tensor x) {
    auto y = torch::empty_like(x);
    int n = x.numel();
    exp2_pairs<<<(n / 2 + 255) / 256, 256>>>(x.data_ptr<float>(), y.data_ptr<float>(), n);
    return y;
}
'''


def test_exp2_poly_relative_error():
    from torch.utils.cpp_extension import load_inline
    build = tempfile.mkdtemp(prefix="still_exp2_")
    ext = load_inline(name="still_exp2_check",
                      cpp_sources="torch::Tensor run(torch::Tensor x);\ntorch::Tensor packed(torch::Tensor a);",
                      cuda_sources=CUDA_SRC, functions=["run", "packed"], extra_include_paths=[CSRC],
                      extra_cuda_cflags=["-gencode", "arch=compute_100a,code=sm_100a", "-O3"],
                      build_directory=build, verbose=False)
    a = torch.tensor([1.5, -2.0, 3.0, 0.25, 0.5, 4.0, -7.0, 2.5], device="cuda")
    got = ext.packed(a).cpu().numpy()
    np.testing.assert_allclose(got, [1.5 * 3.0 + 0.5, -2.0 * 0.25 + 4.0, 4.5, -1.75, 2.5], rtol=1e-6)
    x = np.concatenate([np.linspace(-125.0, 8.0, 200000), np.linspace(-2.0, 2.0, 100000),
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    x = x[: len(x) // 2 * 2]
    y = ext.run(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, rel.max()
    # at and below the clamp (masked scores are -inf) the result is ~2^-125: finite, positive, negligible
    z = ext.run(torch.tensor([-125.0, -125.7, -126.0, -127.0, -127.5, -200.0, -1e30, -float("inf")],
                             device="cuda")).cpu().numpy()
    assert np.isfinite(z).all() and (z > 0).all() and (z < 1e-37).all(), z
