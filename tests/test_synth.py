"""The seeded input generator shared by the oracle and the GPU tests: deterministic per seed,
batch items drawn independently (a subset of batches equals the same items of the whole draw),
heavy tokens as stated, bf16 rounding to nearest-even."""
import numpy as np

from linear_attention_still_b200.synth import Shape, make_inputs, round_to_bf16


def test_deterministic_and_batch_independent():
    sh = Shape(B=3, H=4, Hkv=2, N=300, d=16, D=8, w=64, C=64, k=4, dtype="f32")
    a, b = make_inputs(sh), make_inputs(sh)
    for n in ("q", "k", "v", "wq", "wk", "heavy"):
        np.testing.assert_array_equal(getattr(a, n), getattr(b, n))
    sub = make_inputs(sh, batches=[2, 0])
    np.testing.assert_array_equal(sub.q[0], a.q[2])
    np.testing.assert_array_equal(sub.v[1], a.v[0])
    np.testing.assert_array_equal(sub.wq, a.wq)
    other = make_inputs(sh, seed=1)
    assert not np.array_equal(other.q, a.q)


def test_heavy_tokens():
    sh = Shape(B=2, H=2, Hkv=1, N=1000, d=8, D=4, w=64, C=64, k=4, dtype="f32")
    inp = make_inputs(sh)
    assert inp.heavy.shape == (2, 10)  # 1 % of the tokens
    for b in range(2):
        hv = inp.heavy[b]
        assert len(set(hv.tolist())) == 10 and hv.min() >= 1 and hv.max() < 1000
        # heavy rows carry the x4 factor: their norms stand well above the median row
        norms = np.linalg.norm(inp.k[b, 0], axis=1)
        assert np.median(norms[hv]) > 2.5 * np.median(norms)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 3.1415926], dtype=np.float32)
    vals, bits = round_to_bf16(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa wins (1.0); 1 + 3*2^-8 rounds up to 1 + 2^-6
    np.testing.assert_array_equal(vals[:3], np.array([1.0, 1.0, 1.0 + 2.0 ** -6], dtype=np.float32))
    assert vals[3] == -2.5
    assert abs(vals[4] - 3.140625) < 1e-7
    np.testing.assert_array_equal((bits.astype(np.uint32) << 16).view(np.float32), vals)
    bf = make_inputs(Shape(B=1, H=2, Hkv=1, N=50, d=8, D=4, w=16, C=16, k=2))
    assert np.all((bf.q.view(np.uint32) & 0xFFFF) == 0)  # bf16 workloads hold bf16 values
