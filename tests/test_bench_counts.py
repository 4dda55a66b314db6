"""CPU checks of bench.py's measurement arithmetic: the softmax-set sizes behind the merge FLOP and
exponential counts and the decode bytes per step against the oracle's own routing sets, the w = 0 FLOP count
against an enumeration of its pairs, the --keep shapes, and the traffic lookup from a profile summary (used
only while the kernel sources match its hashes) with the committed summaries' blocks."""
import hashlib
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from linear_attention_still_b200.synth import Shape  # noqa: E402
from oracle import backward  # noqa: E402


def _soft_sets(shape):
    """|Soft(i)| from the oracle backward's routing sets (selection: the first k rows of each chunk)."""
    def sel(c):
        return list(range(c * shape.C, c * shape.C + shape.k))
    return np.array([len(backward.routing_sets(i, shape.N, shape.w, shape.C, sel)[0]) for i in range(shape.N)])


@pytest.mark.parametrize("shape", [Shape(B=1, H=4, Hkv=2, N=1000, d=64, D=64, w=128, C=128, k=16),
                                   Shape(B=2, H=2, Hkv=1, N=777, d=32, D=16, w=256, C=64, k=8),
                                   Shape(B=1, H=2, Hkv=1, N=300, d=32, D=16, w=0, C=64, k=0),
                                   Shape(B=1, H=2, Hkv=1, N=50, d=32, D=16, w=64, C=64, k=8)])
def test_soft_set_sizes_and_merge_flops(shape):
    sizes = _soft_sets(shape)
    np.testing.assert_array_equal(bench.soft_sizes(shape), sizes)
    want = shape.B * shape.H * sum(4 * shape.d * n + 4 * shape.d * shape.D + 2 * shape.D for n in sizes)
    assert bench.merge_flops(shape) == want
    assert bench.merge_exps(shape) == shape.B * shape.H * int(sizes.sum())


def test_exp_pipe_diagnostic():
    shape = Shape(B=1, H=32, Hkv=8, N=16384, d=64, D=64, w=512, C=512, k=64)
    assert bench.exp_pipe_diag(shape, None) is None
    diag = bench.exp_pipe_diag(shape, 0.5, {"sm_mhz": 1000.0}, sms=100)
    assert diag["peak"] == 16 * 100 * 1000.0 * 1e6
    assert diag["achieved"] == pytest.approx(bench.merge_exps(shape) / 0.5e-3)
    assert diag["frac"] == pytest.approx(diag["achieved"] / diag["peak"])
    assert diag["flops_per_exp"] > 4 * shape.d  # 4d per pair plus the per-row linear-branch terms
    # without a clock record the maximum clock is assumed; at d = 64 the exponentials take longer
    # than the tensor work at the measured bf16 peak
    d2 = bench.exp_pipe_diag(shape, 0.5, None)
    assert d2["sm_mhz"] == 1965.0
    assert d2["ms_at_exp_peak"] > bench.merge_flops(shape) / 1653.3e12 * 1e3


def test_decode_bytes_count_the_softmax_rows():
    shape = Shape(B=3, H=8, Hkv=2, N=0, d=64, D=32, w=128, C=64, k=8, decode_steps=1)
    for pos in (0, 63, 64, 191, 192, 500, 1023):
        full = shape.replace(N=pos + 1)
        rows = len(backward.routing_sets(pos, pos + 1, shape.w, shape.C,
                                         lambda c: list(range(c * shape.C, c * shape.C + shape.k)))[0])
        want = shape.B * shape.Hkv * (rows * 2 * shape.d * 2 + shape.D * shape.d * 4 + shape.D * 4) + \
            shape.B * shape.H * 2 * shape.d * 2
        assert bench.decode_step_bytes(full, pos) == want, pos


def test_keep_shapes():
    class A:
        workload = "llama32_1b_layer_n16k"
        keep = "all"
    s = bench.workload_shape(A)
    assert s.k == s.C
    A.keep = "none"
    assert bench.workload_shape(A).k == 0
    A.keep = "config"
    assert bench.workload_shape(A).k == 64
    A.keep = "window"  # every query's window reaches token 0: exact causal softmax attention, no selection
    s = bench.workload_shape(A)
    assert s.k == 0 and s.w % s.C == 0 and s.w >= s.N
    assert (bench.soft_sizes(s) == np.arange(s.N) + 1).all()
    assert bench.merge_flops(s) == bench.merge_flops(bench.workload_shape(type("B", (), {"workload": A.workload,
                                                                                           "keep": "all"})))


@pytest.mark.parametrize("shape", [Shape(B=1, H=4, Hkv=2, N=300, d=64, D=64, w=0, C=128, k=0),
                                   Shape(B=2, H=2, Hkv=1, N=77, d=32, D=16, w=0, C=32, k=0)])
def test_nowin_flops_by_counting(shape):
    """The w = 0 FLOP count against an explicit enumeration of the (query, key) pairs of the
    intra-chunk causal tiles (query i sees the keys of its own chunk up to itself)."""
    pairs = sum(1 for i in range(shape.N) for j in range(shape.N) if j // shape.C == i // shape.C and j <= i)
    d, D = shape.d, shape.D
    want = (shape.B * shape.H * (pairs * 2 * (D + d) + shape.N * (4 * d * D + 2 * D))
            + shape.B * shape.Hkv * shape.N * 4 * d * D)
    assert bench.nowin_flops(shape) == want


def test_committed_profiles_name_known_workloads_and_sources():
    """Every machine-readable block under profiles/ names a workload of the synthetic set, a positive
    byte count and digests of source files that exist (whether they still match is the bench's call)."""
    import glob
    from linear_attention_still_b200.synth import WORKLOADS
    seen = 0
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for line in open(path):
            if not line.startswith("    ") or line.startswith("     "):
                continue
            key, _, val = line.strip().partition(": ")
            if key == "workload":
                assert val in WORKLOADS, (path, val)
                seen += 1
            elif key == "traffic_bytes_per_step":
                assert int(val) > 0, path
            elif key == "source_sha256":
                for item in val.split():
                    name, _, digest = item.partition("=")
                    assert len(digest) == 16, (path, item)
                    assert os.path.exists(os.path.join(ROOT, "linear_attention_still_b200", "csrc", name)), (path, name)
    assert seen >= 4


def test_traffic_lookup_follows_source_hashes(tmp_path, monkeypatch):
    csrc = tmp_path / "linear_attention_still_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "a.cu").write_bytes(b"kernel one")
    digest = hashlib.sha256(b"kernel one").hexdigest()[:16]
    (tmp_path / "profiles" / "merge_tc_x.md").write_text(
        "# summary\n\n    workload: wl\n    traffic_bytes_per_step: 12345\n"
        f"    source_sha256: a.cu={digest}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("wl") == 12345
    assert bench.profiled_traffic("other") is None
    (csrc / "a.cu").write_bytes(b"kernel two")  # the kernel changed since the capture
    assert bench.profiled_traffic("wl") is None


@pytest.mark.parametrize("workload,extra,metric", [
    ("still_f32_b1_h2_n512", [], bench.METRIC),
    ("still_f32_b1_h2_n512", ["--pass", "backward"], bench.METRIC_BACKWARD),
    ("still_f32_decode_b1_ctx512", [], bench.METRIC_DECODE),
])
def test_reference_arm_line(tmp_path, workload, extra, metric):
    """`bench.py --impl reference` on the small fp32 workloads (prefill, its backward, decode): one
    JSON line with the contract's keys and the pass's metric, the oracle's own throughput as value,
    cpu_baseline and e2e carrying the same number."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        workload, "--steps", "3", "--warmup", "1", *extra],
                       capture_output=True, text=True, timeout=600, cwd=tmp_path)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 1
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == workload and line["metric"] == metric


@pytest.mark.parametrize("N,m", [(16384, 64), (16384, 704), (16384, 4352), (16384, 16384), (512, 512),
                                 (65536, 128), (1000, 640)])
def test_row_runs_are_an_unbiased_position_sample(N, m):
    """The CPU baseline's row sample: m distinct positions of [0, N) in runs of 64 consecutive ones,
    with mean position (N - 1)/2 up to one run's rounding, so a per-row cost linear in the position
    sums to the whole slice's when scaled by N/m."""
    pos = bench._row_runs(N, m)
    assert len(pos) == m and len(set(pos.tolist())) == m
    assert pos.min() >= 0 and pos.max() < N
    run = min(64, m)
    runs = pos.reshape(-1, run)
    assert (np.diff(runs, axis=1) == 1).all()
    assert abs(pos.mean() - (N - 1) / 2) <= max(1.0, 0.01 * N)
    cost = lambda p: 3.0 + 0.5 * p  # noqa: E731  (constant plus a term linear in the position)
    full = cost(np.arange(N)).sum()
    assert cost(pos).sum() * N / m == pytest.approx(full, rel=0.01)
