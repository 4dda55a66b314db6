"""The oracle's pins catch plausible mistakes: each mutant below is a copy of oracle/still_oracle.c
with one such mistake planted (a dropped term, a wrong sign, index or direction, a transposed
operand, an off-by-one chunk), built with gcc into a temporary library and run against the pins of
tests/test_oracle_pins.py in a child process; likewise copies of oracle/backward.py against the
pins of tests/test_oracle_backward.py.  Every mutant must fail at least one pin, and the
unmodified source, built and run the same way, must pass them all.  Nothing here touches the
oracle's own files or build."""
import os
import subprocess
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "still_oracle.c")

# name: (what the mistake is, text in still_oracle.c, replacement)
MUTANTS = {
    "kl_direction": ("saliency: KL(p || p') term by term instead of KL(p' || p)",
                     "kl += exp(lp2) * (lp2 - lp);", "kl += exp(lp) * (lp - lp2);"),
    "band_too_long": ("saliency: a band of w + 1 keys", "int lo = i - s->w + 1;", "int lo = i - s->w;"),
    "group_sum": ("saliency: the group score summed over the heads instead of averaged",
                  "acc += sg[((size_t)b * s->H + g * G + hh) * s->N + i];\n"
                  "                    r[((size_t)b * s->Hkv + g) * s->N + i] = acc / G;",
                  "acc += sg[((size_t)b * s->H + g * G + hh) * s->N + i];\n"
                  "                    r[((size_t)b * s->Hkv + g) * s->N + i] = acc;"),
    "tie_break": ("top-k: ties go to the higher position", "return a < b;", "return a > b;"),
    "npmap_norm": ("NP-Map: the input's norm not put back", "phi[c] = nx * phi[c] / nf;", "phi[c] = phi[c] / nf;"),
    "npmap_transposed": ("NP-Map: W read transposed", "y += x[a] * W[(size_t)a * D + c];",
                         "y += x[a] * W[(size_t)c * d + a];"),
    "window_short": ("routing: the window one chunk shorter (a chunk decided one chunk early)",
                     "int lo = (t - m) * s->C;", "int lo = (t - m + 1) * s->C;"),
    "linear_unshifted": ("merge: the linear weights left out of the shared shift", "wgt = dot * exp(-M);",
                         "wgt = dot;"),
    "linear_not_in_denominator": ("merge: the linear weights missing from the normaliser",
                                  "for (int x = 0; x < d; ++x) num[x] += wgt * vj[x];\n        den += wgt;",
                                  "for (int x = 0; x < d; ++x) num[x] += wgt * vj[x];\n        "
                                  "if (route[j] == 1) den += wgt;"),
    "wrong_group": ("merge: query head h mapped to KV head h mod Hkv instead of h / G",
                    "int G = s->H / s->Hkv, g = h / G, d = s->d, D = s->D;",
                    "int G = s->H / s->Hkv, g = h % s->Hkv, d = s->d, D = s->D;"),
    "state_keeps_selected": ("linear state: the kept tokens folded in as well", "            if (sel) continue;\n",
                             ""),
    "state_late": ("linear state: one chunk late", "int last = s->w == 0 ? t - 1 : t - m - 1;",
                   "int last = s->w == 0 ? t - 1 : t - m - 2;"),
    "decode_late": ("decode: a chunk decided one chunk late",
                    "if (p % C == C - 1 && t - m >= 0) {\n                int c = t - m;",
                    "if (p % C == C - 1 && t - m - 1 >= 0) {\n                int c = t - m - 1;"),
    "decode_folds_kept": ("decode: the kept tokens folded into the linear state too", "if (is_sel) continue;",
                          "(void)is_sel;"),
    "diagonal_sign": ("diagonal router: the logit's sign flipped", "acc += s->scale * dot;",
                      "acc -= s->scale * dot;"),
}

_RUNNER = """
import sys
sys.path.insert(0, {root!r})
import pytest
import oracle.oracle as om
om.build = lambda force=False: {lib!r}
om._lib = None
sys.exit(pytest.main(["-q", "-x", "-p", "no:cacheprovider", {pins!r}]))
"""


def _start(tmp_path, name, source):
    c_path = tmp_path / f"{name}.c"
    so_path = tmp_path / f"{name}.so"
    c_path.write_text(source)
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", str(so_path), str(c_path), "-lm", "-lpthread"])
    code = _RUNNER.format(root=ROOT, lib=str(so_path), pins=os.path.join(ROOT, "tests", "test_oracle_pins.py"))
    env = dict(os.environ, OMP_NUM_THREADS="1")
    return subprocess.Popen([sys.executable, "-c", code], cwd=str(tmp_path), env=env, stdout=subprocess.PIPE,
                            stderr=subprocess.STDOUT, text=True)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with open(SRC) as f:
        original = f.read()
    jobs = {"unmodified": original}
    for name, (_, old, new) in MUTANTS.items():
        assert original.count(old) == 1, f"{name}: the mutated text must occur exactly once in still_oracle.c"
        jobs[name] = original.replace(old, new)
    results = {}
    pending = list(jobs.items())
    running = []
    width = max(1, min(len(pending), (os.cpu_count() or 2) // 2))
    while pending or running:
        while pending and len(running) < width:
            name, source = pending.pop(0)
            running.append((name, _start(tmp_path, name, source)))
        name, proc = running.pop(0)
        out, _ = proc.communicate(timeout=900)
        results[name] = (proc.returncode, out)
    rc, out = results.pop("unmodified")
    assert rc == 0, "the unmodified oracle, built the same way, must pass every pin:\n" + out[-3000:]
    survivors = [name for name, (rc, _) in results.items() if rc != 1]
    assert not survivors, {name: (MUTANTS[name][0], results[name][1][-1500:]) for name in survivors}


# name: (what the mistake is, text in oracle/backward.py, replacement)
BACKWARD_MUTANTS = {
    "ds_without_row_term": ("softmax logits: dL/ds without the - <g, o> term", "ds = p * (V[soft] @ gi - go)",
                            "ds = p * (V[soft] @ gi)"),
    "dk_without_scale": ("softmax keys: dk without the logit scale", "dk[b, g, soft] += tau * np.outer(ds, qi)",
                         "dk[b, g, soft] += np.outer(ds, qi)"),
    "dw_unshifted": ("linear weights: dL/dw without the shared shift", "dw = (V[lin] @ gi - go) * math.exp(-M) / Z",
                     "dw = (V[lin] @ gi - go) / Z"),
    "dv_linear_unnormalised": ("linear values: dv without 1/Z", "dv[b, g, lin] += np.outer(wl / Z, gi)",
                               "dv[b, g, lin] += np.outer(wl, gi)"),
    "linear_keys_dropped": ("linear keys: no gradient into phi(k)", "dphik[lin] += np.outer(dw, phiq)",
                            "pass"),
    "npmap_norm_term": ("NP-Map backward: the norm's own gradient dropped",
                        "dx = W @ dy + (dn * x / n if n > 0 else 0.0)", "dx = W @ dy"),
    # (Dropping the softmax Jacobian's mean term f.df would be no mistake here: the gradient that
    # reaches f through u = f / ||f|| is orthogonal to f, so that term is zero.)
    "npmap_projection": ("NP-Map backward: the normalisation's projection dropped",
                         "df = (du - u * float(u @ du)) / nf", "df = du / nf"),
    "npmap_dW_transposed": ("NP-Map backward: dW as the outer product the wrong way round", "dW = np.outer(x, dy)",
                            "dW = np.outer(x, dy)[:, ::-1]"),
}

_BACKWARD_RUNNER = """
import sys, types
sys.path.insert(0, {root!r})
import pytest
import oracle
mod = types.ModuleType("oracle.backward")
mod.__file__ = {path!r}
exec(compile(open({path!r}).read(), {path!r}, "exec"), mod.__dict__)
sys.modules["oracle.backward"] = mod
oracle.backward = mod
sys.exit(pytest.main(["-q", "-x", "-p", "no:cacheprovider", {pins!r}]))
"""


def test_every_planted_backward_mistake_fails_a_pin(tmp_path):
    src_path = os.path.join(ROOT, "oracle", "backward.py")
    with open(src_path) as f:
        original = f.read()
    jobs = {"unmodified": original}
    for name, (_, old, new) in BACKWARD_MUTANTS.items():
        assert original.count(old) == 1, f"{name}: the mutated text must occur exactly once in backward.py"
        jobs[name] = original.replace(old, new)
    procs = {}
    for name, source in jobs.items():
        path = tmp_path / f"{name}.py"
        path.write_text(source)
        code = _BACKWARD_RUNNER.format(root=ROOT, path=str(path),
                                       pins=os.path.join(ROOT, "tests", "test_oracle_backward.py"))
        procs[name] = subprocess.Popen([sys.executable, "-c", code], cwd=str(tmp_path), stdout=subprocess.PIPE,
                                       stderr=subprocess.STDOUT, text=True)
    results = {name: (p.wait(timeout=900), p.stdout.read()) for name, p in procs.items()}
    rc, out = results.pop("unmodified")
    assert rc == 0, "the unmodified backward, loaded the same way, must pass every pin:\n" + out[-3000:]
    survivors = [name for name, (rc, _) in results.items() if rc != 1]
    assert not survivors, {name: (BACKWARD_MUTANTS[name][0], results[name][1][-1500:]) for name in survivors}
