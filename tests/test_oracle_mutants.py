"""The pins reject a broken oracle.

Each case plants one plausible mistake in a copy of oracle/g2ref.c (compiled
on the CPU into a temporary library), then runs the pin suite against it
through G2REF_LIB: the suite must fail. The unmodified copy must pass. This
shows the pins are not tautological: a dropped term, a wrong sign, an
off-by-one or a wrong index anywhere in the definition or in its gradients is
caught.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "g2ref.c")

MUTANTS = {
    "window keeps W+1 keys": ("p - j >= window", "p - j > window"),
    "causal mask drops the query's own key": ("if (j > p) return 0;", "if (j >= p) return 0;"),
    "cap without its outer multiply": ("x = softcap * tanh(x / softcap);", "x = tanh(x / softcap);"),
    "cap of the raw logit without the inner divide": ("softcap * tanh(x / softcap)", "softcap * tanh(x)"),
    "softmax exponent with the wrong sign": ("exp(s[j] - m)", "exp(m - s[j])"),
    "query scale dropped": ("qs[c] = query_scale * widen(qrow[c]);", "qs[c] = widen(qrow[c]);"),
    "wrong GQA head mapping": ("{ return h / (H / Hkv); }", "{ return h % Hkv; }"),
    "lse without the max": ("*lse = m + log(l);", "*lse = log(l);"),
    "values mixed from the mirrored key": ("const uint16_t* vrow = v + ((b * S + j) * Hkv + g) * d;",
                                           "const uint16_t* vrow = v + ((b * S + (S - 1 - j)) * Hkv + g) * d;"),
    "mask before cap (a masked key gets -cap, not -inf)": (
        "s[j] = visible(p, j, window) ? sj : -INFINITY;",
        "s[j] = visible(p, j, window) ? sj : (softcap > 0.0 ? -softcap : -INFINITY);"),
    # gradients
    "backward: cap derivative dropped": ("dx *= 1.0 - t * t;", "dx *= 1.0;"),
    "backward: cap derivative at the capped logit": (
        "const double t = tanh(xl / softcap);", "const double t = tanh(tanh(xl / softcap));"),
    "backward: softmax gradient without the row term": (
        "double dx = w[j] * (x[j] - D);", "double dx = w[j] * x[j];"),
    "backward: dq without the query scale": (
        "dqrow[c] += query_scale * dx * widen(krow[c]);", "dqrow[c] += dx * widen(krow[c]);"),
    "backward: dv without the weight": (
        "dvrow[c] += w[j] * widen(dorow[c]);", "dvrow[c] += widen(dorow[c]);"),
    # gradients at chosen rows and keys
    "sampled backward: key terms without the row's D": (
        "const double dx = wl * (dw - row_D[(b * H + h) * T + i]) * cap_grad;",
        "const double dx = wl * dw * cap_grad;"),
    "sampled backward: cap derivative dropped": ("cap_grad = 1.0 - th * th;", "cap_grad = 1.0;"),
    "sampled backward: weight from the uncapped logit": (
        "const double wl = exp(sl - row_lse", "const double wl = exp(xl - row_lse"),
    "sampled backward: key seen one row late": (
        "if (!visible(i + q_offset, j, window)) continue;",
        "if (!visible(i + q_offset + 1, j, window)) continue;"),
    "sampled backward: one head of the group only": (
        "for (int64_t h = g * group; h < (g + 1) * group; ++h) {\n                    for (int64_t i = 0; i < T; ++i) {\n                        if (!visible",
        "for (int64_t h = g * group; h < g * group + 1; ++h) {\n                    for (int64_t i = 0; i < T; ++i) {\n                        if (!visible"),
}


def _build(tmp_path, name, old=None, new=None):
    src = open(SRC).read()
    if old is not None:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    c.write_text(src)
    lib = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-I",
                    os.path.join(ROOT, "oracle"), "-o", str(lib), str(c), "-lm"], check=True)
    return str(lib)


def _pins_pass(lib):
    env = dict(os.environ, G2REF_LIB=lib, OMP_NUM_THREADS="4")
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                          os.path.join(ROOT, "tests", "test_oracle_backward_pins.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return res.returncode == 0


def test_unmodified_copy_passes_the_pins(tmp_path):
    assert _pins_pass(_build(tmp_path, "control"))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_the_pins(tmp_path, name):
    old, new = MUTANTS[name]
    assert not _pins_pass(_build(tmp_path, "mutant", old, new)), name
