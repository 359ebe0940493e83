"""Power of the oracle pins: plant a plausible mistake in a copy of the
oracle's C source, build it, and require that at least one pin fails.

The mistakes are planted only in a temporary copy of the oracle, on the CPU.
"""
import os
import subprocess

import pytest

import oracle
from oracle import build as obuild
import pins

MUTANTS = [
    ("phi without the +1", "return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x : exp(x);"),
    ("phi with exp(-x)", "return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x + 1.0 : exp(-x);"),
    ("relu map keeps negative inputs", "if (g_phi_kind == 1) return x > 0.0 ? x : 0.0;",
     "if (g_phi_kind == 1) return x;"),
    ("exp map falls back to ELU + 1", "if (g_phi_kind == 2) return exp(x);",
     "if (g_phi_kind == 2) return phi_elu1(x);"),
    ("fp16 exponent bias off by one", "else x = ldexp(1024.0 + m, e - 25);",
     "else x = ldexp(1024.0 + m, e - 24);"),
    ("fp16 subnormals scaled as normals", "if (e == 0) x = ldexp((double)m, -24);",
     "if (e == 0) x = ldexp(1024.0 + m, -25);"),
    ("exclusive causal sum", "causal ? i + 1 : n", "causal ? i : n"),
    ("eps dropped", "(den + eps)", "(den)"),
    ("eps dropped (recurrent)", "double den = eps;", "double den = 0.0;"),
    ("GQA head mapping h % Hkv", "const int g = h / G;", "const int g = h % Hkv;"),
    ("normaliser accumulates phi(k)^2", "z[a] += pk[a];", "z[a] += pk[a] * pk[a];"),
    ("bf16 widened with wrong shift", "<< 16;", "<< 15;"),
    ("non-causal state never filled", "if (!causal) {", "if (0) {"),
    ("packed sequences lose their last token", "*len = (int64_t)cu[s + 1] - cu[s];",
     "*len = (int64_t)cu[s + 1] - cu[s] - (cu[s + 1] > cu[s]);"),
    ("decode reads state before update", "zg[a] += pk;", "zg[a] += 0.0 * pk;"),
    ("numerator sums V of the query row", "num[c] += a * load_elem(v, off(t0 + j,",
     "num[c] += a * load_elem(v, off(t0 + i,"),
    ("initial state ignored", "if (S0) memcpy(", "if (0) memcpy("),
    ("initial normaliser ignored", "if (z0) memcpy(", "if (0) memcpy("),
    ("state indexed by query head", "const int64_t sg = (int64_t)s * Hkv + g;",
     "const int64_t sg = (int64_t)s * Hkv + h % Hkv;"),
    # the selected-rows form only (8-space indentation is unique to it)
    ("rows: non-causal stops at the diagonal",
     "\n        const int64_t jend = causal ? i + 1 : n;",
     "\n        const int64_t jend = i + 1;"),
    ("rows: GQA head mapping h % Hkv", "\n        const int g = h / G;\n        double *pq",
     "\n        const int g = h % Hkv;\n        double *pq"),
    ("bwd: phi' of a negative input taken as 1", "return x > 0.0 ? 1.0 : exp(x);",
     "return x > 0.0 ? 1.0 : 1.0;"),
    ("bwd: normaliser term with the wrong sign (quadratic)", "const double hi = -go / den;",
     "const double hi = go / den;"),
    ("bwd: normaliser term dropped (recurrent)", "hs[i] = -go / den;", "hs[i] = 0.0 * go;"),
    ("bwd: dV weighted by da instead of a", "dv[off(t0 + j, g, Hkv, dvw, c)] += a * gi[c];",
     "dv[off(t0 + j, g, Hkv, dvw, c)] += da * gi[c];"),
    ("bwd: the dK/dV recurrence scans forward instead of in reverse",
     "for (int64_t j = n - 1; j >= 0; --j) {", "for (int64_t j = 0; j < n; ++j) {"),
    ("bwd: dK of a GQA group from its first query head only", "for (int h = g * G; h < (g + 1) * G; ++h) {\n                /* forward recurrence",
     "for (int h = g * G; h < g * G + 1; ++h) {\n                /* forward recurrence"),
    ("window one key too wide", "const int64_t jbeg = i - window + 1 > 0 ? i - window + 1 : 0;",
     "const int64_t jbeg = i - window > 0 ? i - window : 0;"),
    ("lagged state one token late", "const int64_t t = lag ? i - window : i;",
     "const int64_t t = lag ? i - window - 1 : i;"),
    ("rows: packed offsets ignored", "\n        seq_range(s, N, cu_seqlens, &t0, &n);\n        if (i < 0",
     "\n        seq_range(s, N, NULL, &t0, &n);\n        if (i < 0"),
]


def _build_mutant(tmp_path, idx, old, new):
    with open(obuild.SRC) as f:
        src = f.read()
    assert old in src, "mutation target not found: %r" % old
    assert src.count(old) == 1 or not old.startswith("\n"), "ambiguous target: %r" % old
    src = src.replace(old, new)
    c = tmp_path / ("mutant%d.c" % idx)
    so = tmp_path / ("mutant%d.so" % idx)
    c.write_text(src)
    subprocess.run(["gcc", "-std=c11", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                    str(c), "-lm"], check=True)
    return str(so)


@pytest.mark.parametrize("idx", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, monkeypatch, idx):
    name, old, new = MUTANTS[idx]
    path = _build_mutant(tmp_path, idx, old, new)
    monkeypatch.setattr(oracle, "_lib", None)
    monkeypatch.setattr(obuild, "build", lambda force=False: path)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError):  # a wrong value, or a rejected valid call
            failed.append(pin.__name__)
    monkeypatch.setattr(oracle, "_lib", None)
    assert failed, "no pin caught the planted mistake: %s" % name
