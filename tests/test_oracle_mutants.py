"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (never in the product
code), builds it, and runs the pin suite against it in a child process; the suite must
fail.  The untouched source must pass the same suite.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "rr_oracle.c")

MUTANTS = {
    "logit scale drops 1/S": ("double *p) {\n    const double scale = 1.0 / ((double)S * sqrt((double)d));",
                              "double *p) {\n    const double scale = 1.0 / sqrt((double)d);"),
    "stride causality j < i": ("for (long j = 0; j <= i; ++j) {\n        const double *kb",
                               "for (long j = 0; j < i + (i == 0); ++j) {\n        const double *kb"),
    "head offset shifted": ("case RRO_HEAD_RR: return h % S;", "case RRO_HEAD_RR: return (h + 1) % S;"),
    "pool keeps first key only": ("for (int u = 0; u < S; ++u) {\n                const uint16_t *k = K + ((long)g * L + j * S + u) * d;",
                                  "for (int u = 0; u < 1; ++u) {\n                const uint16_t *k = K + ((long)g * L + j * S + u) * d;"),
    "block weight 1/B": ("rro_pool_keys(K, Hkv, L, d, S, Kbar);\n    const double w = (double)S / (double)B;",
                         "rro_pool_keys(K, Hkv, L, d, S, Kbar);\n    const double w = 1.0 / (double)B;"),
    "select strict >": ("if (cum >= thr)", "if (cum > thr)"),
    "tie-break reversed": ("return (u->J > v->J) - (u->J < v->J);", "return (u->J < v->J) - (u->J > v->J);"),
    "prefill drops diagonal key": ("k < (J + 1) * B && k <= t; ++k) {\n                    const uint16_t *kr",
                                   "k < (J + 1) * B && k < t + (k == 0); ++k) {\n                    const uint16_t *kr"),
    "GQA group by modulo": ("const int g = h / G;\n            const long r", "const int g = h % Hkv;\n            const long r"),
    "softmax without max shift uses wrong sign": ("p[j] = exp(p[j] - m);\n        l += p[j];\n    }\n    for (long j = 0; j <= i; ++j) p[j] /= l;",
                                                  "p[j] = exp(m - p[j]);\n        l += p[j];\n    }\n    for (long j = 0; j <= i; ++j) p[j] /= l;"),
    "transposed block accumulation": ("Arow[j / r] += w * p[j];", "Arow[(j / r) % (I + 1)] += w * p[i - j];"),
    "xattn main diagonal": ("Q + ((long)h * L + i * S + (S - 1 - u)) * d;", "Q + ((long)h * L + i * S + u) * d;"),
    "xattn drops 1/S": ("const double scale = 1.0 / ((double)S * sqrt((double)d));\n    const double w = (double)S / (double)B;\n    const long nrows = (long)(h_end - h_begin) * Nb;\n#pragma omp parallel\n    {\n        double *p = (double *)malloc(sizeof(double) * (size_t)Ns + 1);\n#pragma omp for schedule(dynamic, 1)",
                        "const double scale = 1.0 / sqrt((double)d);\n    const double w = (double)S / (double)B;\n    const long nrows = (long)(h_end - h_begin) * Nb;\n#pragma omp parallel\n    {\n        double *p = (double *)malloc(sizeof(double) * (size_t)Ns + 1);\n#pragma omp for schedule(dynamic, 1)"),
    "xattn stride causality j < i": ("for (long j = 0; j <= i; ++j) {\n                    double a = 0.0;", "for (long j = 0; j < i + (i == 0); ++j) {\n                    double a = 0.0;"),
    "diag cum_before reports cum_at": ("diag[1] = cum_before;", "diag[1] = cum;"),
    "diag threshold without tau": ("diag[3] = thr;", "diag[3] = T;"),
    "diag gap one past the cut": ("(kstar < n) ? buf[kstar - 1].a - buf[kstar].a",
                                  "(kstar + 1 < n) ? buf[kstar].a - buf[kstar + 1].a"),
}


def _run_pins(lib_path):
    env = dict(os.environ, RRO_LIB_OVERRIDE=lib_path)
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def _build(src_text, tmp_path, name):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", str(so),
                           str(c), "-lm"])
    return str(so)


def test_unmodified_oracle_passes(tmp_path):
    src = open(SRC).read()
    r = _run_pins(_build(src, tmp_path, "clean"))
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique/present: {name}"
    r = _run_pins(_build(src.replace(old, new), tmp_path, "mutant"))
    assert r.returncode != 0, f"pins did not catch: {name}"
