"""The pins catch planted mistakes: each mutant is a copy of the oracle's C
source with one plausible slip, compiled on the CPU; at least one pin in
tests/test_oracle_pins.py must fail against it."""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "sa_oracle.c")

MUTANTS = {
    "relu dropped": ("const double relu = dot > 0.0 ? dot : 0.0;", "const double relu = dot;"),
    "one head weight for all heads": ("s += (double)w[(int64_t)q * H_I + j] * relu;",
                                      "s += (double)w[(int64_t)q * H_I] * relu;"),
    "last visible key dropped": ("const int64_t n = (int64_t)q_pos[q] + 1;",
                                 "const int64_t n = (int64_t)q_pos[q];"),
    "sequence offset ignored": ("const int64_t base = seq_off[q_seq[q]];", "const int64_t base = 0;"),
    "ties to the higher index": ("return (x->i > y->i) - (x->i < y->i);",
                                 "return (x->i < y->i) - (x->i > y->i);"),
    "output not in index order": ("qsort(row, (size_t)m, sizeof(int32_t), by_index);\n    for (int j = m; j < k; ++j)",
                                  ";\n    for (int j = m; j < k; ++j)"),
    "dynamic k: output not in index order": ("qsort(row, (size_t)m, sizeof(int32_t), by_index);\n    for (int j = m; j < k_max;",
                                             ";\n    for (int j = m; j < k_max;"),
    "scale dropped": ("z[j] = scale * dot;", "z[j] = dot;"),
    "GQA map modulo": ("const int g = h / G;\n    const uint16_t* Kb", "const int g = h % Hkv;\n    const uint16_t* Kb"),
    "ceil block map": ("if (t >= 0) mark[t / block] = 1;", "if (t >= 0) mark[(t + block - 1) / block] = 1;"),
    "causal strict": ("for (int64_t t = b0; t < b0 + block; ++t)\n        if (t <= q_pos[p] && t < S) keys[n++] = t;",
                      "for (int64_t t = b0; t < b0 + block; ++t)\n        if (t < q_pos[p] && t < S) keys[n++] = t;"),
    "ordered skipping: causal strict in the output": (
        "for (int64_t t = t0; t < t0 + block; ++t)\n          if (t <= q_pos[p] && t < S) keys[n++] = t;",
        "for (int64_t t = t0; t < t0 + block; ++t)\n          if (t < q_pos[p] && t < S) keys[n++] = t;"),
    "ordered skipping: causal strict in the shares": ("if (t > q_pos[p] || t >= S) continue;",
                                                       "if (t >= q_pos[p] || t >= S) continue;"),
    "value row of the wrong token": ("const uint16_t* vr = Vb + keys[j] * d;", "const uint16_t* vr = Vb + keys[0] * d;"),
    "routing weights not normalised": ("p[t] = exp(p[t] - m) / den;", "p[t] = exp(p[t] - m);"),
    "routing GQA map modulo": ("const int g = h / G;\n    const int64_t S = seq_len[b];",
                               "const int g = h % Hkv;\n    const int64_t S = seq_len[b];"),
    "routing from the last head only": ("for (int h = 0; h < Hq; ++h) acc += P[",
                                        "for (int h = Hq - 1; h < Hq; ++h) acc += P["),
    "routing logits unscaled": ("p[t] = scale * dot;", "p[t] = dot;"),
    "partial GQA map modulo": ("(int64_t)(h / G) * seq_len[b]) * d;", "(int64_t)(h % Hkv) * seq_len[b]) * d;"),
    "partial max in natural units": ("ml[2 * r] = l > 0.0 ? mz / log(2.0) : -INFINITY;",
                                     "ml[2 * r] = l > 0.0 ? mz : -INFINITY;"),
    "partial scale dropped": ("z[j] = dot * scale;", "z[j] = dot;"),
    "combine weight in natural units": ("const double wgt = pow(2.0, m - M);", "const double wgt = exp(m - M);"),
    "candidates gathered rank-minor": ("rows[(int64_t)b * n + (int64_t)r * k + j] =",
                                       "rows[(int64_t)b * n + (int64_t)j * N + r] ="),
    "selection keeps every rank's share": ("if (pos >= 0 && pos / k == rank) {", "if (pos >= 0) {"),
    "dynamic k: running sum in index order": ("      run += (double)all[j].s;\n      if (run >= target) {",
                                              "      run += (double)scores[(int64_t)q * ld + j];\n      if (run >= target) {"),
    "dynamic k: strict reach": ("      if (run >= target) {", "      if (run > target) {"),
    "dynamic k: total over the kept tokens only": ("    const double target = tau * total;",
                                                  "    const double target = tau * (total < 0 ? 0 : (double)all[0].s * 2);"),
    "dynamic k: cap one short": ("    if (m > k_max) m = k_max;\n    int32_t* row = idx + (int64_t)q * k_max;",
                                 "    if (m >= k_max) m = k_max - 1;\n    int32_t* row = idx + (int64_t)q * k_max;"),
    "proxy order ascending": ("if (x->hits != y->hits) return x->hits > y->hits ? -1 : 1;",
                              "if (x->hits != y->hits) return x->hits < y->hits ? -1 : 1;"),
    "proxy ties to the higher block": ("return (x->id > y->id) - (x->id < y->id);",
                                       "return (x->id < y->id) - (x->id > y->id);"),
    "proxy counts padding entries": ("if (t >= 0 && t < S) hits[t / block] += 1;",
                                     "if (t >= -1 && t < S) hits[t / block] += 1;"),
    "skip rule not strict": ("if (c < tau && N == n_steps)", "if (c <= tau && N == n_steps)"),
    "skip without the steps in flight": ("N = (n + 1 + lag < n_steps) ? n + 1 + lag : n_steps;",
                                         "N = (n + 1 < n_steps) ? n + 1 : n_steps;"),
    "progressive score of the first row only": ("for (int r = 0; r < rows; ++r) {\n        const double s = share",
                                                "for (int r = 0; r < 1; ++r) {\n        const double s = share"),
    "share against the mass before the step": ("share[(int64_t)r * n_steps + n] = L > 0.0 ? a / L : INFINITY;",
                                               "share[(int64_t)r * n_steps + n] = L > a ? a / (L - a) : INFINITY;"),
    "unseen row counts as no gain": ("share[(int64_t)r * n_steps + n] = L > 0.0 ? a / L : INFINITY;",
                                     "share[(int64_t)r * n_steps + n] = L > 0.0 ? a / L : 0.0;"),
    "steps of one block": ("for (int b2 = 2 * n; b2 < 2 * n + 2 && b2 < nT; ++b2) {",
                           "for (int b2 = 2 * n; b2 < 2 * n + 1 && b2 < nT; ++b2) {"),
    "output over N blocks instead of N steps": ("for (int b2 = 0; b2 < 2 * N && b2 < nT; ++b2) {",
                                                "for (int b2 = 0; b2 < N && b2 < nT; ++b2) {"),
    "routing drops the last token": ("for (int64_t t = 0; t < seq_len[b]; ++t) {\n      double acc",
                                     "for (int64_t t = 0; t + 1 < seq_len[b]; ++t) {\n      double acc"),
}

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {name}"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(mut), "-lm"])
    saved = oracle._lib
    oracle._lib = oracle.load(str(so))
    failed = []
    try:
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
    finally:
        oracle._lib = saved
    assert failed, f"no pin catches the mutant '{name}'"
