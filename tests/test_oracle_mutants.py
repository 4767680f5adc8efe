"""Plants plausible mistakes in a scratch copy of the oracle (on the CPU) and
checks that the pin suite rejects every one of them.  The committed oracle is
never modified; each mutant is compiled into its own temporary tree."""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (text in the oracle, its mutated form, what the mistake is[, file under oracle/
# when it is not the C source])
MUTANTS = [
    ("double wj = a1[j] - lambda * a2[j];", "double wj = a1[j] + lambda * a2[j];", "lambda sign"),
    ("1.0 / sqrt((double)d)", "1.0 / sqrt((double)(2 * d))", "scale over the full head width"),
    ("diff_attention_row(qrow, qrow + d, kb, kb + d", "diff_attention_row(qrow, qrow, kb, kb + d", "branch-2 query half"),
    ("diff_attention_row(qrow, qrow + d, kb, kb + d", "diff_attention_row(qrow, qrow + d, kb, kb", "branch-2 key half"),
    ("int64_t n_keys = causal ? (int64_t)i + 1 : (int64_t)N;\n        const float *qrow",
     "int64_t n_keys = causal ? (int64_t)i : (int64_t)N;\n        const float *qrow", "causal diagonal"),
    ("int g = (2 * p) / group;", "int g = p / group;", "GQA head mapping"),
    ("const float *qb = q + ((int64_t)b * N + i) * tok_q + (int64_t)(2 * p + 1) * d;",
     "const float *qb = q + ((int64_t)b * N + i) * tok_q + (int64_t)(2 * p) * d;", "V2 pair member"),
    ("const float *qa = q + ((int64_t)b * Hq + 2 * p) * d;", "const float *qa = q + ((int64_t)b * Hq + p) * d;", "decode query head"),
    ("double inv_rms = 1.0 / sqrt(ss / (double)dv + eps);", "double inv_rms = 1.0 / sqrt(ss + eps);", "RMS mean"),
    ("o[c] = o[c] * inv_rms * gc * (1.0 - lambda_init);", "o[c] = o[c] * inv_rms * gc * lambda_init;", "post-norm scale"),
    ("lambda_out[h] = exp(dot1) - exp(dot2) + linit;", "lambda_out[h] = exp(dot1) + exp(dot2) + linit;", "lambda re-parameterisation sign"),
    ("return 0.8 - 0.6 * exp(-0.3 * (double)(layer - 1));", "return 0.8 - 0.6 * exp(-0.3 * (double)(layer));", "layer base"),
    ("x[j] = exp(x[j] - m);", "x[j] = exp(x[j]);", "softmax without the max shift"),
    ("for (int c = 0; c < dv; ++c) o[c] += wj * (double)vj[c];", "for (int c = 0; c < dv; ++c) o[c] += a1[j] * (double)vj[c];", "second map dropped"),
    ("if (j != pos) ss += w[j] * w[j];", "ss += w[j] * w[j];", "signal counted as noise in the ratio"),
    ("sqrt(ss / (double)(n - 1))", "sqrt(ss / (double)n)", "noise mean over every position"),
    ("? n - (int64_t)window : 0;", "? n - (int64_t)window + 1 : 0;", "window one key short"),
    ("        vb += first * tok_v;\n        if (w) w += first;\n        diff_attention_row(qrow",
     "        if (w) w += first;\n        diff_attention_row(qrow", "window not applied to values (V1)"),
    ("        const int64_t first = window_start(len, window);\n        kb += first * tok_kv;",
     "        const int64_t first = 0;\n        kb += first * tok_kv;", "window ignored in V2 decode"),
    ("        dlam -= a2[j] * dp;", "        dlam += a2[j] * dp;", "backward: lambda gradient sign"),
    ("const double ds = a[j] * (dp - D) * inv_sqrt_d;", "const double ds = a[j] * dp * inv_sqrt_d;",
     "backward: softmax Jacobian without the row term"),
    ("const double coef = r == 0 ? 1.0 : -lambda;", "const double coef = r == 0 ? 1.0 : lambda;",
     "backward: branch-2 upstream sign"),
    ("gro[c] = (cpost / r) * (gc * (double)dy[c] - o[c] * gdo / ((double)dv * r * r));",
     "gro[c] = (cpost / r) * (gc * (double)dy[c]);", "backward: norm Jacobian without the RMS term"),
    ("        for (int c = 0; c < dv; ++c) dvj[c] += wj * dout[c];",
     "        for (int c = 0; c < dv; ++c) dvj[c] += a1[j] * dout[c];", "backward: dV from map 1 only"),
    ("            dlk2[h * dim + c] = -e2 * (double)lq2[h * dim + c];",
     "            dlk2[h * dim + c] = -e2 * (double)lk2[h * dim + c];", "backward: lambda vector swap"),
    ("dot2 += (double)lq2[(size_t)h * dim + c] * (double)lk2[(size_t)h * dim + c];",
     "dot2 += (double)lq2[(size_t)h * dim + c] * (double)lk1[(size_t)h * dim + c];",
     "lambda: second product with the first key vector"),
    ("diff_attention_row(qa, qa + d, kb, kb, tok_kv, vb, tok_kv, len - first, d, d,",
     "diff_attention_row(qa, qa, kb, kb, tok_kv, vb, tok_kv, len - first, d, d,",
     "V2 decode: both branches from the pair's first head"),
    ("int p = (int)(r % P), b = (int)(r / P), g = (2 * p) / group;",
     "int p = (int)(r % P), b = (int)(r / P), g = p / group;", "V2 decode: GQA head mapping"),
    ("diff_attention_row(qr, qr + d, kb, kb + d, tok_k, vb, tok_v, len - first, d, dv,",
     "diff_attention_row(qr, qr + d, kb, kb, tok_k, vb, tok_v, len - first, d, dv,",
     "V1 decode: branch-2 key half"),
    ("lambda[h], a1, a2, NULL, o);\n        if (apply_norm) head_rms_norm(",
     "lambda[h], a1, a2, NULL, o);\n        if (0) head_rms_norm(", "V1 decode: norm skipped"),
    ("const int64_t qb = qa + d;", "const int64_t qb = qa;",
     "V2 backward: both branches from the pair's first head"),
    ("const int g = (2 * p) / group;", "const int g = p / group;", "V2 backward: GQA head mapping"),
    ("dkj[c] += ds * (double)qr[c];", "dkj[c] += ds * (double)kj[c];",
     "backward: dK from the key instead of the query"),
    ("double *dqr = r == 0 ? dq1 : dq2;", "double *dqr = r == 0 ? dq1 : dq1;",
     "backward: branch-2 dQ into branch 1's half"),
    ("dnorm_weight[c] += (double)dy[c] * o[c] * cpost / r;",
     "dnorm_weight[c] += (double)dy[c] * o[c] / r;", "backward: gain gradient without (1 - lambda_init)"),
    ("const int64_t first = window_start(n_keys, window);\n                const int64_t tq",
     "const int64_t first = window_start(n_keys, 0);\n                const int64_t tq",
     "V1 backward: window ignored"),
    ("    for (int64_t j = 0; j < n; ++j) x[j] /= s;", "    (void)s;",
     "softmax not normalised"),
    ("double inv_rms = 1.0 / sqrt(ss / (double)dv + eps);",
     "double inv_rms = 1.0 / (sqrt(ss / (double)dv) + eps);", "RMS norm: epsilon outside the root"),
    ("return 0.8 - 0.6 * exp(-0.3 * (double)(layer - 1));",
     "return 0.8 - 0.6 * exp(-0.03 * (double)(layer - 1));", "lambda_init decay rate"),
    # the output projection is numpy arithmetic in oracle.py
    ("return o.reshape(t.size, P * d) @ w", "return o.reshape(t.size, P * d) @ w.T",
     "output projection: O_W transposed", "oracle.py"),
    ("return o.reshape(t.size, P * d) @ w",
     "return o.reshape(t.size, P, d).transpose(0, 2, 1).reshape(t.size, P * d) @ w",
     "output projection: channel-major flattening of the pair rows", "oracle.py"),
]


def _run_mutant(tmp_root, n, before, after, fname="diffattn_oracle.c"):
    src = open(os.path.join(ROOT, "oracle", fname)).read()
    assert before in src, before
    d = os.path.join(tmp_root, "m%d" % n)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    with open(os.path.join(d, "oracle", fname), "w") as f:
        f.write(src.replace(before, after, 1))
    os.makedirs(os.path.join(d, "tests"))
    for name in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(d, "tests", name))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    os.symlink(os.path.join(ROOT, "differential_attention_sm_b200"),
               os.path.join(d, "differential_attention_sm_b200"))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join("tests", "test_oracle_pins.py")],
                       cwd=d, capture_output=True, text=True, timeout=600)
    return r.returncode


def test_pins_reject_every_planted_mistake(tmp_path):
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        rcs = list(ex.map(lambda a: _run_mutant(str(tmp_path), *a),
                          [(n, m[0], m[1], *m[3:]) for n, m in enumerate(MUTANTS)]))
    missed = [MUTANTS[n][2] for n, rc in enumerate(rcs) if rc == 0]
    assert not missed, "pins did not notice: %s" % missed
