"""The oracle pins catch plausible mistakes (CPU only).

Each case copies the oracle source, plants one mistake (a dropped term, a
wrong sign, index or operand), compiles the copy and runs the pin tests
against it: every mutant must fail at least one pin.
"""
import concurrent.futures
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lisa_ref.cpp")

MUTANTS = {
    "relu_dropped": ("const double relu = dot > 0.0 ? dot : 0.0;", "const double relu = dot;"),
    "weight_dropped": ("total += weight_at(D, w, w_tok_stride, b, t, j) * relu;", "total += relu;"),
    "key_head_fixed": ("const int jk = j % D->H_Ik;", "const int jk = 0;"),
    "causal_off_by_one": ("if (s > p) { out[s] = -INFINITY; continue; }",
                          "if (s >= p) { out[s] = -INFINITY; continue; }"),
    "tie_break_reversed": ("return a.second < c.second;", "return a.second > c.second;"),
    "budget_short": ("const int keep = std::min(D->M, p + 1);", "const int keep = std::min(D->M, p);"),
    "scale_dropped": ("logit[i] = D->sm_scale * dot;", "logit[i] = dot;"),
    "gqa_interleaved": ("attend(D, qh, k_cache, v_cache, b, h / group, pos, npos, out);",
                        "attend(D, qh, k_cache, v_cache, b, h % D->H_kv, pos, npos, out);"),
    "state_transposed": ("Sg[(int64_t)i * d + j] += fk[i] * (double)vt[j];",
                         "Sg[(int64_t)j * d + i] += fk[i] * (double)vt[j];"),
    "normaliser_dropped": ("out[j] = acc / denom;", "out[j] = acc;"),
    "gate_swapped": ("g * o_lin[base + c] + (1.0 - g) * o_sp[base + c]",
                     "g * o_sp[base + c] + (1.0 - g) * o_lin[base + c]"),
    "elu_shift_dropped": ("return x > 0.0 ? x + 1.0 : std::exp(x);", "return x > 0.0 ? x : std::exp(x);"),
    "softmax_max_wrong": ("const double e = std::exp(logit[i] - mx);", "const double e = std::exp(logit[i]);"),
    "window_short": ("const int first = std::max(0, p - D->M + 1);",
                     "const int first = std::max(0, p - D->M + 2);"),
    "transfer_mean_over_t": ("grad_sum[i] / (t - 1)", "grad_sum[i] / t"),
    "transfer_alpha_swapped": ("(1.0 - alpha) * grad_t + alpha * mean_prev",
                               "alpha * grad_t + (1.0 - alpha) * mean_prev"),
    "transfer_start_kept": ("        S_start[i] = S_t;\n", "        S_start[i] = S_start[i];\n"),
    "channel_gate_swapped": ("(1.0 - g) * o_sp[base + c] + g * o_lin[base + c]",
                             "g * o_sp[base + c] + (1.0 - g) * o_lin[base + c]"),
    "channel_weight_transposed": ("W_g[(int64_t)c * D_h + k]", "W_g[(int64_t)k * N + c]"),
}


def _run_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    msrc = os.path.join(tmp, f"{name}.cpp")
    mlib = os.path.join(tmp, f"{name}.so")
    open(msrc, "w").write(src.replace(old, new))
    subprocess.run(["g++", "-O1", "-std=c++17", "-fopenmp", "-fPIC", "-shared", msrc, "-o", mlib],
                   check=True)
    env = dict(os.environ, LISA_REF_LIB=mlib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py"),
                        os.path.join(ROOT, "tests", "test_oracle_next.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with concurrent.futures.ThreadPoolExecutor(max_workers=4) as ex:
            futs = [ex.submit(_run_mutant, n, o, m, tmp) for n, (o, m) in MUTANTS.items()]
            results = dict(f.result() for f in futs)
    survivors = [n for n, rc in results.items() if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
