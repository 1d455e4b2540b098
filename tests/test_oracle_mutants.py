"""Plausible mistakes planted in the oracle must each fail at least one pin.

Each mutant is a textual edit of ``oracle/gdn_oracle.c`` (a dropped term, a
wrong sign, index, operand or mask), compiled into a temporary library with
gcc and loaded in a child process through ``GDN_ORACLE_LIB_OVERRIDE``; the
child runs every pin of ``tests/oracle_pins.py`` and reports which failed.
Nothing here touches a GPU.
"""
import json
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.c")

# (name, text to find, replacement, which occurrence (0-based))
MUTANTS = [
    ("gate_sign", "g[i] = -exp(A_log[h]) * sp;", "g[i] = exp(A_log[h]) * sp;", 0),
    ("softplus_as_exp", "(x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)))", "exp(x)", 0),
    ("sigmoid_sign", "beta[i] = 1.0 / (1.0 + exp(-b[i]));", "beta[i] = 1.0 / (1.0 + exp(b[i]));", 0),
    ("gate_no_bias", "const double x = a[i] + dt_bias[h];", "const double x = a[i];", 0),
    ("no_decay", "S[e] *= alpha;", "S[e] *= 1.0;", 0),
    ("delta_sign", "kv[c] = b * (vt[c] - kv[c]);", "kv[c] = b * (vt[c] + kv[c]);", 0),
    ("kv_uses_query", "kv[c] += S[(size_t)r * dv + c] * kh[r];",
     "kv[c] += S[(size_t)r * dv + c] * qh[r];", 0),
    ("no_beta", "kv[c] = b * (vt[c] - kv[c]);", "kv[c] = (vt[c] - kv[c]);", 0),
    ("output_before_write", "ot[c] += S[(size_t)r * dv + c] * qh[r];",
     "ot[c] += (S[(size_t)r * dv + c] - kh[r] * kv[c]) * qh[r];", 0),
    ("state_transposed_read", "kv[c] += S[(size_t)r * dv + c] * kh[r];",
     "kv[c] += S[(size_t)(c % dk) * dv + (r % dv)] * kh[r];", 0),
    ("gqa_modulo_rec", "const int j = h / group;                     /* qk-head of v-head h */",
     "const int j = h % nqk;", 0),
    ("gqa_modulo_chunk", "const int j = h / group;\n        const long t0",
     "const int j = h % nqk;\n        const long t0", 0),
    ("eps_outside_root", "1.0 / sqrt(ss + ORACLE_EPS)", "1.0 / (sqrt(ss) + ORACLE_EPS)", 0),
    ("no_key_norm", "normalise(k + ((size_t)t * nqk + j) * dk, dk, qk_l2norm, 1.0, kh);",
     "normalise(k + ((size_t)t * nqk + j) * dk, dk, 0, 1.0, kh);", 0),
    ("scale_1_over_dk", "if (scale <= 0.0) scale = 1.0 / sqrt((double)dk);\n    const int group = nv / nqk;\n    const long pairs = (long)num_seqs * nv;\n\n#pragma omp parallel for schedule(dynamic, 1)\n    for (long p = 0; p < pairs; ++p) {\n        const int n = (int)(p / nv), h = (int)(p % nv);\n        const int j = h / group;                     /* qk-head of v-head h */",
     "if (scale <= 0.0) scale = 1.0 / (double)dk;\n    const int group = nv / nqk;\n    const long pairs = (long)num_seqs * nv;\n\n#pragma omp parallel for schedule(dynamic, 1)\n    for (long p = 0; p < pairs; ++p) {\n        const int n = (int)(p / nv), h = (int)(p % nv);\n        const int j = h / group;                     /* qk-head of v-head h */", 0),
    ("no_initial_state", "if (s0) memcpy(S, s0 + sidx, sizeof(double) * (size_t)dk * dv);",
     "if (0) memcpy(S, s0 + sidx, sizeof(double) * (size_t)dk * dv);", 0),
    # chunk form
    ("A_sign", "s = -s * gamma[(size_t)r * C + i];", "s = s * gamma[(size_t)r * C + i];", 0),
    ("A_keeps_diagonal", "if (i < r) {\n                for (int d = 0; d < dk; ++d) s += kb",
     "if (i <= r) {\n                for (int d = 0; d < dk; ++d) s += kb", 0),
    ("exclusive_cumsum", "acc += g[i]; gcum[i] = acc;", "gcum[i] = acc; acc += g[i];", 0),
    ("recursion_short", "for (int m = 0; m < i; ++m) s += A[(size_t)i * C + m] * T[(size_t)m * C + j];",
     "for (int m = 0; m + 1 < i; ++m) s += A[(size_t)i * C + m] * T[(size_t)m * C + j];", 0),
    ("W_without_decay", "s += T[(size_t)r * C + i] * kb[(size_t)i * dk + d] * exp(gcum[i]);",
     "s += T[(size_t)r * C + i] * kb[(size_t)i * dk + d];", 0),
    ("attn_strict", "if (i <= r) {\n                        for (int d = 0; d < dk; ++d) s += Qc",
     "if (i < r) {\n                        for (int d = 0; d < dk; ++d) s += Qc", 0),
    ("state_no_chunk_decay", "double s = S[(size_t)d * dv + x] * exp(glast);",
     "double s = S[(size_t)d * dv + x];", 0),
    ("key_decay_wrong", "exp(glast - gc[i])", "exp(gc[i])", 0),
    ("inter_no_decay", "s1 += Qc[(size_t)r * dk + d] * eg * S[(size_t)d * dv + x];",
     "s1 += Qc[(size_t)r * dk + d] * S[(size_t)d * dv + x];", 0),
    # gated RMSNorm epilogue
    ("norm_eps_outside_root", "const double inv = 1.0 / sqrt(ms + eps);",
     "const double inv = 1.0 / (sqrt(ms) + eps);", 0),
    ("norm_sum_not_mean", "ms /= (double)dv;", "ms /= 1.0;", 0),
    ("norm_gate_sigmoid", "const double gate = zrow[c] / (1.0 + exp(-zrow[c]));",
     "const double gate = 1.0 / (1.0 + exp(-zrow[c]));", 0),
    ("norm_gate_on_o", "const double gate = zrow[c] / (1.0 + exp(-zrow[c]));",
     "const double gate = zrow[c] / (1.0 + exp(-orow[c]));", 0),
    # causal conv1d + SiLU
    ("conv_taps_shifted", "pre += w[(size_t)c * ksize + i] * ext[t + 1 + i];",
     "pre += w[(size_t)c * ksize + i] * ext[t + i];", 0),
    ("conv_taps_reversed", "pre += w[(size_t)c * ksize + i] * ext[t + 1 + i];",
     "pre += w[(size_t)c * ksize + (ksize - 1 - i)] * ext[t + 1 + i];", 0),
    ("conv_no_silu", "y[(t0 + t) * channels + c] = pre / (1.0 + exp(-pre));",
     "y[(t0 + t) * channels + c] = pre;", 0),
    ("conv_state_ignored", "ext[i] = state_in ? state_in[sidx + i] : 0.0;", "ext[i] = 0.0;", 0),
    ("conv_no_bias", "double pre = bias ? bias[c] : 0.0;", "double pre = 0.0;", 0),
    ("conv_state_not_advanced", "state_out[sidx + i] = ext[len + i];",
     "state_out[sidx + i] = ext[i];", 0),
]

CHILD = r"""
import json, sys
sys.path.insert(0, %r)
from tests import oracle_pins as P
failed = []
for pin in P.ALL_PINS:
    try:
        pin()
    except Exception as e:  # AssertionError or a bad-argument error
        failed.append(pin.__name__)
print("PINS_FAILED=" + json.dumps(failed))
""" % ROOT


def _replace_nth(text, old, new, n):
    idx = -1
    for _ in range(n + 1):
        idx = text.find(old, idx + 1)
        if idx < 0:
            return None
    return text[:idx] + new + text[idx + len(old):]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m[0])
def test_mutant_is_caught(mutant, tmp_path):
    name, old, new, nth = mutant
    src = open(SRC).read()
    mutated = _replace_nth(src, old, new, nth)
    assert mutated is not None and mutated != src, "mutation site not found: " + name
    c_path = tmp_path / ("m_%s.c" % name)
    so_path = tmp_path / ("m_%s.so" % name)
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", str(so_path), str(c_path), "-lm"])
    env = dict(os.environ, GDN_ORACLE_LIB_OVERRIDE=str(so_path), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=300)
    if r.returncode != 0:
        return  # the mutant crashed the oracle: caught
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("PINS_FAILED=")][-1]
    failed = json.loads(line.split("=", 1)[1])
    assert failed, "mutant %s passed every pin" % name


def test_unmutated_source_passes_all_pins(tmp_path):
    so_path = tmp_path / "clean.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", str(so_path), SRC, "-lm"])
    env = dict(os.environ, GDN_ORACLE_LIB_OVERRIDE=str(so_path), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("PINS_FAILED=")][-1]
    assert json.loads(line.split("=", 1)[1]) == []
