"""The oracle's pins must fail on plausible mistakes (CPU only).

Each case below compiles a copy of oracle.c with one deliberate slip (a dropped term, a flipped
sign, a transposed state, an operand swapped, an off-by-one in a mask or a window, a wrong GQA
map, a missing ring wrap) and runs the pin suite against that copy; the suite must fail.
Nothing here touches a GPU.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, [(old, new), ...]); every `old` must occur in oracle.c (first occurrence replaced)
MUTANTS = [
    ("gdn_drop_delta_term", [("- g * beta * Sk[j] * k[i]", "")]),
    ("gdn_flip_write_sign", [("+ beta * v[j] * k[i];", "- beta * v[j] * k[i];")]),
    ("gdn_untransposed_state", [
        ("if (kind == OR_GDN) S[(size_t)j * dk + i] = M[(size_t)i * dv + j];",
         "if (kind == OR_GDN) S[(size_t)i * dv + j] = M[(size_t)i * dv + j];"),
        ("(kind == OR_GDN) ? S[(size_t)j * dk + i]", "(kind == OR_GDN) ? S[(size_t)i * dv + j]")]),
    ("kda_gate_dropped_in_correction", [("acc += k[i] * a[i] * S[", "acc += k[i] * S[")]),
    ("kda_output_wrong_operand", [("acc += S[(size_t)i * dv + j] * q[i];",
                                   "acc += S[(size_t)i * dv + j] * k[i];")]),
    ("chunk_T_without_beta", [("(r == c) ? beta[TH(r)] : 0.0", "(r == c) ? 1.0 : 0.0")]),
    ("chunk_solve_drops_a_term", [("for (int s = 0; s < r; ++s) x -=",
                                   "for (int s = 1; s < r; ++s) x -=")]),
    ("chunk_P_excludes_diagonal", [("(s <= r) ? p : 0.0", "(s < r) ? p : 0.0")]),
    ("chunk_state_decay_missing", [("double acc = exp(gC) * M[", "double acc = M[")]),
    ("chunk_decay_split_into_factors", [
        ("const double e = exp(G[(size_t)r * dk + i] - G[(size_t)s * dk + i]);",
         "const double e = exp(G[(size_t)r * dk + i]) * exp(-G[(size_t)s * dk + i]);")]),
    ("chunk_state_factor_split", [("* exp(gC - G[(size_t)s * dk + i]) *",
                                   "* exp(gC) * exp(-G[(size_t)s * dk + i]) *")]),
    ("attn_scale_missing", [("s[j - lo] = acc * inv_sqrt_d;", "s[j - lo] = acc;")]),
    ("swa_window_off_by_one", [("? L - window : 0", "? L - window + 1 : 0")]),
    ("gqa_map_interleaved", [("g = h / group", "g = h % Hkv")]),
    ("ring_not_wrapped", [("idx = pos % (R * page_tokens);", "idx = pos;")]),
    ("new_token_ignored", [("if (j == L - 1) {", "if (0) {")]),
    ("prefill_window_off_by_one", [("? t + 1 - window : 0", "? t - window : 0")]),
    ("prefill_gqa_interleaved", [("kvh = h / group", "kvh = h % Hkv")]),
    ("prefill_scale_missing", [("s[j - lo] = inv_sqrt_d * acc;", "s[j - lo] = acc;")]),
    ("prefill_value_row_shifted", [("const double *vv = v + (((size_t)b * T + j) * Hkv + kvh) * d;",
                                    "const double *vv = v + (((size_t)b * T + (j > lo ? j - 1 : j)) * Hkv + kvh) * d;")]),
    ("verify_window_off_by_one", [("? P_pos + 1 - window : 0", "? P_pos - window : 0")]),
    ("verify_gqa_interleaved", [("kvh_v = h / heads_per_kv", "kvh_v = h % Hkv")]),
    ("verify_ring_not_wrapped", [("ring_idx = pos % ((long)ring_pages * page_tokens);",
                                  "ring_idx = pos;")]),
    ("verify_first_new_key_from_pool", [("if (j >= first_new) {", "if (j > first_new) {")]),
    ("verify_rows_shifted", [("const int P_pos = first_new + i;", "const int P_pos = first_new + i - (i > 0);")]),
    ("act_norm_without_sqrt", [("const double nq = sqrt(sq + eps), nk = sqrt(sk + eps);",
                                "const double nq = sq + eps, nk = sqrt(sk + eps);")]),
    ("act_sigmoid_sign", [("beta[row] = 1.0 / (1.0 + exp(-beta_logit[row]));",
                           "beta[row] = 1.0 / (1.0 + exp(beta_logit[row]));")]),
    ("act_gate_bias_dropped", [("const double x = gate_logit[row * dk + i] + dt_bias[(size_t)h * dk + i];",
                                "const double x = gate_logit[row * dk + i];")]),
    ("act_gate_rate_not_exponentiated", [("const double decay_rate = exp(A_log[h]);",
                                          "const double decay_rate = A_log[h];")]),
]


def _build_mutant(tmp, name, edits):
    with open(SRC) as f:
        src = f.read()
    for old, new in edits:
        assert old in src, f"{name}: pattern not found: {old!r}"
        src = src.replace(old, new, 1)
    c = os.path.join(tmp, f"{name}.c")
    so = os.path.join(tmp, f"{name}.so")
    with open(c, "w") as f:
        f.write(src)
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                    c, "-o", so, "-lm"], check=True)
    return so


def _run_pins(so):
    env = dict(os.environ, ORACLE_LIB=so, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


def test_every_mutant_fails_the_pins():
    with tempfile.TemporaryDirectory() as tmp:
        libs = {name: _build_mutant(tmp, name, edits) for name, edits in MUTANTS}
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            rcs = dict(zip(libs, ex.map(_run_pins, libs.values())))
    survivors = [n for n, rc in rcs.items() if rc == 0]
    assert not survivors, f"mutants not caught by the oracle pins: {survivors}"
