"""The oracle's pins must catch plausible mistakes: plant each one in a copy of the oracle (CPU only).

Each mutant is the oracle source with one edit (a dropped term, a wrong sign
or index, a swapped field); the pin suites must fail on every one of them.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ds4moe_oracle.c")

MUTANTS = {
    "parity_inverted": ("int neg = (i < 7) ? ((bits7 >> i) & 1) : parity;",
                        "int neg = (i < 7) ? ((bits7 >> i) & 1) : !parity;"),
    "iq2x_scale_offset": ("(d * (0.5f + (float)s)) * 0.25f", "(d * (1.0f + (float)s)) * 0.25f"),
    "iq2x_sign_stride": ("(aux >> (7 * j)) & 0x7F", "(aux >> (8 * j)) & 0x7F"),
    "q2k_nibbles_swapped": ("int sc = b[sub] & 0xF;\n        int m = b[sub] >> 4;",
                            "int m = b[sub] & 0xF;\n        int sc = b[sub] >> 4;"),
    "q2k_min_dropped": ("out[i] = a * (float)q - c;\n    }\n}\n\nstatic int q4k",
                        "out[i] = a * (float)q;\n    }\n}\n\nstatic int q4k"),
    "q4k_nibble_order": ("int q = (i & 1) ? (qs[i >> 1] >> 4) : (qs[i >> 1] & 0xF);",
                         "int q = (i & 1) ? (qs[i >> 1] & 0xF) : (qs[i >> 1] >> 4);"),
    "q4k_min_field": ("int m = q4k_field6(sc12, 48 + 6 * sub);", "int m = q4k_field6(sc12, 42 + 6 * sub);"),
    "tie_to_larger_id": ("if (best < 0 || s[e] > s[best]) best = e;", "if (best < 0 || s[e] >= s[best]) best = e;"),
    "bias_after_sigmoid": ("if (bias) acc += (double)bias[e];\n        s[e] = sigmoid(acc);",
                           "s[e] = sigmoid(acc);\n        if (bias) s[e] += (double)bias[e];"),
    "no_renormalise": ("w[j] = s[ids[j]] / tot;", "w[j] = s[ids[j]];"),
    "silu_without_sigmoid": ("static double silu(double g) { return g * sigmoid(g); }",
                             "static double silu(double g) { return g; }"),
    "shared_expert_dropped": ("for (int n = 0; n < d; n++) out[n] += y[n];", "(void)0;"),
    "combine_weight_dropped": ("out[n] += w[j] * y[n];", "out[n] += y[n];"),
}

PIN_FILES = ["tests/test_oracle_formats.py", "tests/test_oracle_route.py", "tests/test_oracle_layer.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor drifted: %s" % name
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                           "-o", str(so), str(msrc), "-lm"])
    env = dict(os.environ, DS4MOE_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] + PIN_FILES,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not catch mutant %s" % name
