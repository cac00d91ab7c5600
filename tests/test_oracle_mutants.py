"""The pins catch plausible mistakes: each test plants one mistake in a copy of
the oracle's C source (on the CPU, in a temporary directory), builds it, and
requires at least one pin to fail. Each mutant runs in its own process so that
a mutant that crashes cannot take the test run down with it."""
import os
import subprocess
import sys
import textwrap

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "kda_oracle.c")

_READOUT = """    /* 3. o_t = scale * S_t^T q with the updated state. */
    if (o) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * q[i];
            o[j] = scale * acc;
        }
    }
"""
_STEP2 = "    /* 2. kS = k^T S' (a row vector over dv), then"

# (name, [(old, new), ...]) — every `old` must occur in the source.
MUTANTS = [
    ("decay_dropped", [("S[i * dv + j] *= a;", "S[i * dv + j] *= 1.0;")]),
    ("decay_sign", [("exp(log_alpha[i])", "exp(-log_alpha[i])")]),
    ("decay_scalar_channel0", [("exp(log_alpha[i])", "exp(log_alpha[0])")]),
    ("decay_on_value_axis", [("S[i * dv + j] *= a;", "S[i * dv + j] *= exp(log_alpha[j]);")]),
    ("delta_term_dropped", [("-beta * k[i] * tmp[j] + ", "")]),
    ("delta_term_sign", [("-beta * k[i] * tmp[j]", "+beta * k[i] * tmp[j]")]),
    ("beta_not_on_write", [("+ beta * k[i] * v[j]", "+ k[i] * v[j]")]),
    ("kS_transposed", [("acc += k[i] * S[i * dv + j]", "acc += k[j] * S[j * dv + i]")]),
    ("readout_transposed", [("acc += S[i * dv + j] * q[i]", "acc += S[j * dv + i] * q[j]")]),
    ("readout_uses_k", [("acc += S[i * dv + j] * q[i]", "acc += S[i * dv + j] * k[i]")]),
    ("scale_dropped", [("o[j] = scale * acc;", "o[j] = acc;")]),
    ("s0_ignored", [("if (J->S0) memcpy", "if (0) memcpy")]),
    ("varlen_off_by_one", [("t0 = J->cu_seqlens[n];", "t0 = J->cu_seqlens[n] + (n > 0);")]),
    ("readout_before_update", [(_READOUT, ""), (_STEP2, _READOUT + _STEP2)]),
]


def _build(tmp_path, name, edits):
    src = open(SRC, encoding="utf-8").read()
    for old, new in edits:
        assert old in src, f"mutant {name}: pattern not found"
        src = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src, encoding="utf-8")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                    "-ffp-contract=off", "-o", str(so), str(c), "-lm"], check=True)
    return str(so)


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, edits):
    so = _build(tmp_path, name, edits)
    code = textwrap.dedent(f"""
        import sys
        sys.path[:0] = [{ROOT!r}, {HERE!r}]
        import oracle, pins
        bad = pins.failing_pins(oracle.OracleLib({so!r}))
        print("FAILING:" + ",".join(bad))
    """)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                       timeout=300)
    if r.returncode != 0:
        return  # the mutant crashed the process: caught
    line = [l for l in r.stdout.splitlines() if l.startswith("FAILING:")][-1]
    failing = [x for x in line[len("FAILING:"):].split(",") if x]
    assert failing, f"mutant {name} passed every pin"


def test_unmutated_source_passes_in_subprocess(tmp_path):
    so = _build(tmp_path, "clean", [])
    code = textwrap.dedent(f"""
        import sys
        sys.path[:0] = [{ROOT!r}, {HERE!r}]
        import oracle, pins
        print("FAILING:" + ",".join(pins.failing_pins(oracle.OracleLib({so!r}))))
    """)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip().endswith("FAILING:"), r.stdout
