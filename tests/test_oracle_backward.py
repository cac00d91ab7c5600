"""The oracle's backward (reverse-mode derivatives of <dO, o> + <dS_final,
S_final>) against its pins, and the pins against planted mistakes: each test
below plants one mistake in a copy of the oracle's C source (on the CPU), builds
it, and requires at least one backward pin to fail. Each mutant runs in its own
process so that a mutant that crashes cannot take the test run down with it."""
import os
import subprocess
import sys
import textwrap

import pytest

import oracle
import pins

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "kda_oracle.c")


@pytest.mark.parametrize("name", list(pins.BACKWARD_ALL))
def test_backward_pin(name):
    e = pins.BACKWARD_ALL[name](oracle.default())
    assert e <= pins.BACKWARD_TOL[name], (name, e)


def test_backward_without_states_or_final_gradient():
    """S0 and dS_final absent mean zero; the gradient of the (zero) initial
    state is still returned."""
    import numpy as np
    r = np.random.default_rng(7)
    q, k, v = r.normal(size=(1, 5, 1, 3)), r.normal(size=(1, 5, 1, 3)), r.normal(size=(1, 5, 1, 2))
    la, b = -np.log1p(np.exp(r.normal(size=(1, 5, 1, 3)))), np.full((1, 5, 1), 0.5)
    dO = r.normal(size=v.shape)
    g = oracle.backward(q, k, v, la, b, dO)
    g0 = oracle.backward(q, k, v, la, b, dO, np.zeros((1, 1, 3, 2)), np.zeros((1, 1, 3, 2)))
    for key in g:
        assert np.array_equal(g[key], g0[key]), key
    assert g["dS0"].shape == (1, 1, 3, 2) and np.any(g["dS0"] != 0)


# (name, [(old, new), ...]) — every `old` must occur in the source.
MUTANTS = [
    ("bwd_dv_beta_dropped", [("J->gv[th * dv + j] = bt * gk_;", "J->gv[th * dv + j] = gk_;")]),
    ("bwd_dk_second_term_sign", [("J->gk[th * dk + i] = bt * (gw - sg);",
                                  "J->gk[th * dk + i] = bt * (gw + sg);")]),
    ("bwd_dbeta_without_prediction", [("db += gk_ * w[j];", "db += gk_ * vt[j];")]),
    ("bwd_dlog_alpha_pre_decay_state", [("dl += d * Sp[i * dv + j];", "dl += d * P[i * dv + j];")]),
    ("bwd_state_gradient_not_decayed", [("G[i * dv + j] = alpha[i] * d;", "G[i * dv + j] = d;")]),
    ("bwd_dq_pre_update_state", [("acc += Q[i * dv + j] * dOt[j];", "acc += P[i * dv + j] * dOt[j];")]),
    ("bwd_readout_gradient_scale_dropped", [("G[i * dv + j] += J->scale * qt[i] * dOt[j];",
                                             "G[i * dv + j] += qt[i] * dOt[j];")]),
    ("bwd_final_gradient_ignored", [("if (J->dS_final) memcpy(G,", "if (0) memcpy(G,")]),
    ("bwd_replay_block_shifted", [("const int64_t a = t0 + b * CKPT,", "const int64_t a = t0 + b * CKPT + (b > 0),")]),
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


def _failing(so):
    code = textwrap.dedent(f"""
        import sys
        sys.path[:0] = [{ROOT!r}, {HERE!r}]
        import oracle, pins
        print("FAILING:" + ",".join(pins.failing_backward_pins(oracle.OracleLib({so!r}))))
    """)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    if r.returncode != 0:
        return None  # crashed
    line = [l for l in r.stdout.splitlines() if l.startswith("FAILING:")][-1]
    return [x for x in line[len("FAILING:"):].split(",") if x]


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_backward_mutant_is_caught(tmp_path, name, edits):
    failing = _failing(_build(tmp_path, name, edits))
    assert failing is None or failing, f"mutant {name} passed every backward pin"


def test_unmutated_backward_passes_in_subprocess(tmp_path):
    assert _failing(_build(tmp_path, "clean", [])) == []
