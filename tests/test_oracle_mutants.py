"""Plants plausible mistakes in copies of the C oracle and checks that the pins
catch every one of them (CPU only; the planted copies live in a temp dir)."""
import os

import pytest

import oracle
from tests import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")

MUTANTS = {
    "decay_dropped": [("S[i * dv + j] *= a;", "S[i * dv + j] *= 1.0;")],
    "decay_sign": [("exp(lat[i])", "exp(-lat[i])")],
    "erase_gate_dropped": [("const double x = bt[i] * kt[i];", "const double x = kt[i];")],
    "erase_sign": [("(wv[j] - e[j])", "(wv[j] + e[j])")],
    "erase_transposed": [("const double x = bt[i] * kt[i];", "const double x = kt[i];"),
                         ("S[i * dv + j] += kt[i] * (wv[j] - e[j]);",
                          "S[i * dv + j] += kt[i] * wv[j] - bt[i] * kt[i] * e[j];")],
    "write_gate_dropped": [("wv[j] = wt[j] * vt[j];", "wv[j] = vt[j];")],
    "write_on_value_gate_index": [("wv[j] = wt[j] * vt[j];", "wv[j] = wt[0] * vt[j];")],
    "readout_uses_key": [("ot[j] += qt[i] *", "ot[j] += kt[i] *")],
    "readout_before_write": [("for (long j = 0; j < dv; ++j) wv[j] = wt[j] * vt[j];",
                              "for (long j = 0; j < dv; ++j) wv[j] = 0.0;"),
                             ("ot[j] += qt[i] * S[i * dv + j];\n        }",
                              "ot[j] += qt[i] * S[i * dv + j];\n        }\n"
                              "        for (long i = 0; i < dk; ++i)"
                              " for (long j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * wt[j] * vt[j];")],
    "head_index": [("const long tok = (bb * J->T + t) * J->H + h;",
                    "const long tok = (bb * J->T + t) * J->H + (J->H - 1 - h);")],
    "initial_state_ignored": [("if (J->S0)", "if (0)")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    with open(SRC) as f:
        text = f.read()
    for old, new in MUTANTS[name]:
        assert old in text, f"mutation site not found: {old!r}"
        text = text.replace(old, new, 1)
    src = tmp_path / "mutant.c"
    src.write_text(text)
    lib = oracle.load(oracle.build(str(src), str(tmp_path / "libmutant.so")))
    caught = []
    for pin in pins.ALL:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
