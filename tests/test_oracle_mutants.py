"""Plants plausible mistakes in copies of the oracle (on the CPU) and checks that the pins
of tests/oracle_pins.py catch every one of them.  This is what makes the pins worth
trusting: a dropped term, a flipped sign, a wrong operand or index, or an ignored initial
state in the token-by-token oracle must each fail at least one closed-form or invariant
check.  The real oracle passes them all (test_oracle_pins.py).
"""
import os
import re

import pytest

from oracle import build as obuild
from tests import oracle_pins as pins

with open(obuild.SRC) as _f:
    SOURCE = _f.read()

# (name, function the edit is confined to, original text, planted mistake)
MUTANTS = [
    ("delta_drops_beta", "seq_unit",
     "- bt * kt[i] * e[j]", "- kt[i] * e[j]"),
    ("delta_sign_flipped", "seq_unit",
     "- bt * kt[i] * e[j]", "+ bt * kt[i] * e[j]"),
    ("decay_hits_write_term", "seq_unit",
     "ai * (S[IDX2(i, j, dv)] - bt * kt[i] * e[j]) + bt * kt[i] * vt[j]",
     "ai * (S[IDX2(i, j, dv)] - bt * kt[i] * e[j] + bt * kt[i] * vt[j])"),
    ("decay_skipped", "seq_unit",
     "ai * (S[IDX2(i, j, dv)] - bt * kt[i] * e[j]) + bt * kt[i] * vt[j]",
     "(S[IDX2(i, j, dv)] - bt * kt[i] * e[j]) + bt * kt[i] * vt[j]"),
    ("projection_uses_query", "seq_unit",
     "e[j] += kt[i] * S[IDX2(i, j, dv)]", "e[j] += qt[i] * S[IDX2(i, j, dv)]"),
    ("readout_uses_key", "seq_unit",
     "acc += qt[i] * S[IDX2(i, j, dv)]", "acc += kt[i] * S[IDX2(i, j, dv)]"),
    ("value_off_by_one", "seq_unit",
     "const double* vt = v + t * dv;", "const double* vt = v + (t > 0 ? t - 1 : 0) * dv;"),
    ("write_transposed_index", "seq_unit",
     "+ bt * kt[i] * vt[j]", "+ bt * kt[j % dk] * vt[i % dv]"),
    ("initial_state_ignored", "seq_unit",
     "if (S0) memcpy(S, S0,", "if (0) memcpy(S, S0,"),
    ("per_key_gate_ignored", "gate_at",
     "return per_key ? alpha[t * dk + i] : alpha[t];",
     "return per_key ? alpha[t * dk] : alpha[t];"),
    ("per_key_gate_reversed", "gate_at",
     "return per_key ? alpha[t * dk + i] : alpha[t];",
     "return per_key ? alpha[t * dk + (dk - 1 - i)] : alpha[t];"),
    # decay-first order: the decay skipped, or applied to the write term as well
    ("decay_first_decay_skipped", "seq_unit",
     "for (int64_t j = 0; j < dv; ++j) S[IDX2(i, j, dv)] *= ai;",
     "for (int64_t j = 0; j < dv; ++j) S[IDX2(i, j, dv)] *= 1.0;"),
    ("decay_first_projects_undecayed", "seq_unit",
     "S[IDX2(i, j, dv)] += bt * kt[i] * (vt[j] - e[j]);",
     "S[IDX2(i, j, dv)] += bt * kt[i] * (vt[j] - e[j] / gate_at(alpha, per_key, t, i, dk));"),
    ("decay_first_delta_first", "seq_unit",
     "if (per_key == 2) {\n            /* decay first", "if (0) {\n            /* decay first"),
]


def _function_span(src, name):
    m = re.search(r"\n(static )?[a-z]+\s+" + name + r"\(", src)
    assert m, f"function {name} not found in the oracle source"
    start = m.start()
    depth, i = 0, src.index("{", start)
    while True:
        if src[i] == "{":
            depth += 1
        elif src[i] == "}":
            depth -= 1
            if depth == 0:
                return start, i + 1
        i += 1


def _mutate(func, old, new):
    a, b = _function_span(SOURCE, func)
    body = SOURCE[a:b]
    assert old in body, f"pattern for the planted mistake no longer in {func}: {old!r}"
    return SOURCE[:a] + body.replace(old, new, 1) + SOURCE[b:]


@pytest.mark.parametrize("name,func,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, func, old, new):
    src = tmp_path / f"mutant_{name}.c"
    src.write_text(_mutate(func, old, new))
    lib = obuild.build(src=str(src), out=str(tmp_path / f"libmutant_{name}.so"))
    caught = []
    for pin_name, check in pins.ALL_PINS:
        try:
            check(lib)
        except AssertionError:
            caught.append(pin_name)
    assert caught, f"no pin caught the planted mistake {name}"
