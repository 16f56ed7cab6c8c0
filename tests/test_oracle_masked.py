"""The masked / packed oracle against its pins, and planted mistakes in copies
of it (on the CPU) that the pins must catch."""
import os

import pytest

import oracle
import oracle_masked_pins

MUTANTS = [
    ("causal mask off by one", "nvis = last + 1 < Lk ? last + 1 : Lk;", "nvis = last < Lk ? last : Lk;"),
    ("causal offset with the wrong sign", "const int64_t last = i + (Lk - Lq);", "const int64_t last = i + (Lq - Lk);"),
    ("causal flag ignored", "if (causal) {", "if (0) {"),
    ("keys of sequence b taken at the query offset",
     "const double *K = k + ((size_t)h * Tk + cu_k[b]) * d,", "const double *K = k + ((size_t)h * Tk + cu_q[b]) * d,"),
    ("empty rows get lse 0", "lse[(size_t)h * Tq + r] = -INFINITY;", "lse[(size_t)h * Tq + r] = 0.0;"),
    ("drop the P.tV term", " + P * tV[j * d + c];", ";"),
    ("wrong sign of mu", "(dS[j] - mu)", "(dS[j] + mu)"),
]


@pytest.mark.parametrize("name", list(oracle_masked_pins.ALL_PINS))
def test_pin(name):
    ok, detail = oracle_masked_pins.ALL_PINS[name](oracle.attn_jvp_packed)
    assert ok, f"{name}: {detail}"


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_masked_pins_catch_mutant(desc, old, new, tmp_path):
    src = oracle.masked_source_text()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    lib = oracle.load_masked_variant(oracle.compile_variant(src.replace(old, new, 1),
                                                            os.path.join(tmp_path, "mutant_masked.so")))

    def f(*args):
        return oracle.attn_jvp_packed(*args, lib=lib)

    results = oracle_masked_pins.run_all(f)
    assert [n for n, (ok, _) in results.items() if not ok], f"no pin caught '{desc}': {results}"
