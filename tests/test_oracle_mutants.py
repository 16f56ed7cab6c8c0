"""Plant plausible mistakes in copies of the oracle (on the CPU) and check
that the pin suite catches every one of them."""
import os

import pytest

import oracle
import oracle_pins

# (description, text in the oracle source, replacement)
MUTANTS = [
    ("drop the P.tV term", "+ P[j] * tV[j * d + c]", ""),
    ("wrong sign of mu", "(dS[j] - mu)", "(dS[j] + mu)"),
    ("drop the centring by mu", "(dS[j] - mu)", "(dS[j])"),
    ("drop the Q.tK term", " + qi[c] * tK[j * d + c]", ""),
    ("drop the tQ.K term", "b += tqi[c] * K[j * d + c] + ", "b += "),
    ("tQ paired with tK (swapped operand)", "b += tqi[c] * K[j * d + c]", "b += tqi[c] * tK[j * d + c]"),
    ("values read from K (transposed operand)", "acc_o += P[j] * V[j * d + c]", "acc_o += P[j] * K[j * d + c]"),
    ("no scale on the score tangent", "dS[j] = scale * b", "dS[j] = b"),
    ("no scale on the scores", "S[j] = scale * a", "S[j] = a"),
    ("softmax not normalised", "for (int64_t j = 0; j < Lk; ++j) P[j] /= Z;", ""),
    ("lse without the max", "m + log(Z)", "log(Z)"),
    ("wrong feature index in the score", "a += qi[c] * K[j * d + c]", "a += qi[c] * K[j * d + (d - 1 - c)]"),
]


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(desc, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    lib = oracle.load_variant(oracle.compile_variant(src.replace(old, new, 1),
                                                     os.path.join(tmp_path, "mutant.so")))

    def f(q, k, v, tq, tk, tv, s):
        return oracle.attn_jvp(q, k, v, tq, tk, tv, s, lib=lib)

    results = oracle_pins.run_all(f)
    failed = [n for n, (ok, _) in results.items() if not ok]
    assert failed, f"no pin caught the planted mistake '{desc}': {results}"
