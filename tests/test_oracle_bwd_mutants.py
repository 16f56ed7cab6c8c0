"""Plant plausible mistakes in copies of the backward oracle (on the CPU) and
check that the backward pin suite catches every one of them."""
import os

import pytest

import oracle
import oracle_bwd_pins

# (description, text in the backward oracle source, replacement)
MUTANTS = [
    ("drop the centred tangent term of P_bar", "Pbar[j] += Pdbar[j] * (dS[j] - mu);", ""),
    ("wrong sign of mu_bar", "mubar -= Pdbar[j] * P[j];", "mubar += Pdbar[j] * P[j];"),
    ("drop mu_bar in P_bar", "Pbar[j] += mubar * dS[j];", ""),
    ("drop mu_bar in dS_bar", "dSbar[j] += mubar * P[j];", ""),
    ("softmax backward without the row sum", "Sbar[j] = P[j] * (Pbar[j] - ps);", "Sbar[j] = P[j] * Pbar[j];"),
    ("drop the dtO.tV term of P_bar", "dot(dtOi, tV + (size_t)j * d, d) + ", ""),
    ("dtV weighted by the tangent of P", "dtVj[c] += pm * dtOi[c];", "dtVj[c] += pdm * dtOi[c];"),
    ("dV without the tangent-of-P term", " + pdm * dtOi[c]", ""),
    ("dK without the tQ term", " + dsb * tQi[c]", ""),
    ("dtK paired with tQ (swapped operand)", "dtKj[c] += scale * dsb * Qi[c];", "dtKj[c] += scale * dsb * tQi[c];"),
    ("dQ without the dS_bar.tK term", " + dSbar[j] * tK[(size_t)j * d + c]", ""),
    ("dtQ paired with tK (swapped operand)", "b += dSbar[j] * K[(size_t)j * d + c];",
     "b += dSbar[j] * tK[(size_t)j * d + c];"),
    ("no scale on dQ", "dQi[c] = scale * a;", "dQi[c] = a;"),
    ("tangent of P stored uncentred", "PDM[at] = P[j] * (dS[j] - mu);", "PDM[at] = P[j] * dS[j];"),
]


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_bwd_pins_catch_mutant(desc, old, new, tmp_path):
    src = oracle.bwd_source_text()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    lib = oracle.load_bwd_variant(oracle.compile_variant(src.replace(old, new, 1),
                                                         os.path.join(tmp_path, "mutant_bwd.so")))

    def g(*args, **kw):
        return oracle.attn_jvp_bwd(*args, lib=lib, **kw)

    results = oracle_bwd_pins.run_all(g)
    failed = [n for n, (ok, _) in results.items() if not ok]
    assert failed, f"no pin caught the planted mistake '{desc}': {results}"
