"""The masked / packed backward oracle against its pins, and planted mistakes
in copies of it (on the CPU) that the pins must catch."""
import os

import pytest

import oracle
import oracle_masked_bwd_pins

MUTANTS = [
    ("causal mask off by one", "return last + 1 < Lk ? last + 1 : Lk;", "return last < Lk ? last : Lk;"),
    ("causal offset with the wrong sign", "const int64_t last = i + (Lk - Lq);", "const int64_t last = i + (Lq - Lk);"),
    ("causal flag ignored", "if (!causal) return Lk;", "if (1) return Lk;"),
    ("keys of sequence b taken at the query offset",
     "const double *K = k + ((size_t)h * Tk + (size_t)cu_k[b]) * d;",
     "const double *K = k + ((size_t)h * Tk + (size_t)cu_q[b]) * d;"),
    ("key-side factors of hidden keys kept", "if (j >= nv) continue;", "if (j >= Lk) continue;"),
    ("key-side sum drops the sequence's last row", "for (int64_t r = cu_q[b]; r < cu_q[b + 1]; ++r) {",
     "for (int64_t r = cu_q[b]; r < cu_q[b + 1] - 1; ++r) {"),
    ("key sequence looked up in the query offsets", "kseq[jj] = seq_of(cu_k, nseq,", "kseq[jj] = seq_of(cu_q, nseq,"),
    ("wrong sign of mu in the tangent of P", "Pbar[j] += Pdbar[j] * (dS[j] - mu);", "Pbar[j] += Pdbar[j] * (dS[j] + mu);"),
    ("dropped mu_bar term of P_bar", "Pbar[j] += mubar * dS[j];", "Pbar[j] += 0.0 * dS[j];"),
    ("softmax backward without its row sum", "Sbar[j] = P[j] * (Pbar[j] - ps);", "Sbar[j] = P[j] * Pbar[j];"),
]


def _oracle(lib=None):
    def g(*args, **kw):
        return oracle.attn_jvp_bwd_packed(*args, lib=lib, **kw)
    return g


@pytest.mark.parametrize("name", list(oracle_masked_bwd_pins.ALL_PINS))
def test_pin(name):
    ok, detail = oracle_masked_bwd_pins.ALL_PINS[name](_oracle())
    assert ok, f"{name}: {detail}"


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_masked_bwd_pins_catch_mutant(desc, old, new, tmp_path):
    src = oracle.bwd_masked_source_text()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    lib = oracle.load_bwd_masked_variant(oracle.compile_variant(src.replace(old, new, 1),
                                                                os.path.join(tmp_path, "mutant_bwd_masked.so")))
    results = oracle_masked_bwd_pins.run_all(_oracle(lib))
    assert [n for n, (ok, _) in results.items() if not ok], f"no pin caught '{desc}': {results}"


def test_causal_wrapper_matches_packed():
    import numpy as np
    rng = np.random.default_rng(3)
    x = [rng.standard_normal((2, 3, L, 4)) for L in (6, 8, 8, 6, 8, 8, 6, 6)]
    got = oracle.attn_jvp_bwd_causal(*x, 0.4)
    flat = [a.reshape(6, a.shape[-2], 4) for a in x]
    ref = oracle.attn_jvp_bwd_packed(*flat, 0.4, [0, 6], [0, 8], True)
    assert all(np.array_equal(got[n].reshape(ref[n].shape), ref[n]) for n in ref)
