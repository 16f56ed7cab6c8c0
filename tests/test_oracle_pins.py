"""The fp64 oracle against facts other than itself (closed forms, central
finite differences, library routines, invariants).  CPU only."""
import numpy as np
import pytest

import oracle
import oracle_pins


def _f(q, k, v, tq, tk, tv, s):
    return oracle.attn_jvp(q, k, v, tq, tk, tv, s)


@pytest.mark.parametrize("name", list(oracle_pins.ALL_PINS))
def test_pin(name):
    ok, detail = oracle_pins.ALL_PINS[name](_f)
    assert ok, f"{name}: {detail}"


def test_rows_are_independent():
    """A gathered subset of query rows gives the same rows as the full call
    (the property the sampled large-size parity tests rely on)."""
    rng = np.random.default_rng(3)
    q, tq = rng.standard_normal((2, 2, 40, 8)), rng.standard_normal((2, 2, 40, 8))
    k, v, tk, tv = (rng.standard_normal((2, 2, 33, 8)) for _ in range(4))
    O, tO, lse = oracle.attn_jvp(q, k, v, tq, tk, tv, 0.3)
    rows = [0, 5, 39]
    o2, to2, l2 = oracle.attn_jvp_rows(q.reshape(4, 40, 8), k.reshape(4, 33, 8),
                                       v.reshape(4, 33, 8), tq.reshape(4, 40, 8),
                                       tk.reshape(4, 33, 8), tv.reshape(4, 33, 8), 0.3,
                                       heads=[1, 3], rows=rows)
    assert np.array_equal(o2[0], O.reshape(4, 40, 8)[1][rows])
    assert np.array_equal(to2[1], tO.reshape(4, 40, 8)[3][rows])
    assert np.array_equal(l2[1], lse.reshape(4, 40)[3][rows])


def test_bad_arguments_rejected():
    lib = oracle._get()
    import ctypes
    dp = ctypes.POINTER(ctypes.c_double)
    buf = (ctypes.c_double * 16)()
    p = ctypes.cast(buf, dp)
    assert lib.oracle_attn_jvp_f64(p, p, p, p, p, p, p, p, p, 1, 1, 0, 4, 1.0) == -1  # Lk == 0
    assert lib.oracle_attn_jvp_f64(p, p, p, p, p, p, p, p, p, 1, 1, 1, 0, 1.0) == -1  # d == 0


def test_golden_regression():
    """The oracle still reproduces the committed small fixture."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")
    g = json.load(open(path))
    arrs = [np.array(g[n], dtype=np.float64) for n in ("q", "k", "v", "tq", "tk", "tv")]
    o, to, lse = oracle.attn_jvp(*arrs, g["scale"])
    assert np.allclose(o, g["o"], rtol=0, atol=1e-14)
    assert np.allclose(to, g["to"], rtol=0, atol=1e-14)
    assert np.allclose(lse, g["lse"], rtol=0, atol=1e-14)
