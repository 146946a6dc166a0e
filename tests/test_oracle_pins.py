"""The fp64 oracle against its pins (CPU only)."""
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins


@pytest.fixture(scope="module")
def orc():
    return oracle.Oracle(oracle.build())


@pytest.mark.parametrize("name", list(pins.ALL_PINS))
def test_pin(orc, name):
    ok, err = pins.ALL_PINS[name](orc)
    assert ok, f"pin {name} failed: err={err:.3e}"


def test_no_s0_equals_zero_s0(orc):
    q, k, v, g, S0 = pins.rand_case(3, L=16)
    o1, s1, _ = orc.forward(q, k, v, g, None)
    o2, s2, _ = orc.forward(q, k, v, g, np.zeros_like(S0))
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_heads_independent(orc):
    q, k, v, g, S0 = pins.rand_case(4, B=2, H=3, L=10)
    o, sf, _ = orc.forward(q, k, v, g, S0)
    o1, sf1, _ = orc.forward(q[1:2, 2:3], k[1:2, 2:3], v[1:2, 2:3], g[1:2, 2:3], S0[1:2, 2:3])
    assert np.array_equal(o[1:2, 2:3], o1) and np.array_equal(sf[1:2, 2:3], sf1)


# Deliberately broken copies of the oracle source: each must fail at least one pin.  This
# shows the pins would catch a dropped term, a wrong sign, a wrong index or operand.
MUTANTS = {
    "dropped_gate": ("Si[j] = a[i] * Si[j] + kt[i] * vt[j];", "Si[j] = Si[j] + kt[i] * vt[j];"),
    "gate_sign": ("for (long i = 0; i < dk; ++i) a[i] = exp(gt[i]);",
                  "for (long i = 0; i < dk; ++i) a[i] = exp(-gt[i]);"),
    "readout_uses_k": ("ot[j] += qt[i] * Si[j];", "ot[j] += kt[i] * Si[j];"),
    "outer_transposed": ("Si[j] = a[i] * Si[j] + kt[i] * vt[j];",
                         "Si[j] = a[i] * Si[j] + kt[j % dk] * vt[i % dv];"),
    "bwd_dq_uses_prev_state": ("acc += dOt[j] * St[i * dv + j];", "acc += dOt[j] * Sm[i * dv + j];"),
    "bwd_dg_no_gate_factor": ("dg[t * dk + i] = a[i] * acc;", "dg[t * dk + i] = acc;"),
    "bwd_carry_no_decay": ("for (long j = 0; j < dv; ++j) dS[i * dv + j] *= a[i];",
                           "for (long j = 0; j < dv; ++j) dS[i * dv + j] *= 1.0;"),
    "bwd_dv_uses_q": ("dv_[t * dv + j] += kt[i] * dS[i * dv + j];",
                      "dv_[t * dv + j] += qt[i] * dS[i * dv + j];"),
    "bwd_dk_transposed": ("acc += dS[i * dv + j] * vt[j];", "acc += dS[i * dv + j] * qt[j % dk];"),
}


@pytest.mark.parametrize("mutant", list(MUTANTS))
def test_pins_catch_mutant(mutant):
    src = open(oracle.SRC_PATH).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) >= 1, "mutation target vanished from the oracle source"
    d = tempfile.mkdtemp(prefix="la_oracle_mut_")
    try:
        path = os.path.join(d, "mut.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new, 1))
        lib = oracle.compile_lib(path, os.path.join(d, "libmut.so"))
        results = pins.run_all(oracle.Oracle(lib))
        failed = [n for n, (ok, _) in results.items() if not ok]
        assert failed, f"no pin caught mutant {mutant}"
    finally:
        shutil.rmtree(d)
