"""The oracle and the input generator reproduce the stored C0 samples (CPU only)."""
import json
import os

from tests.golden import make_golden


def test_c0_samples_reproduce():
    stored = json.load(open(make_golden.OUT))
    now = make_golden.samples()
    assert stored["workload"] == now["workload"]
    for key in ("o", "S_recv"):
        for (i1, v1), (i2, v2) in zip(stored[key], now[key]):
            assert i1 == i2
            assert abs(v1 - v2) <= 1e-12 * max(1.0, abs(v1)), (key, i1, v1, v2)
    assert abs(stored["S_final_sum"] - now["S_final_sum"]) <= 1e-10
