"""Writes tests/golden/c0_oracle_samples.json from the fp64 oracle (and nothing else).

The pages print no worked example, so the stored values here are the oracle's own output on
the seeded fp32 toy workload (B=1, H=2, L=256, d=32, P=4, chunk=16): they freeze the oracle
and the input generator against silent drift.  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sequence_linear_attention_chunked_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "c0_oracle_samples.json")


def samples():
    w = WORKLOADS["C0"]
    x = make_inputs(w, "cpu")
    o, Sf, S_seg = oracle.forward(x["q"], x["k"], x["v"], x["log_g"], None, seg_len=w.L // w.P)
    rng = np.random.default_rng(1234)
    o_idx = [tuple(int(i) for i in (rng.integers(w.B), rng.integers(w.H), rng.integers(w.L),
                                    rng.integers(w.dv))) for _ in range(64)]
    s_idx = [tuple(int(i) for i in (rng.integers(w.B), rng.integers(w.H), rng.integers(w.P),
                                    rng.integers(w.dk), rng.integers(w.dv))) for _ in range(32)]
    return {
        "workload": w.describe(),
        "source": "oracle/la_oracle.c fp64 on sequence_linear_attention_chunked_b200.inputs (seed 0)",
        "o": [[list(i), float(o[i])] for i in o_idx],
        "S_recv": [[list(i), float(S_seg[i])] for i in s_idx],
        "S_final_sum": float(Sf.sum()),
    }


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(samples(), f, indent=1)
    print("wrote", OUT)
