"""Writes tests/golden/*.json: input digests of the seeded workloads and a few oracle
values of the small ungated fp32 workload (B=1 H=1 L=256 Dk=Dv=64, C=64, seed 0).

Run from the repository root: python tests/golden/make_golden.py
It calls only the input generator and oracle/ (never the CUDA library). The stored
values are regression fixtures for the generator and the oracle; their correctness
comes from the pins in tests/test_oracle_pins.py, not from this file.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from linear_rnn_b200 import inputs as I  # noqa: E402

OUT = os.path.dirname(os.path.abspath(__file__))
SAMPLE_ROWS = [0, 1, 63, 64, 127, 200, 255]


def main():
    w = I.WORKLOADS["c1"]
    x = I.make_inputs(w, seed=0)
    o, hT = oracle.gla_fwd(x["q"], x["k"], x["v"], None, None, None, w.scale)
    rec = {
        "workload": "c1: ungated causal linear attention, fp32, B=1 H=1 L=256 Dk=Dv=64, seed 0",
        "input_sha256": I.input_digest(x),
        "o_rows": {str(r): o[0, 0, r, :8].tolist() for r in SAMPLE_ROWS},
        "o_abs_max": float(np.abs(o).max()),
        "hT_trace": float(np.trace(hT[0, 0])),
        "hT_abs_max": float(np.abs(hT).max()),
    }
    with open(os.path.join(OUT, "c1_oracle.json"), "w") as f:
        json.dump(rec, f, indent=1)
    digests = {}
    for name, wl in I.WORKLOADS.items():
        small = I.small(wl)
        digests[name + "-small"] = {"B": small.B, "H": small.H, "L": small.L,
                                    "sha256": I.input_digest(I.make_inputs(small, seed=0))}
    with open(os.path.join(OUT, "input_digests.json"), "w") as f:
        json.dump(digests, f, indent=1)


if __name__ == "__main__":
    main()
