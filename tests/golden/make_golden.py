"""Writes tests/golden/tiny_mha_rows.json from the oracle alone.

The fixture is a regression guard on the oracle's arithmetic for the tiny
MHA workload (B=1, H=2, L=128, D=64, non-causal, scale 1/8, seed 1000): the
first four output features and the LSE of a few rows of both heads.  It calls
only ``oracle`` and the seeded input generator.  Run from the repo root:
``python tests/golden/make_golden.py``.
"""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))

import oracle  # noqa: E402
from workloads import TINY_MHA, prefill_inputs, seed_of  # noqa: E402

ROWS = [0, 1, 63, 64, 127]


def main():
    q, k, v = prefill_inputs(TINY_MHA, seed_of(0))
    o, lse = oracle.attention(q, k, v, TINY_MHA.scale, False, rows=ROWS)
    out = {
        "workload": TINY_MHA.name,
        "seed": seed_of(0),
        "rows": ROWS,
        "o_first4": o[0, :, :, :4].tolist(),
        "lse": lse[0].tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_mha_rows.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
