"""Writes oracle_small.json: oracle outputs at a few entries of a small seeded problem.

Calls only the oracle and the seeded input generator. The fixture guards the
oracle against unintended drift; its correctness rests on the pins in
tests/oracle_pins.py, not on this file.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import trimul_inputs as ti  # noqa: E402

SPEC = dict(B=2, N=6, c_z=8, c_h=6, dtype="f32", seed=5, mask=["uniform_len", 3, 6])

if __name__ == "__main__":
    inp = ti.generate(SPEC["B"], SPEC["N"], SPEC["c_z"], SPEC["c_h"], dtype=SPEC["dtype"],
                      seed=SPEC["seed"], mask=tuple(SPEC["mask"]), affine=True, biases=True)
    rng = np.random.default_rng(99)
    index = [[int(rng.integers(SPEC["B"])), int(rng.integers(SPEC["N"])), int(rng.integers(SPEC["N"])),
              int(rng.integers(SPEC["c_z"]))] for _ in range(24)]
    rec = dict(SPEC, index=index, note="written by tests/golden/make_oracle_small.py from oracle/ only")
    for d in ("outgoing", "incoming"):
        out = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps)
        rec[d] = [float(out[tuple(i)]) for i in index]
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json"), "w") as f:
        json.dump(rec, f, indent=1)
