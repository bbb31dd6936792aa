"""Writes oracle_small.json: oracle outputs at a few entries of a small seeded problem.

Calls only the oracle and the seeded input generator. The fixture guards the
oracle against unintended drift; its correctness rests on the pins in
tests/oracle_pins.py, not on this file.

Entries: the update in both directions; the pair update (z_mid and out) with a second
layer drawn from seed + 1; the pair transition with weights from transition_weights().
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
HIDDEN = 16


def problem(spec, seed_offset=0):
    return ti.generate(spec["B"], spec["N"], spec["c_z"], spec["c_h"], dtype=spec["dtype"],
                       seed=spec["seed"] + seed_offset, mask=tuple(spec["mask"]), affine=True, biases=True)


def transition_weights(c, hidden, seed=101):
    """W1 [hidden, c], b1, W2 [c, hidden], b2 from a fixed seed (N(0, 1/fan_in) weights,
    N(0, 0.1^2) biases)."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((hidden, c)) / np.sqrt(c), 0.1 * rng.standard_normal(hidden),
            rng.standard_normal((c, hidden)) / np.sqrt(hidden), 0.1 * rng.standard_normal(c))


def oracle_values(spec):
    """The oracle's values for every fixture key, as full arrays."""
    inp = problem(spec)
    vals = {d: oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps) for d in ("outgoing", "incoming")}
    z_mid, out = oracle.pair_update(inp.z, inp.mask, inp.weights, problem(spec, 1).weights, inp.eps)
    vals["pair_update_mid"], vals["pair_update_out"] = z_mid, out
    vals["pair_transition"] = oracle.pair_transition(inp.z, inp.mask, *transition_weights(spec["c_z"], HIDDEN))
    return vals


if __name__ == "__main__":
    rng = np.random.default_rng(99)
    index = [[int(rng.integers(SPEC["B"])), int(rng.integers(SPEC["N"])), int(rng.integers(SPEC["N"])),
              int(rng.integers(SPEC["c_z"]))] for _ in range(24)]
    rec = dict(SPEC, index=index, note="written by tests/golden/make_oracle_small.py from oracle/ only")
    for key, arr in oracle_values(SPEC).items():
        rec[key] = [float(arr[tuple(i)]) for i in index]
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json"), "w") as f:
        json.dump(rec, f, indent=1)
