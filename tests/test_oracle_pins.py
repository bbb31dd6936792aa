"""The oracle against library routines, closed forms and invariants (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
import oracle_pins
import trimul_inputs as ti

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.load_library())


def test_golden_regression_fixture():
    """The oracle still reproduces the values its own committed script wrote (drift guard)."""
    with open(os.path.join(GOLDEN, "oracle_small.json")) as f:
        g = json.load(f)
    inp = ti.generate(g["B"], g["N"], g["c_z"], g["c_h"], dtype=g["dtype"], seed=g["seed"],
                      mask=tuple(g["mask"]), affine=True, biases=True)
    for d in ("outgoing", "incoming"):
        out = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps)
        idx = tuple(np.array(g["index"]).T)
        np.testing.assert_allclose(out[idx], np.array(g[d]), rtol=1e-12, atol=1e-14)


def test_empty_problem():
    inp = ti.generate(1, 4, 8, 8, dtype="f32", seed=1)
    out = oracle.trimul(inp.z[:, :0, :0], None, inp.weights, "outgoing")
    assert out.shape == (1, 0, 0, 8)


def test_rejects_bad_direction():
    inp = ti.generate(1, 2, 4, 4, dtype="f32", seed=1)
    with pytest.raises(KeyError):
        oracle.trimul(inp.z, inp.mask, inp.weights, "sideways")
