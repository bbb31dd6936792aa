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
    """The oracle still reproduces the values its own committed script wrote (drift guard):
    the update in both directions, the pair update and the pair transition."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_oracle_small", os.path.join(GOLDEN, "make_oracle_small.py"))
    maker = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(maker)
    with open(os.path.join(GOLDEN, "oracle_small.json")) as f:
        g = json.load(f)
    idx = tuple(np.array(g["index"]).T)
    vals = maker.oracle_values({k: g[k] for k in ("B", "N", "c_z", "c_h", "dtype", "seed", "mask")})
    keys = ("outgoing", "incoming", "pair_update_mid", "pair_update_out", "pair_transition")
    assert set(keys) <= set(g) and set(vals) == set(keys)
    for k in keys:
        np.testing.assert_allclose(vals[k][idx], np.array(g[k]), rtol=1e-12, atol=1e-14, err_msg=k)


def test_empty_problem():
    inp = ti.generate(1, 4, 8, 8, dtype="f32", seed=1)
    out = oracle.trimul(inp.z[:, :0, :0], None, inp.weights, "outgoing")
    assert out.shape == (1, 0, 0, 8)


def test_rejects_bad_direction():
    inp = ti.generate(1, 2, 4, 4, dtype="f32", seed=1)
    with pytest.raises(KeyError):
        oracle.trimul(inp.z, inp.mask, inp.weights, "sideways")
