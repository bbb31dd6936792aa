"""The bench's context figure (an eager PyTorch composition of the update) computes the same
update as the oracle: fp64 on the CPU, both directions, affine LayerNorms, biases and a ragged
mask."""
import numpy as np
import pytest
import torch

import bench
import oracle
import trimul_inputs as ti


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_torch_composition_is_the_update(direction):
    inp = ti.generate(2, 9, 12, 10, dtype="f32", seed=5, mask=("uniform_len", 5, 9), affine=True, biases=True)
    w = {k: (None if v is None else torch.as_tensor(np.asarray(v, dtype=np.float64))) for k, v in inp.weights.items()}
    z = torch.as_tensor(np.asarray(inp.z, dtype=np.float64))
    m = torch.as_tensor(np.asarray(inp.mask, dtype=np.float64))
    got = bench.torch_composition(z, m, w, direction, inp.eps).numpy()
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))


def test_torch_composition_without_mask():
    inp = ti.generate(1, 6, 8, 6, dtype="f32", seed=6, affine=True, biases=True)
    w = {k: (None if v is None else torch.as_tensor(np.asarray(v, dtype=np.float64))) for k, v in inp.weights.items()}
    got = bench.torch_composition(torch.as_tensor(np.asarray(inp.z, dtype=np.float64)), None, w, "outgoing", inp.eps)
    ref = oracle.trimul(inp.z, None, inp.weights, "outgoing", inp.eps)
    assert np.max(np.abs(got.numpy() - ref)) <= 1e-10 * np.max(np.abs(ref))
