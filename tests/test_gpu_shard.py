"""The row-sharded update on one B200, every shard in turn (needs a B200).

Shard g runs phase 1 (K1 on its rows and the offsets pass) with its own layer handle, as a
rank would on its own GPU; then every shard runs phase 2 (the contraction reading all shards'
a and b, and K3 on its rows). The shards' rows of the update, put together, must match the
fp64 oracle on the whole pair tensor to the 2e-2 RMS bound, in both directions, for even and
uneven splits, c_z 128 and 384, and padding masks.
"""
import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import assert_close_rms, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _run_shards(inp, direction, G, bounds=None):
    z, m, w = upload(inp)
    N = inp.N
    bounds = bounds or tm.shard_bounds(N, G)
    layers = [tm.TriMulLayer(w, eps=inp.eps) for _ in range(G)]
    zs = [z[:, bounds[g]:bounds[g + 1]].contiguous() for g in range(G)]
    ms = [m[:, bounds[g]:bounds[g + 1]].contiguous() for g in range(G)]
    ab = [layers[g].shard_project(zs[g], ms[g], bounds[g], N) for g in range(G)]
    a_all = [x[0] for x in ab]
    b_all = [x[1] for x in ab]
    outs = [layers[g].shard_finish(zs[g], ms[g], bounds[g], N, direction, bounds,
                                   a_all if direction == "incoming" else [a_all[h] if h == g else None for h in range(G)],
                                   b_all) for g in range(G)]
    torch.cuda.synchronize()
    tm.check_device_status()
    full = layers[0]
    return torch.cat(outs, dim=1).cpu().numpy(), z, m, full


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
@pytest.mark.parametrize("N,G,c_z,bounds", [
    (256, 2, 128, None),
    (512, 4, 128, None),
    (384, 2, 128, [0, 256, 384]),      # uneven shards
    (256, 2, 384, None),
])
def test_shards_match_the_oracle(direction, N, G, c_z, bounds):
    B = 2 if c_z == 384 else 1
    inp = ti.generate(B, N, c_z, 128, dtype="bf16", seed=N + G + c_z, z_std=0.5 if c_z == 384 else 1.0,
                      mask=("uniform_len", N * 3 // 4, N), biases=True)
    got, z, m, layer = _run_shards(inp, direction, G, bounds)
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    r = assert_close_rms(got, ref, TOL_BF16, what=f"N={N} G={G} c_z={c_z} {direction}")
    valid = inp.mask.astype(bool)
    assert not np.any(got[~valid]), "masked pairs must be exactly 0"
    print(f"N={N} G={G} c_z={c_z} {direction}: max|err|/RMS = {r:.3e}")


def test_shards_match_the_unsharded_forward_with_common_mode():
    inp = ti.generate(1, 512, 128, 128, dtype="bf16", seed=31, mask=("uniform_len", 384, 512))
    w = dict(inp.weights)
    for k in ("b_ap", "b_bp"):
        w[k] = ti.round_to_bf16(np.full_like(w[k], 3.0))
    inp.weights = w
    for d in ("outgoing", "incoming"):
        got, z, m, layer = _run_shards(inp, d, 2)
        ref = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps)
        assert_close_rms(got, ref, TOL_BF16, what=f"sharded common mode {d}")
        dense = layer.forward(z, m, d).cpu().numpy()
        assert_close_rms(got, dense.astype(np.float64), TOL_BF16, what=f"sharded vs unsharded {d}")


def test_phase_two_rejects_a_bad_shard_table():
    inp = ti.generate(1, 256, 128, 128, dtype="bf16", seed=3)
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    zs = z[:, :128].contiguous()
    a, b = layer.shard_project(zs, m[:, :128].contiguous(), 0, 256)
    for bounds, status in (([0, 128, 200], 1), ([0, 100, 256], 2), ([0, 128], 1)):
        with pytest.raises(tm.TriMulError) as e:
            layer.shard_finish(zs, m[:, :128].contiguous(), 0, 256, "outgoing", bounds, [a, None, None][:len(bounds) - 1],
                               [b, b, b][:len(bounds) - 1])
        assert e.value.status == status, (bounds, e.value)
