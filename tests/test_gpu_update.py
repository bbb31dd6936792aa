"""The whole update through tri_mul_forward against the fp64 oracle (needs a B200).

Tolerances: fp32 path max|err| <= 1e-4 * RMS(out); bf16 path (bf16 z, weights, a, b
and x, fp32 accumulation, fp32 out) max|err| <= 2e-2 * RMS(out). RMS is taken over
all compared entries of the oracle output (masked entries are 0 on both sides).
"""
import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import BF16_REL, assert_close_rms, max_err_ratio, rms, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def _run(inp, direction, out_dtype=torch.float32, use_mask=True):
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    out = layer.forward(z, m if use_mask else None, direction, out_dtype=out_dtype)
    torch.cuda.synchronize()
    tm.check_device_status()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_fp32_n64(direction):
    inp = ti.make_config("fp32_n64")
    got = _run(inp, direction)
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    r = assert_close_rms(got, ref, TOL_F32, what=f"fp32 N=64 {direction}")
    print(f"fp32_n64 {direction}: max|err|/RMS = {r:.3e}")


@pytest.mark.parametrize("name", ["bf16_n256_tail10", "bf16_n512_ragged", "bf16_b4_n256_cz384"])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_configs(name, direction):
    inp = ti.make_config(name)
    got = _run(inp, direction)
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    r = assert_close_rms(got, ref, TOL_BF16, what=f"{name} {direction}")
    valid = inp.mask[..., None].astype(bool) & np.ones_like(ref, dtype=bool)
    r_valid = float(np.max(np.abs(got - ref)[valid]) / rms(ref[valid]))
    print(f"{name} {direction}: max|err|/RMS = {r:.3e} (unmasked-only RMS: {r_valid:.3e})")
    # masked pairs are exactly zero
    assert not np.any(got[~valid])


def test_bf16_n2048_sampled_incoming_then_outgoing():
    inp = ti.make_config("bf16_n2048")
    I, J = ti.sample_indices(inp.N, 64, seed=inp.seed)
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    outs = {}
    for d in ("incoming", "outgoing"):          # back to back on the same z
        outs[d] = layer.forward(z, m, d)
    torch.cuda.synchronize()
    tm.check_device_status()
    It, Jt = torch.from_numpy(I).cuda(), torch.from_numpy(J).cuda()
    for d in ("incoming", "outgoing"):
        got = outs[d][:, It][:, :, Jt].cpu().numpy()
        ref = oracle.trimul_sampled(inp.z, inp.mask, inp.weights, d, I, J, inp.eps)
        r = assert_close_rms(got, ref, TOL_BF16, what=f"N=2048 {d} sampled")
        print(f"bf16_n2048 {d}: max|err|/RMS over 4096 sampled entries = {r:.3e}")


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_affine_layernorm_and_biases(direction):
    """Random gamma, beta and biases exercise every term of the LayerNorm folding."""
    inp = ti.generate(2, 96, 128, 128, dtype="bf16", seed=17, mask=("uniform_len", 60, 96), affine=True, biases=True)
    got = _run(inp, direction)
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    assert_close_rms(got, ref, TOL_BF16, what=f"affine {direction}")


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_output_in_bf16(direction):
    """bf16 out adds its own rounding (half an ulp of |out|) on top of the fp32-out error."""
    inp = ti.make_config("bf16_n256_tail10")
    got = _run(inp, direction, out_dtype=torch.bfloat16)
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    bound = TOL_BF16 * rms(ref) + 0.5 * BF16_REL * np.abs(ref)
    assert np.all(np.abs(got - ref) <= bound)


@pytest.mark.parametrize("N", [8, 16, 136])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_small_and_ragged_sizes(N, direction):
    inp = ti.generate(3, N, 128, 128, dtype="bf16", seed=N, mask=("uniform_len", max(1, N // 2), N), affine=True,
                      biases=True)
    got = _run(inp, direction)
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    assert_close_rms(got, ref, TOL_BF16, what=f"N={N} {direction}")


def test_fully_masked_batch_element_and_no_mask():
    inp = ti.generate(2, 32, 128, 128, dtype="bf16", seed=5, mask=("lengths", [0, 32]))
    got = _run(inp, "outgoing")
    assert not np.any(got[0]), "a fully masked element must give exact zeros"
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, "outgoing", inp.eps)
    assert_close_rms(got[1], ref[1], TOL_BF16)
    # mask=None means all ones
    inp1 = ti.generate(1, 40, 128, 128, dtype="bf16", seed=6)
    got1 = _run(inp1, "incoming", use_mask=False)
    ref1 = oracle.trimul(inp1.z, None, inp1.weights, "incoming", inp1.eps)
    assert_close_rms(got1, ref1, TOL_BF16)


def test_deterministic():
    inp = ti.generate(1, 128, 128, 128, dtype="bf16", seed=9, mask=("uniform_len", 100, 128))
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    o1 = layer.forward(z, m, "outgoing").clone()
    o2 = layer.forward(z, m, "outgoing")
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_stage_entry_points_compose_to_forward():
    """K1, K2 and K3 called one by one compute the update too. They store x without the
    per-channel offset the forward subtracts (a different rounding of the same function), so
    both are held to the oracle's bound and to each other."""
    inp = ti.generate(1, 64, 128, 128, dtype="bf16", seed=11, mask=("uniform_len", 40, 64), biases=True)
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    for d in ("outgoing", "incoming"):
        full = layer.forward(z, m, d)
        a, b = layer.project(z, m)
        scale = tm.contract_scale(z.shape[1])
        x = tm.contract(a, b, d, x_scale=scale)
        staged = layer.output_gate(z, x, m, x_scale=scale)
        torch.cuda.synchronize()
        ref = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps)
        assert_close_rms(full.cpu().numpy(), ref, TOL_BF16, what=f"forward {d}")
        assert_close_rms(staged.cpu().numpy(), ref, TOL_BF16, what=f"stages {d}")
        assert_close_rms(staged.cpu().numpy(), full.cpu().numpy().astype(np.float64), TOL_BF16, what=f"stages vs forward {d}")


def test_errors_are_reported_not_fallen_back():
    inp = ti.generate(1, 16, 256, 128, dtype="bf16", seed=1)
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)     # (256, 128) has no bf16 kernels
    with pytest.raises(tm.TriMulError) as e:
        layer.forward(z, m, "outgoing")
    assert e.value.status == 2
    inp2 = ti.generate(1, 16, 128, 128, dtype="bf16", seed=1)
    z2, m2, w2 = upload(inp2)
    layer2 = tm.TriMulLayer(w2, eps=inp2.eps)
    out = torch.empty(z2.shape, dtype=torch.float32, device="cuda")
    zp, op = tm._pair(z2), tm._pair(out)
    lib = tm.load_library()
    import ctypes
    assert lib.tri_mul_forward(ctypes.byref(zp), None, layer2.handle, 0, ctypes.byref(op), None) == 4  # no workspace
    with pytest.raises(tm.TriMulError):
        layer2.forward(z2[:, :12, :12].contiguous(), None, "outgoing")    # N not a multiple of 8
    bad_mask = torch.ones((1, 16, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        layer2.forward(z2, bad_mask, "outgoing")                            # mask dtype differs from z
