"""The pair update (outgoing then incoming update, each a masked residual) through the
C-ABI, eager and as a CUDA graph, against the fp64 oracle (needs a B200).

Tolerance, from the arithmetic of the path: each update carries the bf16-path bound of a
single update (max|err| <= 2e-2 * RMS(update)); z_mid is stored in z's dtype, so on the
bf16 path it also carries its own rounding (half a bf16 ulp: bf16 keeps 8 significant
bits, so at most 2^-8 of |z_mid|), which the second step's residual passes on to out (the
bound allows it twice, for the second update's response to it); a bf16 out adds its own
half ulp. The fp32 path keeps 1e-4 * RMS(update) per step and rounds nothing in between.
"""
import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import rms, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu


def _layers(B, N, c_z, dtype, seed, mask):
    a = ti.generate(B, N, c_z, 128, dtype=dtype, seed=seed, mask=mask, affine=True, biases=True)
    b = ti.generate(B, N, c_z, 128, dtype=dtype, seed=seed + 1, mask=mask, affine=True, biases=True)
    z, m, w_out = upload(a)
    _, _, w_in = upload(b)
    lo = tm.TriMulLayer(w_out, eps=a.eps)
    li = tm.TriMulLayer(w_in, eps=a.eps)
    return a, b.weights, z, m, lo, li


def _bound(ref_mid, ref_out, z, tol, mid_rel, out_rel):
    u1, u2 = ref_mid - z, ref_out - ref_mid
    b_mid = tol * rms(u1) + mid_rel * np.abs(ref_mid)
    b_out = tol * (rms(u1) + rms(u2)) + 2 * mid_rel * np.abs(ref_mid) + out_rel * np.abs(ref_out)
    return b_mid, b_out


@pytest.mark.parametrize("c_z,N,B,out_dtype", [(128, 96, 2, torch.float32), (128, 96, 2, torch.bfloat16),
                                               (128, 88, 2, torch.bfloat16), (384, 64, 2, torch.float32)])
def test_pair_update_bf16_against_oracle(c_z, N, B, out_dtype):
    inp, w_in, z, m, lo, li = _layers(B, N, c_z, "bf16", seed=7 * N + c_z, mask=("uniform_len", N // 2, N))
    z_mid = torch.empty_like(z)
    out = tm.pair_update(z, m, lo, li, z_mid=z_mid, out_dtype=out_dtype)
    torch.cuda.synchronize()
    tm.check_device_status()
    ref_mid, ref_out = oracle.pair_update(inp.z, inp.mask, inp.weights, w_in, inp.eps)
    z64 = np.asarray(inp.z, dtype=np.float64)
    half_ulp = 2.0 ** -8          # relative bound of half a bf16 ulp
    b_mid, b_out = _bound(ref_mid, ref_out, z64, 2e-2, half_ulp, half_ulp if out_dtype == torch.bfloat16 else 0.0)
    got_mid = z_mid.float().cpu().numpy()
    got = out.float().cpu().numpy()
    assert np.all(np.abs(got_mid - ref_mid) <= b_mid), f"z_mid: worst excess {np.max(np.abs(got_mid - ref_mid) - b_mid):.3e}"
    assert np.all(np.abs(got - ref_out) <= b_out), f"out: worst excess {np.max(np.abs(got - ref_out) - b_out):.3e}"
    masked = inp.mask == 0
    assert masked.any()
    assert np.array_equal(got_mid[masked], z64[masked]) and np.array_equal(got[masked], z64[masked])


def test_pair_update_full_size_bench_workload():
    """The bench's pair-update leg: B=1 N=512 c_z=128, bf16 z, z_mid and out, ragged mask,
    every entry against the oracle."""
    inp, w_in, z, m, lo, li = _layers(1, 512, 128, "bf16", seed=512, mask=("uniform_len", 384, 512))
    z_mid = torch.empty_like(z)
    out = tm.pair_update(z, m, lo, li, z_mid=z_mid, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    tm.check_device_status()
    ref_mid, ref_out = oracle.pair_update(inp.z, inp.mask, inp.weights, w_in, inp.eps)
    z64 = np.asarray(inp.z, dtype=np.float64)
    half_ulp = 2.0 ** -8
    b_mid, b_out = _bound(ref_mid, ref_out, z64, 2e-2, half_ulp, half_ulp)
    got_mid, got = z_mid.float().cpu().numpy(), out.float().cpu().numpy()
    assert np.all(np.abs(got_mid - ref_mid) <= b_mid), f"z_mid: worst excess {np.max(np.abs(got_mid - ref_mid) - b_mid):.3e}"
    assert np.all(np.abs(got - ref_out) <= b_out), f"out: worst excess {np.max(np.abs(got - ref_out) - b_out):.3e}"
    masked = inp.mask == 0
    assert np.array_equal(got[masked], z64[masked])


def test_pair_update_fp32_against_oracle():
    inp, w_in, z, m, lo, li = _layers(2, 48, 128, "f32", seed=5, mask=("uniform_len", 20, 48))
    out = tm.pair_update(z, m, lo, li)
    torch.cuda.synchronize()
    tm.check_device_status()
    ref_mid, ref_out = oracle.pair_update(inp.z, inp.mask, inp.weights, w_in, inp.eps)
    z64 = np.asarray(inp.z, dtype=np.float64)
    _, b_out = _bound(ref_mid, ref_out, z64, 1e-4, 0.0, 0.0)
    got = out.cpu().numpy()
    assert np.all(np.abs(got - ref_out) <= b_out), f"worst excess {np.max(np.abs(got - ref_out) - b_out):.3e}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_residual_forward_is_z_plus_update_bitwise(dtype):
    """The fused residual adds z to the same fp32 update the plain forward writes."""
    inp, _, z, m, lo, _ = _layers(1, 64, 128, dtype, seed=11, mask=("uniform_len", 40, 64))
    for d in ("outgoing", "incoming"):
        u = lo.forward(z, m, d, out_dtype=torch.float32)
        r = lo.forward(z, m, d, out_dtype=torch.float32, residual=True)
        torch.cuda.synchronize()
        assert torch.equal(r, z.float() + u), d


@pytest.mark.parametrize("N,B", [(64, 1), (88, 2)])
def test_residual_forward_bf16_out_is_rounded_z_plus_update(N, B):
    """bf16 out with the fused residual is bf16(z + update) of the same fp32 update. N=88 has
    7744 pairs per batch element: the last 128-pair tile holds 64, and the next tile belongs to
    the second element."""
    inp, _, z, m, lo, _ = _layers(B, N, 128, "bf16", seed=17 + N, mask=("uniform_len", N // 2, N))
    for d in ("outgoing", "incoming"):
        u = lo.forward(z, m, d, out_dtype=torch.float32)
        r = lo.forward(z, m, d, out_dtype=torch.bfloat16, residual=True)
        torch.cuda.synchronize()
        assert torch.equal(r, (z.float() + u).to(torch.bfloat16)), d


def test_graph_replay_equals_eager_and_follows_new_inputs():
    inp, _, z, m, lo, li = _layers(2, 64, 128, "bf16", seed=13, mask=("uniform_len", 30, 64))
    eager = tm.pair_update(z, m, lo, li, out_dtype=torch.float32).clone()
    g = tm.PairUpdateGraph(z, m, lo, li, out_dtype=torch.float32)
    got = g.launch().clone()
    torch.cuda.synchronize()
    assert torch.equal(got, eager)
    # new contents in the captured input buffer: the replay reads them
    z.copy_(torch.flip(z, dims=[1, 2]))
    m.copy_(torch.flip(m, dims=[1, 2]))
    eager2 = tm.pair_update(z, m, lo, li, out_dtype=torch.float32).clone()
    got2 = g.launch().clone()
    torch.cuda.synchronize()
    tm.check_device_status()
    assert torch.equal(got2, eager2) and not torch.equal(got2, got)
    g.close()


def test_pair_update_rejects_overlapping_buffers():
    _, _, z, m, lo, li = _layers(1, 16, 128, "bf16", seed=17, mask=("all",))
    with pytest.raises(tm.TriMulError):
        tm.pair_update(z, m, lo, li, z_mid=z)
