"""Each CUDA kernel against the fp64 oracle on independent seeded inputs (needs a B200).

K2 (contraction) gets random bf16 a, b; K1 (projection) and K3 (output gate) get seeded
z, x and weights. No input or expected value comes from another kernel.
"""
import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import assert_close_bf16, assert_close_rms, to_pair_major, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu


def _rand_planes(B, C, N, seed, dtype=torch.bfloat16, scale=1.0):
    g = np.random.default_rng(seed)
    a = (g.standard_normal((B, C, N, N)) * scale).astype(np.float32)
    b = (g.standard_normal((B, C, N, N)) * scale).astype(np.float32)
    if dtype == torch.bfloat16:
        a, b = ti.round_to_bf16(a), ti.round_to_bf16(b)
    return torch.from_numpy(a).cuda().to(dtype), torch.from_numpy(b).cuda().to(dtype)


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
@pytest.mark.parametrize("B,C,N", [(1, 2, 8), (1, 3, 64), (2, 2, 136), (1, 2, 256), (1, 1, 328), (1, 2, 512)])
def test_contract_bf16(direction, B, C, N):
    a, b = _rand_planes(B, C, N, seed=N + C)
    x = tm.contract(a, b, direction)
    torch.cuda.synchronize()
    ref = oracle.contract(to_pair_major(a), to_pair_major(b), direction)
    # fp32 accumulation of exact bf16 products, then one bf16 rounding of x
    assert_close_bf16(to_pair_major(x), ref, 1e-4, what=f"K2 {direction} N={N}")
    tm.check_device_status()


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
@pytest.mark.parametrize("B,C,N", [(1, 2, 8), (2, 3, 72), (1, 2, 200)])
def test_contract_f32(direction, B, C, N):
    a, b = _rand_planes(B, C, N, seed=7 * N, dtype=torch.float32)
    x = tm.contract(a, b, direction)
    ref = oracle.contract(to_pair_major(a), to_pair_major(b), direction)
    assert_close_rms(to_pair_major(x), ref, 1e-5, what=f"fp32 K2 {direction} N={N}")


def _layer_inputs(B, N, c_z, dtype, seed, mask=("uniform_len", 5, 8), affine=True, biases=True):
    inp = ti.generate(B, N, c_z, 128, dtype=dtype, seed=seed, mask=mask, affine=affine, biases=biases)
    z, m, w = upload(inp)
    return inp, z, m, w


def _oracle_ab(inp):
    w = inp.weights
    zh = oracle.layernorm(inp.z, w["ln_in_g"], w["ln_in_b"], inp.eps)
    a = oracle.gated_projection(zh, inp.mask, w["w_ag"], w["b_ag"], w["w_ap"], w["b_ap"])
    b = oracle.gated_projection(zh, inp.mask, w["w_bg"], w["b_bg"], w["w_bp"], w["b_bp"])
    return zh, a, b


@pytest.mark.parametrize("c_z", [128, 384])
@pytest.mark.parametrize("B,N,mask", [(1, 8, ("all",)), (2, 40, ("uniform_len", 20, 40)), (1, 136, ("lengths", [100])),
                                      (1, 256, ("tail_fraction", 0.1))])
def test_project_bf16(c_z, B, N, mask):
    inp, z, m, w = _layer_inputs(B, N, c_z, "bf16", seed=N + c_z, mask=mask)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    a, b = layer.project(z, m)
    torch.cuda.synchronize()
    _, ra, rb = _oracle_ab(inp)
    # a, b are stored bf16; the tanh-based gate adds well under 1e-3 of RMS
    assert_close_bf16(to_pair_major(a), ra, 3e-3, what=f"K1 a c_z={c_z} N={N}")
    assert_close_bf16(to_pair_major(b), rb, 3e-3, what=f"K1 b c_z={c_z} N={N}")
    tm.check_device_status()


@pytest.mark.parametrize("c_z", [128, 384])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,N,mask", [(1, 8, ("all",)), (2, 48, ("uniform_len", 20, 48)), (1, 136, ("lengths", [130])),
                                      (1, 256, ("tail_fraction", 0.1))])
def test_output_gate_bf16(c_z, out_dtype, B, N, mask):
    inp, z, m, w = _layer_inputs(B, N, c_z, "bf16", seed=3 * N + c_z, mask=mask)
    gx = np.random.default_rng(N).standard_normal((B, 128, N, N)).astype(np.float32) * 3.0
    gx = ti.round_to_bf16(gx)
    x = torch.from_numpy(gx).cuda().to(torch.bfloat16)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    out = layer.output_gate(z, x, m, out_dtype=out_dtype)
    torch.cuda.synchronize()
    wt = inp.weights
    zh = oracle.layernorm(inp.z, wt["ln_in_g"], wt["ln_in_b"], inp.eps)
    ref = oracle.output_gate(zh, np.transpose(gx, (0, 2, 3, 1)), inp.mask, wt["w_g"], wt["b_g"], wt["ln_out_g"],
                             wt["ln_out_b"], inp.eps, wt["w_o"], wt["b_o"])
    got = out.float().cpu().numpy()
    if out_dtype == torch.float32:
        # folded LayerNorms in fp32, bf16 weights after gamma folding: far inside 2e-2 * RMS
        assert_close_rms(got, ref, 5e-3, what=f"K3 c_z={c_z} N={N}")
    else:
        assert_close_bf16(got, ref, 5e-3, what=f"K3 bf16-out c_z={c_z} N={N}")
    tm.check_device_status()


@pytest.mark.parametrize("c_z,c_h", [(128, 128), (64, 96), (384, 128)])
def test_fp32_project_and_output(c_z, c_h):
    inp = ti.generate(2, 24, c_z, c_h, dtype="f32", seed=c_z + c_h, mask=("uniform_len", 10, 24), affine=True,
                      biases=True)
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    a, b = layer.project(z, m)
    zh, ra, rb = _oracle_ab(inp)
    assert_close_rms(to_pair_major(a), ra, 1e-5, what="fp32 K1 a")
    assert_close_rms(to_pair_major(b), rb, 1e-5, what="fp32 K1 b")
    gx = np.random.default_rng(5).standard_normal((2, c_h, 24, 24)).astype(np.float32)
    x = torch.from_numpy(gx).cuda()
    out = layer.output_gate(z, x, m)
    wt = inp.weights
    ref = oracle.output_gate(zh, np.transpose(gx, (0, 2, 3, 1)), inp.mask, wt["w_g"], wt["b_g"], wt["ln_out_g"],
                             wt["ln_out_b"], inp.eps, wt["w_o"], wt["b_o"])
    assert_close_rms(out.cpu().numpy(), ref, 1e-5, what="fp32 K3")
