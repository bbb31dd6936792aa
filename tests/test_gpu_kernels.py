"""Each CUDA kernel against the fp64 oracle on independent seeded inputs (needs a B200).

K2 (contraction) gets random 16-bit a, b; K1 (projection) and K3 (output gate) get
seeded z, x and weights. No input or expected value comes from another kernel.
"""
import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import F16_REL, assert_close_bf16, assert_close_f16, assert_close_rms, assert_close_ulp, to_pair_major, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu


def _round(x, dtype):
    if dtype == torch.bfloat16:
        return ti.round_to_bf16(x)
    if dtype == torch.float16:
        return x.astype(np.float16).astype(np.float32)
    return x


def _rand_planes(B, C, N, seed, dtype=torch.float16, scale=1.0):
    g = np.random.default_rng(seed)
    a = _round((g.standard_normal((B, C, N, N)) * scale).astype(np.float32), dtype)
    b = _round((g.standard_normal((B, C, N, N)) * scale).astype(np.float32), dtype)
    return torch.from_numpy(a).cuda().to(dtype), torch.from_numpy(b).cuda().to(dtype)


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("B,C,N", [(1, 2, 8), (1, 3, 64), (2, 2, 136), (1, 2, 256), (1, 1, 328), (1, 2, 512)])
def test_contract_tensor_cores(direction, dtype, B, C, N):
    a, b = _rand_planes(B, C, N, seed=N + C, dtype=dtype)
    scale = tm.contract_scale(N) if dtype == torch.float16 else 1.0
    x = tm.contract(a, b, direction, x_scale=scale)
    torch.cuda.synchronize()
    ref = oracle.contract(to_pair_major(a), to_pair_major(b), direction) * scale
    # fp32 accumulation of exact 16-bit products, exact power-of-two scaling, one rounding
    check = assert_close_f16 if dtype == torch.float16 else assert_close_bf16
    check(to_pair_major(x), ref, 1e-4, what=f"K2 {direction} {dtype} N={N}")
    tm.check_device_status()


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
@pytest.mark.parametrize("B,C,N", [(1, 2, 8), (2, 3, 72), (1, 2, 200)])
def test_contract_f32(direction, B, C, N):
    a, b = _rand_planes(B, C, N, seed=7 * N, dtype=torch.float32)
    x = tm.contract(a, b, direction, x_scale=0.5)
    ref = oracle.contract(to_pair_major(a), to_pair_major(b), direction) * 0.5
    assert_close_rms(to_pair_major(x), ref, 1e-5, what=f"fp32 K2 {direction} N={N}")


def _layer_inputs(B, N, c_z, dtype, seed, mask, affine):
    inp = ti.generate(B, N, c_z, 128, dtype=dtype, seed=seed, mask=mask, affine=affine, biases=True)
    z, m, w = upload(inp)
    return inp, z, m, w


def _oracle_ab(inp):
    w = inp.weights
    zh = oracle.layernorm(inp.z, w["ln_in_g"], w["ln_in_b"], inp.eps)
    a = oracle.gated_projection(zh, inp.mask, w["w_ag"], w["b_ag"], w["w_ap"], w["b_ap"])
    b = oracle.gated_projection(zh, inp.mask, w["w_bg"], w["b_bg"], w["w_bp"], w["b_bp"])
    return zh, a, b


SIZES = [(1, 8, ("all",)), (2, 40, ("uniform_len", 20, 40)), (1, 136, ("lengths", [100])),
         (1, 256, ("tail_fraction", 0.1))]


@pytest.mark.parametrize("c_z", [128, 384])
@pytest.mark.parametrize("affine", [False, True])
@pytest.mark.parametrize("B,N,mask", SIZES)
def test_project_bf16(c_z, affine, B, N, mask):
    inp, z, m, w = _layer_inputs(B, N, c_z, "bf16", seed=N + c_z, mask=mask, affine=affine)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    a, b = layer.project(z, m)
    torch.cuda.synchronize()
    assert a.dtype == torch.float16
    _, ra, rb = _oracle_ab(inp)
    # gamma = 1: the folded weights are exact; the tanh-based gate adds < 1e-3 of RMS.
    # random gamma: W * gamma is rounded to bf16 (up to 2^-9 per weight), which the
    # end-to-end tolerance absorbs; checked here at that tolerance.
    tol = 2e-2 if affine else 2e-3
    # c_z = 128 evaluates sigmoid(g) * p * m in f16x2: up to ~3 half-precision roundings
    rel = (4 if c_z == 128 else 1) * F16_REL
    assert_close_ulp(to_pair_major(a), ra, tol, rel, what=f"K1 a c_z={c_z} N={N}")
    assert_close_ulp(to_pair_major(b), rb, tol, rel, what=f"K1 b c_z={c_z} N={N}")
    tm.check_device_status()


@pytest.mark.parametrize("c_z", [128, 384])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("affine", [False, True])
@pytest.mark.parametrize("B,N,mask", SIZES)
def test_output_gate_bf16(c_z, out_dtype, affine, B, N, mask):
    inp, z, m, w = _layer_inputs(B, N, c_z, "bf16", seed=3 * N + c_z, mask=mask, affine=affine)
    scale = tm.contract_scale(N)
    # stored x (fp16) holds scale * x; the oracle gets the unscaled x (exact: scale is 2^-k)
    xs = (np.random.default_rng(N).standard_normal((B, 128, N, N)) * 3.0).astype(np.float16).astype(np.float32)
    x = torch.from_numpy(xs).cuda().to(torch.float16)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    out = layer.output_gate(z, x, m, out_dtype=out_dtype, x_scale=scale)
    torch.cuda.synchronize()
    wt = inp.weights
    zh = oracle.layernorm(inp.z, wt["ln_in_g"], wt["ln_in_b"], inp.eps)
    ref = oracle.output_gate(zh, np.transpose(xs, (0, 2, 3, 1)).astype(np.float64) / scale, inp.mask, wt["w_g"],
                             wt["b_g"], wt["ln_out_g"], wt["ln_out_b"], inp.eps, wt["w_o"], wt["b_o"])
    got = out.float().cpu().numpy()
    tol = 2e-2 if affine else 2e-3
    if out_dtype == torch.float32:
        assert_close_rms(got, ref, tol, what=f"K3 c_z={c_z} N={N}")
    else:
        assert_close_bf16(got, ref, tol, what=f"K3 bf16-out c_z={c_z} N={N}")
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
    out = layer.output_gate(z, x, m, x_scale=0.25)
    wt = inp.weights
    ref = oracle.output_gate(zh, np.transpose(gx, (0, 2, 3, 1)).astype(np.float64) * 4.0, inp.mask, wt["w_g"],
                             wt["b_g"], wt["ln_out_g"], wt["ln_out_b"], inp.eps, wt["w_o"], wt["b_o"])
    assert_close_rms(out.cpu().numpy(), ref, 1e-5, what="fp32 K3")
