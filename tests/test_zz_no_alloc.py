"""tri_mul_forward_noalloc against tri_mul_forward and the oracle (needs a B200).

tri_mul_forward_noalloc is for callers that cannot allocate device memory themselves,
for instance a plug-in inside a framework that owns the allocator, or a path that must
not risk an allocation failing mid-work: it keeps the intermediates in an array built into
the library instead of a caller-bound workspace. Both entry points launch the same
deterministic kernels on the same inputs, so their outputs must agree bit for bit. These
tests call it through the C ABI on two calls in a row (the second call finds the first
call's data still in the shared array), on the bf16 path at c_z 128 and 384 and on the fp32
path, and hold one problem to the oracle's bound as well. The file is named so that pytest
collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import assert_close_rms, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
TOL_F32 = 1e-4


def _noalloc_fn():
    fn = tm.load_library().tri_mul_forward_noalloc
    fn.argtypes = [ctypes.POINTER(tm._Pair), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                   ctypes.POINTER(tm._Pair), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _call_noalloc(z, mask, layer, direction, out):
    zp, op = tm._pair(z), tm._pair(out)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _noalloc_fn()(ctypes.byref(zp), None if mask is None else mask.data_ptr(), layer.handle,
                         tm._DIRS[direction], ctypes.byref(op), stream)


PROBLEMS = [
    # the array's full size: a, b, x of B=1 N=256 c_h=128 take 48 MiB
    ("bf16 N=256 c_z=128", lambda: ti.make_config("bf16_n256_tail10"), ("outgoing", "incoming")),
    ("bf16 B=2 N=128 c_z=384", lambda: ti.generate(2, 128, 384, 128, dtype="bf16", seed=3,
                                                    mask=("uniform_len", 80, 128), affine=True, biases=True),
     ("incoming", "outgoing")),
    ("fp32 N=64", lambda: ti.make_config("fp32_n64"), ("outgoing", "incoming")),
]


@pytest.mark.parametrize("name,make,directions", PROBLEMS, ids=[p[0] for p in PROBLEMS])
def test_noalloc_equals_forward_on_two_calls_in_a_row(name, make, directions):
    inp = make()
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    for direction in directions:                 # two calls in a row, the second over the first's data
        ref = layer.forward(z, m, direction)
        got = torch.full_like(ref, float("nan"))
        assert _call_noalloc(z, m, layer, direction, got) == 0, tm.load_library().tri_mul_last_error()
        torch.cuda.synchronize()
        tm.check_device_status()
        assert torch.equal(got, ref), f"{name} {direction}: the no-allocation result differs from tri_mul_forward"


def test_noalloc_matches_the_oracle():
    inp = ti.make_config("bf16_n256_tail10")
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    for direction in ("incoming", "outgoing"):
        got = torch.empty(z.shape, dtype=torch.float32, device="cuda")
        assert _call_noalloc(z, m, layer, direction, got) == 0, tm.load_library().tri_mul_last_error()
        torch.cuda.synchronize()
        tm.check_device_status()
        ref = oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
        assert_close_rms(got.cpu().numpy(), ref, TOL_BF16, what=f"no-allocation {direction}")
    inp32 = ti.make_config("fp32_n64")
    z, m, w = upload(inp32)
    layer = tm.TriMulLayer(w, eps=inp32.eps)
    got = torch.empty(z.shape, dtype=torch.float32, device="cuda")
    assert _call_noalloc(z, m, layer, "outgoing", got) == 0, tm.load_library().tri_mul_last_error()
    torch.cuda.synchronize()
    ref = oracle.trimul(inp32.z, inp32.mask, inp32.weights, "outgoing", inp32.eps)
    assert_close_rms(got.cpu().numpy(), ref, TOL_F32, what="no-allocation fp32")


def test_noalloc_rejects_problems_larger_than_its_array():
    inp = ti.generate(1, 264, 128, 128, dtype="bf16", seed=1)   # 3 * 128 * 264^2 * 2 bytes > the array
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    out = torch.full(z.shape, 7.0, dtype=torch.float32, device="cuda")
    assert _call_noalloc(z, m, layer, "outgoing", out) == 4
    assert b"TRIMUL_NOALLOC_SCRATCH_BYTES" in tm.load_library().tri_mul_last_error()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()), "a rejected call must not write out"
