"""tri_mul_forward_noalloc against tri_mul_forward (needs a B200).

tri_mul_forward_noalloc is for callers that cannot allocate device memory themselves,
for instance a plug-in inside a framework that owns the allocator, or a path that must
not risk an allocation failing mid-work: it keeps a, b and x in an array built into the
library instead of a caller-bound workspace. These tests call it through the C ABI and
compare it with tri_mul_forward, the entry point that uses a workspace, on two calls in
a row (the second call finds the first call's data still in the shared array). The file
is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import trimul_inputs as ti
from gpu_helpers import max_err_ratio, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


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


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    problems = [
        (ti.make_config("bf16_n256_tail10"), "outgoing"),      # a, b, x fill the whole array (48 MiB)
        (ti.generate(2, 128, 384, 128, dtype="bf16", seed=3, mask=("uniform_len", 80, 128), affine=True,
                     biases=True), "incoming"),
    ]
    for inp, direction in problems:
        z, m, w = upload(inp)
        layer = tm.TriMulLayer(w, eps=inp.eps)
        ref = layer.forward(z, m, direction)
        got = torch.full_like(ref, float("nan"))
        assert _call_noalloc(z, m, layer, direction, got) == 0, tm.load_library().tri_mul_last_error()
        torch.cuda.synchronize()
        tm.check_device_status()
        r = max_err_ratio(got.cpu().numpy(), ref.cpu().numpy())
        assert r <= TOL_BF16, f"no-allocation entry point differs from tri_mul_forward: {r:.3e} of RMS"
        print(f"N={inp.N} c_z={inp.c_z} {direction}: max|diff|/RMS = {r:.3e}, identical = {torch.equal(got, ref)}")


def test_noalloc_rejects_problems_larger_than_its_array():
    inp = ti.generate(1, 264, 128, 128, dtype="bf16", seed=1)   # 3 * 128 * 264^2 * 2 bytes > 48 MiB
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    out = torch.empty(z.shape, dtype=torch.float32, device="cuda")
    assert _call_noalloc(z, m, layer, "outgoing", out) == 4
    assert b"TRIMUL_NOALLOC_SCRATCH_BYTES" in tm.load_library().tri_mul_last_error()
