"""A bounded device wait that runs out is reported on the host and leaves the GPU usable.

The self-test kernel waits on an mbarrier that nothing arrives at; after about one
second the wait gives up, sets the library's device error word and the kernel returns.
No fault, trap or unbounded wait is involved.
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


def test_timed_out_wait_is_reported_and_the_context_survives():
    lib = tm.load_library()
    lib.tri_mul_selftest_bounded_wait.argtypes = [ctypes.c_void_p]
    lib.tri_mul_selftest_bounded_wait.restype = ctypes.c_int
    tm.check_device_status()                       # clean start
    assert lib.tri_mul_selftest_bounded_wait(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    with pytest.raises(tm.TriMulError) as e:
        tm.check_device_status()
    assert e.value.status == 6                     # TRIMUL_ERR_DEVICE_TIMEOUT
    tm.check_device_status()                       # the word was cleared
    # the device still computes correctly afterwards
    inp = ti.generate(1, 32, 128, 128, dtype="bf16", seed=2, mask=("uniform_len", 20, 32))
    z, m, w = upload(inp)
    out = tm.TriMulLayer(w, eps=inp.eps).forward(z, m, "outgoing")
    torch.cuda.synchronize()
    tm.check_device_status()
    ref = oracle.trimul(inp.z, inp.mask, inp.weights, "outgoing", inp.eps)
    assert_close_rms(out.cpu().numpy(), ref, 2e-2)
