"""The C-ABI library builds, loads and exports what include/trimul.h declares (no GPU needed).

Only calls that are answered on the host before any CUDA work are made here: status
strings, version queries and argument validation that must fail before a launch.
"""
import ctypes
import os
import re

import pytest

from protein_pair_representation_b200 import build
from protein_pair_representation_b200 import trimul as tm

HEADER = os.path.join(build.ROOT, "include", "trimul.h")


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return tm.load_library()


def declared_functions():
    with open(HEADER) as f:
        src = f.read()
    return sorted(set(re.findall(r"\b(tri_mul_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("tri_mul_forward", "tri_mul_layer_create", "tri_mul_layer_destroy", "tri_mul_project",
                 "tri_mul_contract", "tri_mul_output_gate", "tri_mul_workspace_bytes",
                 "tri_mul_layer_bind_workspace", "tri_mul_check_device_status"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_library_is_built_for_sm100a(lib):
    # the fatbin must carry sm_100a code: cuobjdump is not used; nvcc's -gencode list is the record
    assert "arch=compute_100a,code=sm_100a" in build.NVCC_FLAGS


def test_status_strings_and_versions(lib):
    for code in range(9):
        assert lib.tri_mul_status_string(code)
    assert lib.tri_mul_status_string(99) == b"unknown status"
    assert lib.tri_mul_abi_version() == 103
    assert lib.tri_mul_kernels_per_forward() == 4


def test_null_arguments_are_rejected_on_the_host(lib):
    handle = ctypes.c_void_p()
    assert lib.tri_mul_layer_create(None, None, ctypes.byref(handle)) == 1
    z = tm._Pair(0, 1, 8, 128, tm.BF16)
    out = tm._Pair(0, 1, 8, 128, tm.F32)
    assert lib.tri_mul_forward(ctypes.byref(z), None, None, 0, ctypes.byref(out), None) == 1
    assert b"z: NULL tensor" in lib.tri_mul_last_error()
    z = tm._Pair(1 << 24, 1, 8, 128, tm.BF16)        # aligned, never dereferenced
    assert lib.tri_mul_forward(ctypes.byref(z), None, None, 0, ctypes.byref(out), None) == 1
    assert b"out: NULL tensor" in lib.tri_mul_last_error()
    out = tm._Pair(1 << 30, 1, 8, 128, tm.F32)
    assert lib.tri_mul_forward(ctypes.byref(z), None, None, 0, ctypes.byref(out), None) == 1
    assert b"layer is NULL" in lib.tri_mul_last_error()


def test_forward_validates_sizes_before_the_layer(lib):
    """N a multiple of 8 in [8, 16384]; on the bf16 path B * N^2 / 128 tiles at most 2^30
    (int tile indices in the kernels). Checked before the layer and any device call."""
    def status(B, N, dtype=tm.BF16):
        z = tm._Pair(1 << 24, B, N, 128, dtype)
        out = tm._Pair(1 << 46, B, N, 128, tm.F32)
        return lib.tri_mul_forward(ctypes.byref(z), None, None, 0, ctypes.byref(out), None)
    assert status(1, 4) == 2
    assert status(1, 100) == 2
    assert status(1, 16392) == 2 and b"exceeds 16384" in lib.tri_mul_last_error()
    assert status(513, 16384) == 2 and b"too large" in lib.tri_mul_last_error()
    assert status(513, 16384, tm.F32) == 1               # the fp32 path has no tile limit
    assert status(512, 16384) == 1 and b"layer is NULL" in lib.tri_mul_last_error()


def test_contract_validation_happens_before_any_launch(lib):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    # N not a multiple of 8
    assert lib.tri_mul_contract(fake, fake, fake, 1, 4, 12, tm.F16, 0, 1.0, None) == 2
    # unknown direction
    assert lib.tri_mul_contract(fake, fake, fake, 1, 4, 16, tm.F16, 7, 1.0, None) == 1
    # misaligned pointer
    bad = ctypes.c_void_p((1 << 20) + 8)
    assert lib.tri_mul_contract(bad, fake, ctypes.c_void_p(1 << 24), 1, 4, 16, tm.F16, 0, 1.0, None) == 7
    # x overlapping a
    assert lib.tri_mul_contract(fake, ctypes.c_void_p(1 << 24), fake, 1, 4, 16, tm.BF16, 0, 1.0, None) == 1
    # too many channels for the grid
    assert lib.tri_mul_contract(fake, ctypes.c_void_p(1 << 30), ctypes.c_void_p(1 << 34), 1, 70000, 16, tm.F32, 0,
                                1.0, None) == 2
    # scale must be positive
    assert lib.tri_mul_contract(fake, ctypes.c_void_p(1 << 30), ctypes.c_void_p(1 << 34), 1, 4, 16, tm.F16, 0,
                                0.0, None) == 1


def test_contract_scale_is_a_power_of_two_near_inverse_sqrt_n(lib):
    import math
    for N, expect in ((1, 1.0), (8, 0.25), (64, 0.125), (256, 1 / 16), (512, 1 / 32), (2048, 1 / 64)):
        s = lib.tri_mul_contract_scale(N)
        assert s == expect, (N, s)
        assert math.log2(s) == int(math.log2(s))
    assert lib.tri_mul_contract_scale(0) == 0.0


def test_layer_create_rejects_bad_widths_before_allocating(lib):
    desc = tm._WeightsDesc()
    desc.c_z, desc.c_h, desc.dtype, desc.eps = 100, 128, tm.BF16, 1e-5
    handle = ctypes.c_void_p()
    assert lib.tri_mul_layer_create(ctypes.byref(desc), None, ctypes.byref(handle)) == 2
    desc.c_z, desc.eps = 128, 0.0
    assert lib.tri_mul_layer_create(ctypes.byref(desc), None, ctypes.byref(handle)) == 1


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="would launch on fake pointers")
def test_adjacent_f16_planes_pass_validation(lib):
    """Planes placed back to back (2 bytes per element for F16) do not count as overlapping:
    validation passes and the call only fails later, at the CUDA device query, on a GPU-less host."""
    B, C, N = 1, 4, 16
    plane = B * C * N * N * 2
    a, b, x = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + plane), ctypes.c_void_p((1 << 20) + 2 * plane)
    st = lib.tri_mul_contract(a, b, x, B, C, N, tm.F16, 0, 1.0, None)
    assert st in (3, 5), lib.tri_mul_last_error()


def test_transition_validates_sizes_on_the_host(lib):
    """Size rules are checked before the handle and before any device call: N a multiple of
    8 in [8, 16384] (int pair coordinates in the kernel), B * N^2 / 64 tiles below 2^31."""
    fake = 1 << 24                             # aligned, never dereferenced
    def status(B, N, dtype=tm.BF16):
        z = tm._Pair(fake, B, N, 128, dtype)
        out = tm._Pair(fake << 8, B, N, 128, tm.BF16)
        return lib.tri_mul_transition_forward(ctypes.byref(z), None, None, ctypes.byref(out), None)
    assert status(1, 16392) == 2 and b"[8, 16384]" in lib.tri_mul_last_error()
    assert status(1, 12) == 2
    assert status(1, 64, tm.F32) == 2
    assert status(600, 16384) == 2 and b"too large" in lib.tri_mul_last_error()
    assert status(1, 16384) == 1 and b"handle is NULL" in lib.tri_mul_last_error()
    z = tm._Pair(fake, 1, 64, 128, tm.BF16)
    out = tm._Pair(fake, 1, 64, 128, tm.BF16)
    assert lib.tri_mul_transition_forward(ctypes.byref(z), None, None, ctypes.byref(out), None) == 1
    assert lib.tri_mul_transition_forward(None, None, None, None, None) == 1


def test_pair_update_and_graph_validate_on_the_host(lib):
    z = tm._Pair(0, 1, 8, 128, tm.BF16)
    mid = tm._Pair(0, 1, 8, 128, tm.BF16)
    out = tm._Pair(0, 1, 8, 128, tm.F32)
    assert lib.tri_mul_pair_update(ctypes.byref(z), None, None, None, ctypes.byref(mid), ctypes.byref(out),
                                   None) == 1
    assert lib.tri_mul_pair_update_graph_create(ctypes.byref(z), None, None, None, ctypes.byref(mid),
                                                ctypes.byref(out), None) == 1
    assert lib.tri_mul_graph_launch(None, None) == 1
    lib.tri_mul_graph_destroy(None)          # NULL is ignored
    assert lib.tri_mul_forward_residual(None, None, None, 0, None, None) != 0


def test_forward_and_noalloc_check_out_before_the_layer_and_the_device(lib):
    """Every rule on `out` that needs no layer (present, aligned, z's shape, fp32 on the fp32
    path, apart from z) is checked before the layer handle, so a bad `out` is reported with
    nothing launched (here: no device at all) by both the workspace and the no-allocation
    entry points."""
    fn = lib.tri_mul_forward_noalloc
    fn.argtypes = [ctypes.POINTER(tm._Pair), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                   ctypes.POINTER(tm._Pair), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    z = tm._Pair(1 << 24, 1, 64, 128, tm.BF16)           # aligned, never dereferenced
    bad_outs = {
        b"out shape differs": tm._Pair(1 << 32, 1, 32, 128, tm.F32),
        b"fp32 path writes fp32 out": None,
        b"out overlaps z": tm._Pair((1 << 24) + 4096, 1, 64, 128, tm.F32),
        b"not 16-byte aligned": tm._Pair((1 << 32) + 8, 1, 64, 128, tm.F32),
        b"out: NULL tensor": tm._Pair(0, 1, 64, 128, tm.F32),
    }
    for entry in (lib.tri_mul_forward, fn):
        for msg, out in bad_outs.items():
            zz = z
            if out is None:                               # an fp32 z with a bf16 out
                zz = tm._Pair(1 << 24, 1, 64, 128, tm.F32)
                out = tm._Pair(1 << 32, 1, 64, 128, tm.BF16)
            st = entry(ctypes.byref(zz), None, None, 0, ctypes.byref(out), None)
            assert st in (1, 7) and msg in lib.tri_mul_last_error(), (entry, msg, lib.tri_mul_last_error())
        good = tm._Pair(1 << 32, 1, 64, 128, tm.F32)
        assert entry(ctypes.byref(z), None, None, 0, ctypes.byref(good), None) == 1
        assert b"layer is NULL" in lib.tri_mul_last_error()


def test_skip_rule_and_valid_length_validation(lib):
    """The skipping rule's measure (host only): no saving at full length, all of it at zero
    length, K2's cubic share in between; the headline's 493 of 512 stays under the 0.15 rule,
    the c_z = 384 workload's lengths (162-237 of 256) are over it."""
    assert tm.skip_saving([512], 512) == 0.0
    assert tm.skip_saving([0, 0], 64) == 1.0
    half = tm.skip_saving([128], 256)
    assert 0.75 < half < 0.875                    # between 1 - 1/4 (pairs) and 1 - 1/8 (cube)
    assert tm.skip_saving([493], 512) < 0.15
    assert tm.skip_saving([237, 210, 193, 162], 256, 384, 128) > 0.15
    assert lib.tri_mul_layer_set_valid_lengths(None, None, 0, 0, None) == 1
    assert lib.tri_mul_forward_extents(None, None, None, None, 0, None, None) == 1
    fake = ctypes.c_void_p(1 << 24)
    assert lib.tri_mul_mask_extents(fake, 1, 12, tm.BF16, fake, None) == 2
    assert lib.tri_mul_mask_extents(fake, 1, 16, tm.F32, fake, None) == 2
