"""Skipping of wholly masked tiles (needs a B200).

With mask skipping switched on, tri_mul_forward with a mask finds the mask's extents and
leaves out tiles that are masked in full and the k-range beyond them; with it off nothing is
left out. Every product left out is an exact zero (and adds nothing to the channel sums the
offsets of the stored x come from), so the two must agree bitwise, for masks of any pattern
(here: a valid block [0, R) x [0, C) with R != C and random holes inside it, the second batch
element with the block transposed), and both must match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import assert_close_rms, upload
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu


def _holey_mask(N, R, C, seed):
    rng = np.random.default_rng(seed)
    m = np.zeros((2, N, N), dtype=np.float32)
    m[0, :R, :C] = rng.random((R, C)) > 0.1
    m[1, :C, :R] = rng.random((C, R)) > 0.1
    return m


@pytest.mark.parametrize("N,R,C,c_z,check_oracle", [
    (256, 100, 100, 128, True),     # rows and k-chunks past 100 left out; an output m-tile too
    (256, 130, 70, 128, True),      # R != C: outgoing and incoming bound k differently
    (136, 100, 60, 128, True),      # N % 128 != 0: tiles straddle rows, no output tile skipped
    (128, 60, 90, 384, True),       # c_z = 384 kernels
    (512, 493, 200, 128, False),    # headline size, columns cut short
])
def test_forward_with_extents_matches_dense_forward_bitwise(N, R, C, c_z, check_oracle):
    inp = ti.generate(2, N, c_z, 128, dtype="bf16", seed=N + R + C, mask=("all",), biases=True)
    inp.mask = _holey_mask(N, R, C, seed=R * C)
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    dense = tm.TriMulLayer(w, eps=inp.eps)
    layer.set_mask_skipping(True)
    for d in ("outgoing", "incoming"):
        full = layer.forward(z, m, d)
        ref_dense = dense.forward(z, m, d)
        torch.cuda.synchronize()
        tm.check_device_status()
        assert torch.equal(full, ref_dense), d
        got = full.cpu().numpy()
        assert not np.any(got[inp.mask == 0]), "masked pairs must be exactly 0"
        if check_oracle:
            ref = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps)
            assert_close_rms(got, ref, 2e-2, what=f"N={N} R={R} C={C} {d}")


def test_all_masked_element_next_to_a_full_one():
    inp = ti.generate(2, 256, 128, 128, dtype="bf16", seed=3, mask=("lengths", [0, 256]))
    z, m, w = upload(inp)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    layer.set_mask_skipping(True)
    for d in ("outgoing", "incoming"):
        got = layer.forward(z, m, d)
        torch.cuda.synchronize()
        tm.check_device_status()
        assert not torch.any(got[0])
        assert torch.isfinite(got[1]).all()


def test_mask_extents_values():
    m = _holey_mask(136, 100, 60, seed=1)
    m = np.concatenate([m, np.zeros((1, 136, 136), np.float32)])       # a third element fully masked
    mt = torch.from_numpy(m).cuda().to(torch.bfloat16)
    ext = tm.mask_extents(mt).cpu().numpy()
    for b in range(3):
        rows = np.nonzero(m[b].any(axis=1))[0]
        cols = np.nonzero(m[b].any(axis=0))[0]
        assert ext[b, 0] == (rows.max() + 1 if rows.size else 0)
        assert ext[b, 1] == (cols.max() + 1 if cols.size else 0)


@pytest.mark.parametrize("c_z", [128, 384])
def test_given_extents_and_valid_lengths_match_the_dense_forward_bitwise(c_z):
    lengths = [237, 210, 193, 162] if c_z == 384 else [200, 256, 90, 131]
    inp = ti.generate(4, 256, c_z, 128, dtype="bf16", seed=c_z + 2, mask=("lengths", lengths), biases=True)
    z, m, w = upload(inp)
    dense = tm.TriMulLayer(w, eps=inp.eps)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    ext = tm.mask_extents(m)
    assert ext.cpu().numpy().tolist() == [[L, L] for L in lengths]
    assert layer.set_valid_lengths(lengths, 256) is (tm.skip_saving(lengths, 256, c_z, 128) >= 0.15)
    for d in ("outgoing", "incoming"):
        ref = dense.forward(z, m, d)
        got_ext = layer.forward_extents(z, m, ext, d)
        got_len = layer.forward(z, m, d)
        torch.cuda.synchronize()
        tm.check_device_status()
        assert torch.equal(ref, got_ext), d
        assert torch.equal(ref, got_len), d
    layer.set_valid_lengths(None)


def test_headline_lengths_do_not_choose_skipping():
    layer_inp = ti.generate(1, 512, 128, 128, dtype="bf16", seed=0, mask=("lengths", [493]))
    z, m, w = upload(layer_inp)
    layer = tm.TriMulLayer(w, eps=layer_inp.eps)
    assert layer.set_valid_lengths([493], 512) is False


def test_pair_update_finds_the_extents_once_and_matches_dense():
    inp = ti.generate(2, 256, 128, 128, dtype="bf16", seed=12, mask=("lengths", [150, 256]), biases=True)
    z, m, w = upload(inp)
    dense = tm.TriMulLayer(w, eps=inp.eps)
    skip = tm.TriMulLayer(w, eps=inp.eps)
    skip.set_mask_skipping(True)
    ref = tm.pair_update(z, m, dense, dense, out_dtype=torch.float32)
    got = tm.pair_update(z, m, skip, skip, out_dtype=torch.float32)
    torch.cuda.synchronize()
    tm.check_device_status()
    assert torch.equal(ref, got)


def test_pair_update_with_valid_lengths_matches_dense():
    lengths = [150, 256]
    inp = ti.generate(2, 256, 128, 128, dtype="bf16", seed=13, mask=("lengths", lengths), biases=True)
    z, m, w = upload(inp)
    dense = tm.TriMulLayer(w, eps=inp.eps)
    vl_out = tm.TriMulLayer(w, eps=inp.eps)
    vl_in = tm.TriMulLayer(w, eps=inp.eps)
    assert vl_out.set_valid_lengths(lengths, 256) is (tm.skip_saving(lengths, 256) >= 0.15)
    vl_in.set_valid_lengths(lengths, 256)
    ref = tm.pair_update(z, m, dense, dense, out_dtype=torch.float32)
    got = tm.pair_update(z, m, vl_out, vl_in, out_dtype=torch.float32)
    torch.cuda.synchronize()
    tm.check_device_status()
    assert torch.equal(ref, got)


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_given_extents_with_no_valid_k_leave_no_stale_intermediates(direction):
    """Extents {100, 0} are a legal bound for an all-zero mask (no nonzero entry anywhere). At
    N = 136 the output kernel's tiles straddle rows, so it still reads x for rows < 100: the
    contraction must write those tiles (exact zeros) rather than leave the workspace's old
    contents, here NaN bit patterns, under masked pairs."""
    inp = ti.generate(2, 136, 128, 128, dtype="bf16", seed=17, mask=("lengths", [0, 136]), biases=True)
    z, m, w = upload(inp)
    dense = tm.TriMulLayer(w, eps=inp.eps)
    layer = tm.TriMulLayer(w, eps=inp.eps)
    layer.ensure_workspace(2, 136, torch.bfloat16)
    layer._ws.fill_(255)                        # every fp16 intermediate reads as NaN
    ext = torch.tensor([[100, 0], [136, 136]], dtype=torch.int32, device="cuda")
    got = layer.forward_extents(z, m, ext, direction)
    ref = dense.forward(z, m, direction)
    torch.cuda.synchronize()
    tm.check_device_status()
    assert torch.isfinite(got).all()
    assert not torch.any(got[0])
    assert torch.equal(got, ref)
