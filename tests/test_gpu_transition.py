"""The fused pair transition through the C-ABI against the fp64 oracle (needs a B200).

Tolerance, from the arithmetic of the kernel: z and the weights are bf16 (the oracle reads the
same rounded values), products are accumulated in fp32, and the hidden activation is rounded
to f16 on chip (at most 2^-11 relative, summed over 256 terms with random signs), so the
update stays well inside max|err| <= 2e-2 * RMS(update), the bf16 bound of the triangle
update; a bf16 out adds half an ulp of out (at most 2^-8 relative). A masked pair keeps its
z bitwise.
"""
import numpy as np
import pytest
import torch

import oracle
import trimul_inputs as ti
from gpu_helpers import rms
from protein_pair_representation_b200 import trimul as tm

pytestmark = pytest.mark.gpu


def _problem(B, N, seed, biases=True, lengths=None):
    rng = np.random.default_rng(seed)
    z = ti.round_to_bf16(rng.standard_normal((B, N, N, 128)).astype(np.float32))
    L = lengths if lengths is not None else rng.integers(N // 2, N + 1, size=B)
    s = (np.arange(N)[None, :] < np.asarray(L)[:, None]).astype(np.float32)
    mask = s[:, :, None] * s[:, None, :]
    w1 = ti.round_to_bf16((rng.standard_normal((256, 128)) / np.sqrt(128)).astype(np.float32))
    w2 = ti.round_to_bf16((rng.standard_normal((128, 256)) / np.sqrt(256)).astype(np.float32))
    b1 = ti.round_to_bf16((0.1 * rng.standard_normal(256)).astype(np.float32)) if biases else None
    b2 = ti.round_to_bf16((0.1 * rng.standard_normal(128)).astype(np.float32)) if biases else None
    return z, mask, w1, b1, w2, b2


def _cuda(x):
    return None if x is None else torch.from_numpy(np.ascontiguousarray(x)).cuda().to(torch.bfloat16)


@pytest.mark.parametrize("B,N,out_dtype,biases", [(2, 64, torch.float32, True), (1, 136, torch.float32, True),
                                                  (2, 96, torch.bfloat16, True), (1, 256, torch.float32, False)])
def test_pair_transition_against_oracle(B, N, out_dtype, biases):
    z, mask, w1, b1, w2, b2 = _problem(B, N, seed=N + B, biases=biases)
    pt = tm.PairTransition(_cuda(w1), _cuda(w2), _cuda(b1), _cuda(b2))
    out = pt.forward(_cuda(z), _cuda(mask), out_dtype=out_dtype)
    torch.cuda.synchronize()
    tm.check_device_status()
    ref = oracle.pair_transition(z, mask, w1, b1, w2, b2)
    got = out.float().cpu().numpy()
    z64 = z.astype(np.float64)
    bound = 2e-2 * rms(ref - z64) + (2.0 ** -8 * np.abs(ref) if out_dtype == torch.bfloat16 else 0.0)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"worst excess {np.max(err - bound):.3e}; max err / RMS(update) {np.max(err) / rms(ref - z64):.3e}"
    masked = mask == 0
    assert masked.any() or B * N * N == 0
    assert np.array_equal(got[masked], z64[masked])
    print(f"pair transition B={B} N={N} {out_dtype}: max|err| / RMS(update) = {np.max(err) / rms(ref - z64):.3e}")


def test_pair_transition_full_size_sampled():
    """The bench's launch: B=1 N=512 (67 MB of z, 28 tiles per CTA), bf16 in and out, the
    ragged mask of length 493; 4096 sampled pairs against the oracle (the transition acts on
    each pair alone), every masked pair bitwise z."""
    z, mask, w1, b1, w2, b2 = _problem(1, 512, seed=512, lengths=[493])
    zd, md = _cuda(z), _cuda(mask)
    pt = tm.PairTransition(_cuda(w1), _cuda(w2), _cuda(b1), _cuda(b2))
    out = pt.forward(zd, md, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    tm.check_device_status()
    rng = np.random.default_rng(7)
    flat = rng.choice(512 * 512, size=4096, replace=False)
    i, j = flat // 512, flat % 512
    zs, ms = z[0, i, j][None, None], mask[0, i, j][None, None]
    ref = oracle.pair_transition(zs, ms, w1, b1, w2, b2)[0, 0]
    got = out[0, torch.from_numpy(i).cuda(), torch.from_numpy(j).cuda()].float().cpu().numpy()
    z64 = zs[0, 0].astype(np.float64)
    upd = ref - z64
    bound = 2e-2 * rms(upd) + 2.0 ** -8 * np.abs(ref)
    assert np.all(np.abs(got - ref) <= bound), f"worst excess {np.max(np.abs(got - ref) - bound):.3e}"
    masked = md == 0
    assert bool(masked.any()) and torch.equal(out[masked], zd[masked])


def test_pair_transition_tiles_across_batch_elements():
    """B=3 N=200: 625 tiles per batch element, about 13 per CTA, so a CTA's tiles (and the
    next-tile loads of the output warpgroups) cross from one batch element to the next."""
    z, mask, w1, b1, w2, b2 = _problem(3, 200, seed=200, lengths=[200, 131, 77])
    pt = tm.PairTransition(_cuda(w1), _cuda(w2), _cuda(b1), _cuda(b2))
    out = pt.forward(_cuda(z), _cuda(mask), out_dtype=torch.float32)
    torch.cuda.synchronize()
    tm.check_device_status()
    ref = oracle.pair_transition(z, mask, w1, b1, w2, b2)
    got = out.cpu().numpy()
    z64 = z.astype(np.float64)
    err = np.abs(got - ref)
    assert np.max(err) <= 2e-2 * rms(ref - z64), f"max err / RMS(update) {np.max(err) / rms(ref - z64):.3e}"
    assert np.array_equal(got[mask == 0], z64[mask == 0])


def test_pair_transition_without_mask_and_rejections():
    z, _, w1, b1, w2, b2 = _problem(1, 32, seed=3)
    pt = tm.PairTransition(_cuda(w1), _cuda(w2), _cuda(b1), _cuda(b2))
    out = pt.forward(_cuda(z), None, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.pair_transition(z, None, w1, b1, w2, b2)
    assert np.max(np.abs(out.cpu().numpy() - ref)) <= 2e-2 * rms(ref - z)
    with pytest.raises(tm.TriMulError):          # c = 384 is not a supported shape
        tm.PairTransition(torch.zeros(768, 384, dtype=torch.bfloat16, device="cuda"),
                          torch.zeros(384, 768, dtype=torch.bfloat16, device="cuda"))
