"""Seeded synthetic inputs for the triangle multiplicative update.

This module only draws random numbers and rounds them to the storage type.
It holds none of the operation's arithmetic, so both the CPU oracle (through
the tests) and the CUDA path can be fed from it without sharing any code.

Shapes and distributions stand in for the pair tracks the pages describe:
OpenFold's Evoformer pair width of 128 (OpenFold-TRT summary, section on the
Evoformer optimisation) and RFProteína's pair track [B, N, N, 384] ("RFProteína
architecture", section "Inside the velocity network"). The pages' own
workloads (CASP14 targets, designed dimers) are datasets that are not
available; these seeded tensors take their place.

Draw order, fixed for a given seed (numpy ``default_rng(seed)``):
  1. valid lengths L_b, one per batch element (only for ragged masks),
  2. z, row block by row block,
  3. the sixteen weight arrays in the C-ABI struct order
     (ln_in_g, ln_in_b, w_ag, b_ag, w_ap, b_ap, w_bg, b_bg, w_bp, b_bp,
      w_g, b_g, ln_out_g, ln_out_b, w_o, b_o).
Sampled (i, j) index sets come from a separate generator seeded ``seed + 7``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

WEIGHT_ORDER = (
    "ln_in_g", "ln_in_b", "w_ag", "b_ag", "w_ap", "b_ap", "w_bg", "b_bg",
    "w_bp", "b_bp", "w_g", "b_g", "ln_out_g", "ln_out_b", "w_o", "b_o",
)


def weight_shapes(c_z: int, c_h: int) -> dict:
    """Shapes of the weight arrays; linear weights are [out, in] (y = x W^T + b)."""
    return {
        "ln_in_g": (c_z,), "ln_in_b": (c_z,),
        "w_ag": (c_h, c_z), "b_ag": (c_h,), "w_ap": (c_h, c_z), "b_ap": (c_h,),
        "w_bg": (c_h, c_z), "b_bg": (c_h,), "w_bp": (c_h, c_z), "b_bp": (c_h,),
        "w_g": (c_z, c_z), "b_g": (c_z,),
        "ln_out_g": (c_h,), "ln_out_b": (c_h,),
        "w_o": (c_z, c_h), "b_o": (c_z,),
    }


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-representable."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


@dataclass
class TriMulInputs:
    B: int
    N: int
    c_z: int
    c_h: int
    dtype: str                      # "f32" or "bf16": storage type of z, mask and weights
    eps: float
    lengths: np.ndarray             # [B] valid residues per batch element
    z: np.ndarray                   # [B, N, N, c_z] float32 (bf16-representable when dtype == "bf16")
    mask: np.ndarray                # [B, N, N] float32, 0/1
    weights: dict = field(default_factory=dict)   # name -> float32 array
    seed: int = 0

    def weights_swapped_ab(self) -> dict:
        """The same weights with the a- and b-projections exchanged."""
        w = dict(self.weights)
        for x, y in (("w_ag", "w_bg"), ("b_ag", "b_bg"), ("w_ap", "w_bp"), ("b_ap", "b_bp")):
            w[x], w[y] = self.weights[y], self.weights[x]
        return w


def _mask_from_lengths(B: int, N: int, lengths: np.ndarray) -> np.ndarray:
    idx = np.arange(N)
    s = (idx[None, :] < lengths[:, None]).astype(np.float32)      # [B, N] residue validity
    return s[:, :, None] * s[:, None, :]


def generate(B: int, N: int, c_z: int, c_h: int, *, dtype: str = "bf16", seed: int = 0,
             z_std: float = 1.0, mask: tuple = ("all",), eps: float = 1e-5,
             affine: bool = False, biases: bool = False, block_rows: int = 64) -> TriMulInputs:
    """Draw one seeded problem.

    mask: ("all",) all ones; ("tail_fraction", f) last ceil(f*N) residues masked on both
    axes; ("uniform_len", lo, hi) per-sample valid length L_b ~ UniformInt[lo, hi].
    affine/biases: when False, LayerNorm gamma=1, beta=0 and all biases 0 (the values
    are still drawn, so the draw order does not depend on these flags).
    """
    if dtype not in ("f32", "bf16"):
        raise ValueError(dtype)
    rng = np.random.default_rng(seed)
    kind = mask[0]
    if kind == "all":
        lengths = np.full(B, N, dtype=np.int64)
    elif kind == "tail_fraction":
        lengths = np.full(B, N - int(math.ceil(mask[1] * N)), dtype=np.int64)
    elif kind == "uniform_len":
        lengths = rng.integers(mask[1], mask[2] + 1, size=B).astype(np.int64)
    elif kind == "lengths":
        lengths = np.asarray(mask[1], dtype=np.int64).reshape(B)
    else:
        raise ValueError(mask)

    rnd = round_to_bf16 if dtype == "bf16" else (lambda a: a.astype(np.float32))
    z = np.empty((B, N, N, c_z), dtype=np.float32)
    for b in range(B):
        for i0 in range(0, N, block_rows):
            i1 = min(N, i0 + block_rows)
            blk = rng.standard_normal((i1 - i0, N, c_z), dtype=np.float32)
            if z_std != 1.0:
                blk *= np.float32(z_std)
            z[b, i0:i1] = rnd(blk)

    shapes = weight_shapes(c_z, c_h)
    fan_in = {"w_ag": c_z, "w_ap": c_z, "w_bg": c_z, "w_bp": c_z, "w_g": c_z, "w_o": c_h}
    w = {}
    for name in WEIGHT_ORDER:
        draw = rng.standard_normal(shapes[name]).astype(np.float32)
        if name in fan_in:
            val = draw / np.float32(math.sqrt(fan_in[name]))
        elif name.endswith("_g") and name.startswith("ln"):
            val = (1.0 + 0.25 * draw) if affine else np.ones_like(draw)
        elif name.startswith("ln"):
            val = (0.25 * draw) if affine else np.zeros_like(draw)
        else:  # biases
            val = (0.5 * draw) if biases else np.zeros_like(draw)
        w[name] = rnd(np.asarray(val, dtype=np.float32))

    return TriMulInputs(B=B, N=N, c_z=c_z, c_h=c_h, dtype=dtype, eps=eps, lengths=lengths,
                        z=z, mask=_mask_from_lengths(B, N, lengths), weights=w, seed=seed)


def sample_indices(N: int, n: int = 64, seed: int = 0) -> tuple:
    """Distinct sorted row indices I and column indices J for sampled comparisons."""
    rng = np.random.default_rng(seed + 7)
    n = min(n, N)
    I = np.sort(rng.choice(N, size=n, replace=False)).astype(np.int64)
    J = np.sort(rng.choice(N, size=n, replace=False)).astype(np.int64)
    return I, J


# The five measured workloads. Each entry: shape, storage type, z spread, mask recipe and
# the directions it runs.
CONFIGS = {
    "fp32_n64": dict(B=1, N=64, c_z=128, c_h=128, dtype="f32", z_std=1.0, mask=("all",),
                     directions=("outgoing",)),
    "bf16_n256_tail10": dict(B=1, N=256, c_z=128, c_h=128, dtype="bf16", z_std=1.0,
                             mask=("tail_fraction", 0.1), directions=("outgoing", "incoming")),
    "bf16_n512_ragged": dict(B=1, N=512, c_z=128, c_h=128, dtype="bf16", z_std=1.0,
                             mask=("uniform_len", 384, 512), directions=("outgoing", "incoming")),
    "bf16_b4_n256_cz384": dict(B=4, N=256, c_z=384, c_h=128, dtype="bf16", z_std=0.5,
                               mask=("uniform_len", 128, 256), directions=("outgoing", "incoming")),
    "bf16_n2048": dict(B=1, N=2048, c_z=128, c_h=128, dtype="bf16", z_std=1.0, mask=("all",),
                       directions=("incoming", "outgoing"), sampled=64),
}


def make_config(name: str, seed: int = 0) -> TriMulInputs:
    c = CONFIGS[name]
    return generate(c["B"], c["N"], c["c_z"], c["c_h"], dtype=c["dtype"], seed=seed,
                    z_std=c["z_std"], mask=c["mask"])
