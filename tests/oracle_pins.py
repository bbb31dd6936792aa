"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an oracle library handle and raises AssertionError
when the oracle disagrees with what the mathematics or a library routine fixes.
``test_oracle_pins.py`` runs them against the real oracle; ``test_oracle_mutants.py``
runs them against copies of the oracle with planted mistakes and requires that
at least one pin fails for every mistake.

Sources of truth used here:
  * library routines in float64: torch.nn.functional.layer_norm / linear,
    torch.sigmoid, torch.bmm (the contraction of one channel is a matrix product),
  * closed forms: constant pair field, a hand-worked N=3 example,
  * invariants of the definition: incoming = swap(outgoing(swap z)) with the a/b
    projections exchanged, residue-permutation equivariance, masked residues k
    contribute nothing, padding equals truncation, sampled entries equal the
    full computation, invariance of the output under scaling of the b projection,
  * the pair update (two residual steps): masked pairs keep z bitwise, with one step's
    output projection zeroed it reduces to the other step's single update in its own
    direction, and a constant field goes through both steps in closed form.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import trimul_inputs as ti

F = torch.nn.functional


def _t(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def _close(a, b, rtol=1e-12, atol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = np.max(np.abs(b)) if b.size else 0.0
    assert err <= atol + rtol * scale, f"{what}: max err {err:.3e} (scale {scale:.3e})"


def _small(seed=3, B=2, N=7, c_z=12, c_h=10, mask=("uniform_len", 4, 7)):
    return ti.generate(B, N, c_z, c_h, dtype="f32", seed=seed, mask=mask, affine=True, biases=True)


# ---------------------------------------------------------------- library routines

def pin_layernorm_library(lib):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((37, 19)) * 3 + 1.5
    g = 1 + 0.3 * rng.standard_normal(19)
    b = 0.2 * rng.standard_normal(19)
    for eps in (1e-5, 0.3):
        ref = F.layer_norm(_t(x), (19,), _t(g), _t(b), eps).numpy()
        _close(oracle.layernorm(x, g, b, eps, lib=lib), ref, what=f"layernorm eps={eps}")


def pin_linear_library(lib):
    rng = np.random.default_rng(12)
    x, W, bias = rng.standard_normal((23, 9)), rng.standard_normal((5, 9)), rng.standard_normal(5)
    _close(oracle.linear(x, W, bias, lib=lib), F.linear(_t(x), _t(W), _t(bias)).numpy(), what="linear")
    _close(oracle.linear(x, W, None, lib=lib), F.linear(_t(x), _t(W)).numpy(), what="linear nobias")


def pin_gated_projection_library(lib):
    rng = np.random.default_rng(13)
    x = rng.standard_normal((31, 8))
    m = (rng.random(31) > 0.3).astype(np.float64)
    Wg, bg, Wp, bp = (rng.standard_normal((6, 8)), rng.standard_normal(6),
                      rng.standard_normal((6, 8)), rng.standard_normal(6))
    ref = _t(m)[:, None] * torch.sigmoid(F.linear(_t(x), _t(Wg), _t(bg))) * F.linear(_t(x), _t(Wp), _t(bp))
    _close(oracle.gated_projection(x, m, Wg, bg, Wp, bp, lib=lib), ref.numpy(), what="gated projection")


def pin_contract_library(lib):
    """One channel of the contraction is a matrix product: out = A B^T, in = A^T B."""
    rng = np.random.default_rng(14)
    B, N, C = 2, 9, 5
    a, b = rng.standard_normal((B, N, N, C)), rng.standard_normal((B, N, N, C))
    A = _t(a).permute(0, 3, 1, 2).reshape(B * C, N, N)       # [(b,c), row, col]
    Bm = _t(b).permute(0, 3, 1, 2).reshape(B * C, N, N)
    out_ref = torch.bmm(A, Bm.transpose(1, 2)).reshape(B, C, N, N).permute(0, 2, 3, 1)
    in_ref = torch.bmm(A.transpose(1, 2), Bm).reshape(B, C, N, N).permute(0, 2, 3, 1)
    _close(oracle.contract(a, b, "outgoing", lib=lib), out_ref.numpy(), what="contract outgoing")
    _close(oracle.contract(a, b, "incoming", lib=lib), in_ref.numpy(), what="contract incoming")


def pin_output_gate_library(lib):
    rng = np.random.default_rng(15)
    R, c_z, c_h = 29, 7, 6
    zh, x = rng.standard_normal((R, c_z)), rng.standard_normal((R, c_h)) * 4
    m = (rng.random(R) > 0.25).astype(np.float64)
    Wg, bg = rng.standard_normal((c_z, c_z)), rng.standard_normal(c_z)
    g, bt = 1 + 0.2 * rng.standard_normal(c_h), 0.3 * rng.standard_normal(c_h)
    Wo, bo = rng.standard_normal((c_z, c_h)), rng.standard_normal(c_z)
    eps = 1e-5
    ref = (_t(m)[:, None] * torch.sigmoid(F.linear(_t(zh), _t(Wg), _t(bg)))
           * F.linear(F.layer_norm(_t(x), (c_h,), _t(g), _t(bt), eps), _t(Wo), _t(bo)))
    _close(oracle.output_gate(zh, x, m, Wg, bg, g, bt, eps, Wo, bo, lib=lib), ref.numpy(),
           what="output gate")


def _torch_modules_reference(inp, direction):
    """The update written with torch.nn modules (LayerNorm, Linear) and torch.einsum."""
    w = {k: _t(v) for k, v in inp.weights.items()}
    c_z, c_h, eps = inp.c_z, inp.c_h, inp.eps
    ln_in = torch.nn.LayerNorm(c_z, eps=eps, dtype=torch.float64)
    ln_out = torch.nn.LayerNorm(c_h, eps=eps, dtype=torch.float64)
    lins = {n: torch.nn.Linear(*reversed(w["w_" + n].shape), dtype=torch.float64)
            for n in ("ag", "ap", "bg", "bp", "g", "o")}
    with torch.no_grad():
        ln_in.weight.copy_(w["ln_in_g"]); ln_in.bias.copy_(w["ln_in_b"])
        ln_out.weight.copy_(w["ln_out_g"]); ln_out.bias.copy_(w["ln_out_b"])
        for n, lin in lins.items():
            lin.weight.copy_(w["w_" + n]); lin.bias.copy_(w["b_" + n])
        z = _t(inp.z)
        m = _t(inp.mask)[..., None]
        zh = ln_in(z)
        a = m * torch.sigmoid(lins["ag"](zh)) * lins["ap"](zh)
        b = m * torch.sigmoid(lins["bg"](zh)) * lins["bp"](zh)
        eq = "bikc,bjkc->bijc" if direction == "outgoing" else "bkic,bkjc->bijc"
        x = torch.einsum(eq, a, b)
        out = m * torch.sigmoid(lins["g"](zh)) * lins["o"](ln_out(x))
    return out.numpy(), a.numpy(), b.numpy(), x.numpy()


def pin_full_update_library(lib):
    for seed, mask in ((3, ("uniform_len", 4, 7)), (4, ("all",))):
        inp = _small(seed=seed, mask=mask)
        for d in ("outgoing", "incoming"):
            out, a, b, x = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps, intermediates=True, lib=lib)
            ro, ra, rb, rx = _torch_modules_reference(inp, d)
            _close(a, ra, what=f"a {d}")
            _close(b, rb, what=f"b {d}")
            _close(x, rx, what=f"x {d}")
            _close(out, ro, what=f"out {d}")


# ---------------------------------------------------------------- closed forms

def _constant_field_update(v, weights, N):
    """The update of the constant field z_ij = v (all-ones mask) at every pair: every
    a_ik = alpha, b_jk = beta, so x_ij = N alpha*beta. alpha, beta, the LayerNorm of
    N alpha*beta and the gate are torch library calls on a single pair; the N^3 contraction
    is replaced by the scalar N."""
    w = {k: _t(x) for k, x in weights.items()}
    c_z, c_h = w["w_ag"].shape[1], w["w_ag"].shape[0]
    zh = F.layer_norm(_t(v), (c_z,), w["ln_in_g"], w["ln_in_b"], 1e-5)
    alpha = torch.sigmoid(F.linear(zh, w["w_ag"], w["b_ag"])) * F.linear(zh, w["w_ap"], w["b_ap"])
    beta = torch.sigmoid(F.linear(zh, w["w_bg"], w["b_bg"])) * F.linear(zh, w["w_bp"], w["b_bp"])
    xv = N * alpha * beta
    o = torch.sigmoid(F.linear(zh, w["w_g"], w["b_g"])) * F.linear(
        F.layer_norm(xv, (c_h,), w["ln_out_g"], w["ln_out_b"], 1e-5), w["w_o"], w["b_o"])
    return o.numpy()


def pin_constant_field_closed_form(lib):
    """z_ij = v everywhere, all-ones mask: the update is the closed form above at every pair,
    in both directions."""
    rng = np.random.default_rng(21)
    c_z, c_h = 6, 5
    base = ti.generate(1, 1, c_z, c_h, dtype="f32", seed=21, affine=True, biases=True)
    v = rng.standard_normal(c_z) * 2 + 0.5
    for N in (1, 4, 9):
        z = np.broadcast_to(v, (1, N, N, c_z)).copy()
        expect = np.broadcast_to(_constant_field_update(v, base.weights, N), (1, N, N, c_z))
        for d in ("outgoing", "incoming"):
            _close(oracle.trimul(z, None, base.weights, d, 1e-5, lib=lib), expect,
                   rtol=1e-11, what=f"constant field N={N} {d}")


def _hand_problem(masked_last: bool):
    """N=3, c_z=2, c_h=3. z_ij = t_ij [1, -1] with t_ij = s_ij (1 + i + 2j), so with gamma=1,
    beta=0 the normalized pair is s_ij [1, -1] / sqrt(1 + eps/t^2) (exactly s_ij [1, -1] at eps=0).

      a_ik = 1/2 * [s_ik, 1, 1]          (gate weight 0 -> sigmoid(0) = 1/2; proj [s, 1, 1])
      b_jk = 1/2 * [1, s_jk, 2]          (proj [1, s, 2])
      outgoing x_ij = sum_k a_ik b_jk = [R_i / 4, R_j / 4, n / 2]   (R = row sums of s over valid k)
      incoming x_ij = sum_k a_ki b_kj = [C_i / 4, C_j / 4, n / 2]   (C = column sums)
      LN(x_ij) over the three channels, written out for a 3-vector
      out_ij = m_ij [sigmoid(s_ij) * L0, 1/2 * (L1 + L2 + 1/2)]
    """
    s = np.array([[1, 1, 1], [1, -1, -1], [-1, 1, -1]], dtype=np.float64)
    N = 3
    t = np.array([[s[i, j] * (1 + i + 2 * j) for j in range(N)] for i in range(N)])
    z = np.stack([t, -t], axis=-1)[None]                    # [1, 3, 3, 2]
    valid = np.array([1.0, 1.0, 0.0 if masked_last else 1.0])
    mask = (valid[:, None] * valid[None, :])[None]
    zero32 = np.zeros((3, 2))
    w = {
        "ln_in_g": np.ones(2), "ln_in_b": np.zeros(2),
        "w_ag": zero32, "b_ag": np.zeros(3),
        "w_ap": np.array([[1.0, 0], [0, 0], [0, 0]]), "b_ap": np.array([0.0, 1, 1]),
        "w_bg": zero32, "b_bg": np.zeros(3),
        "w_bp": np.array([[0.0, 0], [1, 0], [0, 0]]), "b_bp": np.array([1.0, 0, 2]),
        "w_g": np.array([[1.0, 0], [0, 0]]), "b_g": np.zeros(2),
        "ln_out_g": np.ones(3), "ln_out_b": np.zeros(3),
        "w_o": np.array([[1.0, 0, 0], [0, 1, 1]]), "b_o": np.array([0.0, 0.5]),
    }
    return s, valid, z, mask, w


def _ln3(v, eps):
    mu = sum(v) / 3.0
    d = [x - mu for x in v]
    var = sum(x * x for x in d) / 3.0
    return [x / math.sqrt(var + eps) for x in d]


def pin_hand_worked_example(lib):
    # eps = 0 makes the input LayerNorm return s_ij [1, -1] exactly. With a masked residue the
    # masked pairs have x = 0, so that case uses eps > 0 (LN(0) would be 0/0 otherwise); then the
    # normalized pair is u_ij [1, -1] with u_ij = t_ij / sqrt(t_ij^2 + eps), and s is replaced by
    # u throughout the closed form (row/column sums and the output gate).
    for masked_last, eps in ((False, 0.0), (True, 1e-3)):
        s, valid, z, mask, w = _hand_problem(masked_last)
        t = z[0, :, :, 0]
        u = t / np.sqrt(t * t + eps)
        n = int(valid.sum())
        R = [sum(u[i, k] for k in range(3) if valid[k]) for i in range(3)]
        C = [sum(u[k, i] for k in range(3) if valid[k]) for i in range(3)]
        for d, S in (("outgoing", R), ("incoming", C)):
            expect = np.zeros((1, 3, 3, 2))
            for i in range(3):
                for j in range(3):
                    if not (valid[i] and valid[j]):
                        continue
                    L = _ln3([S[i] / 4.0, S[j] / 4.0, n / 2.0], eps)
                    sig = 1.0 / (1.0 + math.exp(-u[i, j]))
                    expect[0, i, j] = [sig * L[0], 0.5 * (L[1] + L[2] + 0.5)]
            got = oracle.trimul(z, mask, w, d, eps, lib=lib)
            _close(got, expect, rtol=1e-13, atol=1e-13, what=f"hand example {d} masked={masked_last}")


# ---------------------------------------------------------------- invariants

def _swap(x):
    return np.swapaxes(x, 1, 2)


def pin_transpose_identity(lib):
    """incoming(z, m; W_a, W_b) = swap(outgoing(swap z, swap m; W_b, W_a))."""
    inp = _small(seed=31, N=8)
    inc = oracle.trimul(inp.z, inp.mask, inp.weights, "incoming", inp.eps, lib=lib)
    via = _swap(oracle.trimul(_swap(inp.z), _swap(inp.mask), inp.weights_swapped_ab(), "outgoing",
                              inp.eps, lib=lib))
    _close(inc, via, rtol=1e-13, atol=1e-14, what="transpose identity")
    # without the a/b exchange the identity must not hold (the pin is not vacuous)
    wrong = _swap(oracle.trimul(_swap(inp.z), _swap(inp.mask), inp.weights, "outgoing", inp.eps, lib=lib))
    assert np.max(np.abs(wrong - inc)) > 1e-3


def pin_permutation_equivariance(lib):
    inp = _small(seed=41, N=8)
    perm = np.random.default_rng(41).permutation(inp.N)
    zp = inp.z[:, perm][:, :, perm]
    mp = inp.mask[:, perm][:, :, perm]
    for d in ("outgoing", "incoming"):
        ref = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps, lib=lib)
        got = oracle.trimul(zp, mp, inp.weights, d, inp.eps, lib=lib)
        _close(got, ref[:, perm][:, :, perm], rtol=1e-12, atol=1e-13, what=f"permutation {d}")


def pin_masked_k_contributes_nothing(lib):
    """Changing z on pairs that touch a masked residue leaves every valid (i, j) bitwise unchanged."""
    inp = _small(seed=51, N=8, mask=("lengths", [5, 6]))
    z2 = inp.z.copy()
    rng = np.random.default_rng(51)
    for b in range(inp.B):
        L = int(inp.lengths[b])
        z2[b, L:, :, :] = rng.standard_normal(z2[b, L:].shape) * 5
        z2[b, :, L:, :] = rng.standard_normal(z2[b, :, L:].shape) * 5
    for d in ("outgoing", "incoming"):
        o1 = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps, lib=lib)
        o2 = oracle.trimul(z2, inp.mask, inp.weights, d, inp.eps, lib=lib)
        for b in range(inp.B):
            L = int(inp.lengths[b])
            assert np.array_equal(o1[b, :L, :L], o2[b, :L, :L]), f"masked k leaked ({d})"
            assert not np.any(o1[b, L:]) and not np.any(o1[b, :, L:]), f"masked rows not zero ({d})"


def pin_padding_equals_truncation(lib):
    inp = _small(seed=61, B=1, N=9, mask=("lengths", [6]))
    L = 6
    w = inp.weights
    for d in ("outgoing", "incoming"):
        full = oracle.trimul(inp.z, inp.mask, w, d, inp.eps, lib=lib)
        trunc = oracle.trimul(inp.z[:, :L, :L], None, w, d, inp.eps, lib=lib)
        assert np.array_equal(full[:, :L, :L], trunc), f"padding != truncation ({d})"


def pin_sampled_equals_full(lib):
    inp = _small(seed=71, N=9, mask=("lengths", [7, 9]))
    I = np.array([0, 3, 8, 5])
    J = np.array([2, 8, 1])
    for d in ("outgoing", "incoming"):
        full = oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps, lib=lib)
        samp = oracle.trimul_sampled(inp.z, inp.mask, inp.weights, d, I, J, inp.eps, lib=lib)
        assert np.array_equal(samp, full[:, I][:, :, J]), f"sampled != full ({d})"


def pin_b_projection_scale_invariance(lib):
    """With W_bg = 0 the gate on b is a constant; scaling W_bp and b_bp by s > 0 scales x by s,
    which the output LayerNorm removes up to its eps term (eps = 0 here for an exact check)."""
    inp = _small(seed=81, N=6, mask=("all",))
    w = dict(inp.weights)
    w["w_bg"] = np.zeros_like(w["w_bg"])
    w2 = dict(w)
    w2["w_bp"] = np.asarray(w["w_bp"], dtype=np.float64) * 3.0
    w2["b_bp"] = np.asarray(w["b_bp"], dtype=np.float64) * 3.0
    for d in ("outgoing", "incoming"):
        o1 = oracle.trimul(inp.z, inp.mask, w, d, 0.0, lib=lib)
        o2 = oracle.trimul(inp.z, inp.mask, w2, d, 0.0, lib=lib)
        _close(o2, o1, rtol=1e-12, atol=1e-13, what=f"scale invariance {d}")
        # a negative scale flips the sign of x, which LayerNorm does not undo
        w3 = dict(w)
        w3["w_bp"] = -w["w_bp"]
        w3["b_bp"] = -w["b_bp"]
        o3 = oracle.trimul(inp.z, inp.mask, w3, d, 0.0, lib=lib)
        assert np.max(np.abs(o3 - o1)) > 1e-3


def pin_single_residue_directions_agree(lib):
    """At N = 1 the only k is the pair itself, so both directions give the same result."""
    inp = ti.generate(3, 1, 8, 6, dtype="f32", seed=91, affine=True, biases=True)
    o1 = oracle.trimul(inp.z, inp.mask, inp.weights, "outgoing", inp.eps, lib=lib)
    o2 = oracle.trimul(inp.z, inp.mask, inp.weights, "incoming", inp.eps, lib=lib)
    assert np.array_equal(o1, o2)


# ---------------------------------------------------------------- pair update (two residual steps)


def _zero_output_projection(weights):
    """Weights whose update is exactly 0 everywhere (W_o = 0 and b_o = 0)."""
    w = {k: (None if v is None else np.array(v, dtype=np.float64, copy=True)) for k, v in weights.items()}
    w["w_o"][:] = 0.0
    if w.get("b_o") is not None:
        w["b_o"][:] = 0.0
    return w


def _two_layers(seed=41):
    inp = _small(seed=seed)
    other = _small(seed=seed + 1)          # a second layer: same shapes, other weights
    return inp, inp.weights, other.weights


def pin_pair_update_masked_pairs_keep_z(lib):
    """Both updates are exactly 0 at a masked pair, so z_mid and out keep z there bitwise."""
    inp, w1, w2 = _two_layers()
    z_mid, out = oracle.pair_update(inp.z, inp.mask, w1, w2, inp.eps, lib=lib)
    masked = inp.mask == 0
    assert masked.any()
    z = np.asarray(inp.z, dtype=np.float64)
    assert np.array_equal(z_mid[masked], z[masked]) and np.array_equal(out[masked], z[masked])


def pin_pair_update_first_step_is_outgoing(lib):
    """With a zero second update the pair update is z + outgoing(z) with the first layer's
    weights (the incoming update or the other weights give a different result here)."""
    inp, w1, w2 = _two_layers()
    _, out = oracle.pair_update(inp.z, inp.mask, w1, _zero_output_projection(w2), inp.eps, lib=lib)
    z = np.asarray(inp.z, dtype=np.float64)
    ref = z + oracle.trimul(inp.z, inp.mask, w1, "outgoing", inp.eps, lib=lib)
    wrong = z + oracle.trimul(inp.z, inp.mask, w1, "incoming", inp.eps, lib=lib)
    _close(out, ref, what="pair update, step 1")
    assert np.max(np.abs(out - wrong)) > 1e-6


def pin_pair_update_second_step_is_incoming(lib):
    """With a zero first update the pair update is z + incoming(z) with the second layer's
    weights."""
    inp, w1, w2 = _two_layers()
    z_mid, out = oracle.pair_update(inp.z, inp.mask, _zero_output_projection(w1), w2, inp.eps, lib=lib)
    z = np.asarray(inp.z, dtype=np.float64)
    assert np.array_equal(z_mid, z)
    ref = z + oracle.trimul(inp.z, inp.mask, w2, "incoming", inp.eps, lib=lib)
    wrong = z + oracle.trimul(inp.z, inp.mask, w2, "outgoing", inp.eps, lib=lib)
    _close(out, ref, what="pair update, step 2")
    assert np.max(np.abs(out - wrong)) > 1e-6


def pin_pair_update_constant_field(lib):
    """A constant field stays constant through both steps: z_mid = v + u1(v) and
    out = z_mid + u2(z_mid), with u1, u2 the closed-form constant-field updates of the two
    layers. The second step must see z_mid, not z."""
    rng = np.random.default_rng(23)
    c_z, c_h, N = 6, 5, 4
    l1 = ti.generate(1, 1, c_z, c_h, dtype="f32", seed=23, affine=True, biases=True).weights
    l2 = ti.generate(1, 1, c_z, c_h, dtype="f32", seed=24, affine=True, biases=True).weights
    v = rng.standard_normal(c_z) * 2 + 0.5
    z = np.broadcast_to(v, (1, N, N, c_z)).copy()
    mid = v + _constant_field_update(v, l1, N)
    out = mid + _constant_field_update(mid, l2, N)
    z_mid, got = oracle.pair_update(z, None, l1, l2, 1e-5, lib=lib)
    _close(z_mid, np.broadcast_to(mid, z.shape), rtol=1e-11, what="pair update z_mid, constant field")
    _close(got, np.broadcast_to(out, z.shape), rtol=1e-11, what="pair update out, constant field")


# ---------------------------------------------------------------- pair transition


def _transition_inputs(seed=61, B=2, N=5, c=12, h=24):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((B, N, N, c))
    mask = (rng.random((B, N, N)) > 0.3).astype(np.float64)
    w1 = rng.standard_normal((h, c)) / math.sqrt(c)
    b1 = rng.standard_normal(h) * 0.1
    w2 = rng.standard_normal((c, h)) / math.sqrt(h)
    b2 = rng.standard_normal(c) * 0.1
    return z, mask, w1, b1, w2, b2


def pin_pair_transition_library(lib):
    """Against torch's float64 linear and relu, composed as the pages list the steps."""
    z, mask, w1, b1, w2, b2 = _transition_inputs()
    ref = _t(z) + _t(mask)[..., None] * F.linear(torch.relu(F.linear(_t(z), _t(w1), _t(b1))), _t(w2), _t(b2))
    _close(oracle.pair_transition(z, mask, w1, b1, w2, b2), ref.numpy(), what="pair transition")


def pin_pair_transition_closed_forms(lib):
    """With b1 so negative that every hidden unit is cut by the ReLU, out = z + m b2; masked
    pairs keep z bitwise; scaling W2 and b2 by s scales the update by s."""
    z, mask, w1, b1, w2, b2 = _transition_inputs()
    out = oracle.pair_transition(z, mask, w1, np.full_like(b1, -1e6), w2, b2)
    _close(out, z + mask[..., None] * b2, what="all hidden units cut")
    out = oracle.pair_transition(z, mask, w1, b1, w2, b2)
    assert np.array_equal(out[mask == 0], z[mask == 0])
    out2 = oracle.pair_transition(z, mask, w1, b1, 3.0 * w2, 3.0 * b2)
    _close(out2 - z, 3.0 * (out - z), what="update linear in W2, b2")


ALL_PINS = [
    pin_layernorm_library, pin_linear_library, pin_gated_projection_library, pin_contract_library,
    pin_output_gate_library, pin_full_update_library, pin_constant_field_closed_form,
    pin_hand_worked_example, pin_transpose_identity, pin_permutation_equivariance,
    pin_masked_k_contributes_nothing, pin_padding_equals_truncation, pin_sampled_equals_full,
    pin_b_projection_scale_invariance, pin_single_residue_directions_agree,
    pin_pair_update_masked_pairs_keep_z, pin_pair_update_first_step_is_outgoing,
    pin_pair_update_second_step_is_incoming, pin_pair_update_constant_field, pin_pair_transition_library,
    pin_pair_transition_closed_forms,
]
