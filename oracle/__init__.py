"""fp64 CPU oracle for the triangle multiplicative update.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library and
its Python binding never import it and share no code with it.

The arithmetic lives in ``trimul_oracle.c`` (plain C loops, fp64, sums in
stated order, OpenMP only across independent rows). This module compiles it
with gcc on first use and marshals numpy arrays through ctypes.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
library routines (torch LayerNorm / Linear / bmm in float64), a closed form,
hand-derived fixtures, the incoming/outgoing transpose identity, residue
permutation equivariance and the mask invariants; ``tests/test_oracle_mutants.py``
plants plausible mistakes in a copy of the C source and checks that a pin fails.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "trimul_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11"]

OUTGOING = 0
INCOMING = 1
_DIRS = {"outgoing": OUTGOING, "incoming": INCOMING, OUTGOING: OUTGOING, INCOMING: INCOMING}

WEIGHT_ORDER = (
    "ln_in_g", "ln_in_b", "w_ag", "b_ag", "w_ap", "b_ap", "w_bg", "b_bg",
    "w_bp", "b_bp", "w_g", "b_g", "ln_out_g", "ln_out_b", "w_o", "b_o",
)

_lock = threading.Lock()
_lib = None


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_ORDER]


def compile_library(source: str = SOURCE, out_path: str = LIB_PATH, force: bool = False) -> str:
    """Compile the oracle C source into a shared library (gcc); returns its path."""
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    if (not force and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(source)):
        return out_path
    tmp = out_path + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, source, "-lm"], check=True)
    os.replace(tmp, out_path)
    return out_path


def _bind(lib):
    i64, dp, vp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_layernorm.argtypes = [i64, i64, dp, dp, dp, ctypes.c_double, dp]
    lib.oracle_linear.argtypes = [i64, i64, i64, dp, dp, dp, dp]
    lib.oracle_gated_projection.argtypes = [i64, i64, i64, dp, dp, dp, dp, dp, dp, dp]
    lib.oracle_contract.argtypes = [i64, i64, i64, dp, dp, ctypes.c_int, dp]
    lib.oracle_output_gate.argtypes = [i64, i64, i64, dp, dp, dp, dp, dp, dp, dp,
                                       ctypes.c_double, dp, dp, dp]
    lib.oracle_trimul_ex.argtypes = [i64, i64, i64, i64, dp, dp, ctypes.POINTER(_Weights),
                                     ctypes.c_int, ctypes.c_double, dp, vp, vp, vp]
    lib.oracle_trimul_sampled.argtypes = [i64, i64, i64, i64, dp, dp, ctypes.POINTER(_Weights),
                                          ctypes.c_int, ctypes.c_double, dp, i64, dp, i64, dp]
    for name in ("oracle_layernorm", "oracle_linear", "oracle_gated_projection", "oracle_contract",
                 "oracle_output_gate", "oracle_trimul_ex", "oracle_trimul_sampled"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


def load_library(path: str | None = None):
    """Load (compiling if needed) the oracle library. A custom path returns a fresh handle."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(compile_library()))
    return _lib


def num_threads(lib=None) -> int:
    return int((lib or load_library()).oracle_num_threads())


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def layernorm(x, gamma=None, beta=None, eps=1e-5, lib=None):
    lib = lib or load_library()
    x = _f64(x)
    C = x.shape[-1]
    y = np.empty_like(x)
    g, b = _f64(gamma), _f64(beta)
    _check(lib.oracle_layernorm(x.size // C, C, _ptr(x), _ptr(g), _ptr(b), eps, _ptr(y)), "layernorm")
    return y


def linear(x, W, bias=None, lib=None):
    lib = lib or load_library()
    x, W, bias = _f64(x), _f64(W), _f64(bias)
    c_out, c_in = W.shape
    y = np.empty(x.shape[:-1] + (c_out,), dtype=np.float64)
    _check(lib.oracle_linear(x.size // c_in, c_in, c_out, _ptr(x), _ptr(W), _ptr(bias), _ptr(y)), "linear")
    return y


def gated_projection(xhat, mask, Wg, bg, Wp, bp, lib=None):
    lib = lib or load_library()
    xhat, mask, Wg, bg, Wp, bp = map(_f64, (xhat, mask, Wg, bg, Wp, bp))
    c_out, c_in = Wg.shape
    y = np.empty(xhat.shape[:-1] + (c_out,), dtype=np.float64)
    _check(lib.oracle_gated_projection(xhat.size // c_in, c_in, c_out, _ptr(xhat), _ptr(mask),
                                       _ptr(Wg), _ptr(bg), _ptr(Wp), _ptr(bp), _ptr(y)), "gated_projection")
    return y


def contract(a, b, direction, lib=None):
    """x from a, b of shape [B, N, N, C] (pair-major, channel-last)."""
    lib = lib or load_library()
    a, b = _f64(a), _f64(b)
    B, N, _, C = a.shape
    x = np.empty_like(a)
    _check(lib.oracle_contract(B, N, C, _ptr(a), _ptr(b), _DIRS[direction], _ptr(x)), "contract")
    return x


def output_gate(zhat, x, mask, Wg, bg, ln_out_g, ln_out_b, eps, Wo, bo, lib=None):
    lib = lib or load_library()
    zhat, x, mask, Wg, bg, ln_out_g, ln_out_b, Wo, bo = map(
        _f64, (zhat, x, mask, Wg, bg, ln_out_g, ln_out_b, Wo, bo))
    c_z = zhat.shape[-1]
    c_h = x.shape[-1]
    out = np.empty(zhat.shape[:-1] + (c_z,), dtype=np.float64)
    _check(lib.oracle_output_gate(zhat.size // c_z, c_z, c_h, _ptr(zhat), _ptr(x), _ptr(mask),
                                  _ptr(Wg), _ptr(bg), _ptr(ln_out_g), _ptr(ln_out_b), eps,
                                  _ptr(Wo), _ptr(bo), _ptr(out)), "output_gate")
    return out


def _weights_struct(weights):
    arrs = {n: _f64(weights.get(n)) for n in WEIGHT_ORDER}
    s = _Weights(**{n: (_ptr(a) if a is not None else None) for n, a in arrs.items()})
    return s, arrs


def trimul(z, mask, weights, direction, eps=1e-5, intermediates=False, lib=None):
    """The full update on z [B, N, N, c_z]; returns out (and a, b, x when asked)."""
    lib = lib or load_library()
    z, mask = _f64(z), _f64(mask)
    B, N, _, c_z = z.shape
    c_h = np.asarray(weights["w_ag"]).shape[0]
    ws, keep = _weights_struct(weights)
    out = np.empty((B, N, N, c_z), dtype=np.float64)
    extra = [np.empty((B, N, N, c_h), dtype=np.float64) for _ in range(3)] if intermediates else [None] * 3
    _check(lib.oracle_trimul_ex(B, N, c_z, c_h, _ptr(z), _ptr(mask), ctypes.byref(ws),
                                _DIRS[direction], eps, _ptr(out), *[_ptr(e) for e in extra]), "trimul")
    del keep
    if intermediates:
        return out, extra[0], extra[1], extra[2]
    return out


def trimul_sampled(z, mask, weights, direction, I, J, eps=1e-5, lib=None):
    """out at the entries (I[p], J[q]) of every batch element: [B, len(I), len(J), c_z]."""
    lib = lib or load_library()
    z, mask = _f64(z), _f64(mask)
    B, N, _, c_z = z.shape
    c_h = np.asarray(weights["w_ag"]).shape[0]
    I = np.ascontiguousarray(I, dtype=np.int64)
    J = np.ascontiguousarray(J, dtype=np.int64)
    ws, keep = _weights_struct(weights)
    out = np.empty((B, len(I), len(J), c_z), dtype=np.float64)
    _check(lib.oracle_trimul_sampled(B, N, c_z, c_h, _ptr(z), _ptr(mask), ctypes.byref(ws),
                                     _DIRS[direction], eps, I.ctypes.data, len(I), J.ctypes.data,
                                     len(J), _ptr(out)), "trimul_sampled")
    del keep
    return out


def pair_update(z, mask, weights_out, weights_in, eps=1e-5, lib=None):
    """One pair update of the triangle stage, in fp64: the outgoing update applied as a
    masked residual, then the incoming one ("RFProteina architecture", section "Two networks
    around one state", subsection "Inside the velocity network"):
        z_mid = z + trimul(z, outgoing; weights_out)
        out   = z_mid + trimul(z_mid, incoming; weights_in)
    Returns (z_mid, out). A masked pair keeps its z: its updates are exactly 0."""
    z = _f64(z)
    z_mid = z + trimul(z, mask, weights_out, "outgoing", eps, lib=lib)
    out = z_mid + trimul(z_mid, mask, weights_in, "incoming", eps, lib=lib)
    return z_mid, out


def pair_transition(z, mask, w1, b1, w2, b2):
    """The fused pair transition, in fp64 ("RFProteina architecture", section "Kernel support":
    both linears, the ReLU, the mask and the residual in one step):
        out_ij = z_ij + m_ij * (relu(z_ij . W1^T + b1) . W2^T + b2)
    z [B, N, N, c], mask [B, N, N] (None: all ones), W1 [h, c], b1 [h], W2 [c, h], b2 [c]
    (None biases: 0). A masked pair keeps its z bitwise."""
    z = _f64(z)
    hid = z @ _f64(w1).T
    if b1 is not None:
        hid = hid + _f64(b1)
    hid = np.maximum(hid, 0.0)
    upd = hid @ _f64(w2).T
    if b2 is not None:
        upd = upd + _f64(b2)
    if mask is not None:
        upd = upd * _f64(mask)[..., None]
    return z + upd
