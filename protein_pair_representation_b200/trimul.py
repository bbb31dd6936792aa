"""Python binding of the C ABI in include/trimul.h (argument marshalling only).

Every step of the update runs in the CUDA library; this module only turns torch
tensors into pointers and sizes, allocates the workspace through torch (the
caller's allocator) and turns status codes into exceptions. If the library is
missing the calls raise; there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

OUTGOING = 0
INCOMING = 1
F32 = 0
BF16 = 1
F16 = 2
_DIRS = {"outgoing": OUTGOING, "incoming": INCOMING, OUTGOING: OUTGOING, INCOMING: INCOMING}

WEIGHT_ORDER = (
    "ln_in_g", "ln_in_b", "w_ag", "b_ag", "w_ap", "b_ap", "w_bg", "b_bg",
    "w_bp", "b_bp", "w_g", "b_g", "ln_out_g", "ln_out_b", "w_o", "b_o",
)

STATUS_NAMES = {
    0: "TRIMUL_OK", 1: "TRIMUL_ERR_INVALID_ARG", 2: "TRIMUL_ERR_UNSUPPORTED_SHAPE",
    3: "TRIMUL_ERR_UNSUPPORTED_DEVICE", 4: "TRIMUL_ERR_WORKSPACE", 5: "TRIMUL_ERR_CUDA",
    6: "TRIMUL_ERR_DEVICE_TIMEOUT", 7: "TRIMUL_ERR_ALIGNMENT", 8: "TRIMUL_ERR_RANGE",
}


class TriMulError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {detail}")
        self.status = status
        self.detail = detail


class _Pair(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("B", ctypes.c_int64), ("N", ctypes.c_int64),
                ("C", ctypes.c_int64), ("dtype", ctypes.c_int)]


class _Rows(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("B", ctypes.c_int64), ("R", ctypes.c_int64), ("N", ctypes.c_int64),
                ("C", ctypes.c_int64), ("row0", ctypes.c_int64), ("dtype", ctypes.c_int)]


class _WeightsDesc(ctypes.Structure):
    _fields_ = [("c_z", ctypes.c_int32), ("c_h", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("eps", ctypes.c_float)] + [(n, ctypes.c_void_p) for n in WEIGHT_ORDER]


_lib = None
_lib_lock = threading.Lock()


def library_path() -> str:
    return _build.LIB_PATH


def load_library():
    """Load libtrimul.so (built in-tree by protein_pair_representation_b200.build)."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        path = _build.LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path} is missing "
                               "(run python -m protein_pair_representation_b200.build)")
        lib = ctypes.CDLL(path)
        vp, i64, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        P = ctypes.POINTER
        lib.tri_mul_layer_create.argtypes = [P(_WeightsDesc), vp, P(vp)]
        lib.tri_mul_layer_destroy.argtypes = [vp]
        lib.tri_mul_layer_destroy.restype = None
        lib.tri_mul_workspace_bytes.argtypes = [vp, i64, i64, st]
        lib.tri_mul_workspace_bytes.restype = ctypes.c_size_t
        lib.tri_mul_layer_bind_workspace.argtypes = [vp, vp, ctypes.c_size_t]
        lib.tri_mul_forward.argtypes = [P(_Pair), vp, vp, st, P(_Pair), vp]
        lib.tri_mul_forward_residual.argtypes = [P(_Pair), vp, vp, st, P(_Pair), vp]
        lib.tri_mul_pair_update.argtypes = [P(_Pair), vp, vp, vp, P(_Pair), P(_Pair), vp]
        lib.tri_mul_pair_update_graph_create.argtypes = [P(_Pair), vp, vp, vp, P(_Pair), P(_Pair), P(vp)]
        lib.tri_mul_graph_launch.argtypes = [vp, vp]
        lib.tri_mul_graph_destroy.argtypes = [vp]
        lib.tri_mul_graph_destroy.restype = None
        lib.tri_mul_project.argtypes = [P(_Pair), vp, vp, vp, vp, vp]
        lib.tri_mul_contract.argtypes = [vp, vp, vp, i64, i64, i64, st, st, ctypes.c_float, vp]
        lib.tri_mul_contract_scale.argtypes = [i64]
        lib.tri_mul_contract_scale.restype = ctypes.c_float
        lib.tri_mul_output_gate.argtypes = [P(_Pair), vp, vp, ctypes.c_float, vp, P(_Pair), vp]
        lib.tri_mul_layer_set_timing_events.argtypes = [vp, P(vp)]
        lib.tri_mul_layer_set_mask_skipping.argtypes = [vp, st]
        lib.tri_mul_transition_create.argtypes = [st, st, st, vp, vp, vp, vp, vp, P(vp)]
        lib.tri_mul_transition_destroy.argtypes = [vp]
        lib.tri_mul_transition_destroy.restype = None
        lib.tri_mul_transition_forward.argtypes = [P(_Pair), vp, vp, P(_Pair), vp]
        lib.tri_mul_shard_workspace_bytes.argtypes = [vp, i64, i64, i64]
        lib.tri_mul_shard_workspace_bytes.restype = ctypes.c_size_t
        lib.tri_mul_shard_project.argtypes = [P(_Rows), vp, vp, vp, vp, vp]
        lib.tri_mul_shard_finish.argtypes = [P(_Rows), vp, vp, st, st, P(i64), P(vp), P(vp), P(_Rows), vp]
        lib.tri_mul_mask_extents.argtypes = [vp, i64, i64, st, vp, vp]
        lib.tri_mul_forward_extents.argtypes = [P(_Pair), vp, vp, vp, st, P(_Pair), vp]
        lib.tri_mul_skip_saving.argtypes = [P(i64), i64, i64, ctypes.c_int32, ctypes.c_int32]
        lib.tri_mul_skip_saving.restype = ctypes.c_double
        lib.tri_mul_layer_set_valid_lengths.argtypes = [vp, P(i64), i64, i64, P(ctypes.c_int32)]
        lib.tri_mul_kernels_per_forward.argtypes = []
        lib.tri_mul_check_device_status.argtypes = []
        lib.tri_mul_status_string.argtypes = [st]
        lib.tri_mul_status_string.restype = ctypes.c_char_p
        lib.tri_mul_last_error.argtypes = []
        lib.tri_mul_last_error.restype = ctypes.c_char_p
        lib.tri_mul_abi_version.argtypes = []
        for name in ("tri_mul_layer_create", "tri_mul_layer_bind_workspace", "tri_mul_forward",
                     "tri_mul_forward_residual", "tri_mul_pair_update", "tri_mul_pair_update_graph_create",
                     "tri_mul_graph_launch", "tri_mul_layer_set_mask_skipping", "tri_mul_transition_create",
                     "tri_mul_transition_forward",
                     "tri_mul_project", "tri_mul_contract", "tri_mul_output_gate",
                     "tri_mul_shard_project", "tri_mul_shard_finish", "tri_mul_mask_extents",
                     "tri_mul_forward_extents", "tri_mul_layer_set_valid_lengths",
                     "tri_mul_layer_set_timing_events", "tri_mul_check_device_status"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def _check(status: int):
    if status != 0:
        lib = load_library()
        raise TriMulError(status, lib.tri_mul_last_error().decode(errors="replace"))


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return F32
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float16:
        return F16
    raise TypeError(f"unsupported dtype {dt}")


def intermediate_dtype(z_dtype: torch.dtype) -> torch.dtype:
    """Storage type of a, b and x: float16 for a bfloat16 z, float32 for a float32 z."""
    return torch.float16 if z_dtype == torch.bfloat16 else torch.float32


def contract_scale(N: int) -> float:
    """The power of two tri_mul_forward stores x multiplied by on the tensor-core path."""
    return float(load_library().tri_mul_contract_scale(N))


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _pair(t: torch.Tensor) -> _Pair:
    if t.dim() != 4 or t.shape[1] != t.shape[2]:
        raise ValueError(f"pair tensor must be [B, N, N, C], got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError("pair tensor must be contiguous")
    return _Pair(t.data_ptr(), t.shape[0], t.shape[1], t.shape[3], _dtype_code(t.dtype))


def _rows(t: torch.Tensor, row0: int, N: int) -> _Rows:
    """[B, R, N, C] rows [row0, row0 + R) of an N x N pair tensor."""
    if t.dim() != 4 or t.shape[2] != N:
        raise ValueError(f"row slab must be [B, R, N={N}, C], got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError("row slab must be contiguous")
    return _Rows(t.data_ptr(), t.shape[0], t.shape[1], N, t.shape[3], row0, _dtype_code(t.dtype))


def shard_bounds(N: int, G: int) -> list:
    """Row boundaries of G shards of an N x N pair tensor: whole 128-row blocks, as even as they go
    (the first shards take the extra blocks)."""
    if N % 128 or G < 1 or G > N // 128:
        raise ValueError(f"N={N} must be a multiple of 128 with at least one 128-row block per shard (G={G})")
    blocks = N // 128
    bounds = [0]
    for g in range(G):
        bounds.append(bounds[-1] + 128 * (blocks // G + (1 if g < blocks % G else 0)))
    return bounds


def _mask_ptr(mask, z):
    if mask is None:
        return None
    if mask.dtype != z.dtype or tuple(mask.shape) != tuple(z.shape[:3]) or not mask.is_contiguous():
        raise ValueError("mask must be a contiguous [B, N, N] tensor in z's dtype")
    return mask.data_ptr()


class TriMulLayer:
    """A triangle multiplicative update layer (weights repacked on the device).

    weights: dict name -> CUDA tensor (all float32 or all bfloat16), names as in
    WEIGHT_ORDER; biases and LayerNorm parameters may be missing (None).
    """

    def __init__(self, weights: dict, eps: float = 1e-5, stream=None):
        self._lib = load_library()
        w_ag = weights["w_ag"]
        c_h, c_z = w_ag.shape
        dt = w_ag.dtype
        self._keep = []
        desc = _WeightsDesc()
        desc.c_z, desc.c_h, desc.dtype, desc.eps = c_z, c_h, _dtype_code(dt), eps
        for n in WEIGHT_ORDER:
            t = weights.get(n)
            if t is None:
                setattr(desc, n, None)
                continue
            if t.dtype != dt or not t.is_cuda:
                raise ValueError(f"weight {n} must be a CUDA tensor of dtype {dt}")
            t = t.contiguous()
            self._keep.append(t)
            setattr(desc, n, t.data_ptr())
        handle = ctypes.c_void_p()
        _check(self._lib.tri_mul_layer_create(ctypes.byref(desc), _stream_ptr(stream), ctypes.byref(handle)))
        self._keep = []
        self.handle = handle
        self.c_z, self.c_h, self.eps = c_z, c_h, eps
        self.device = w_ag.device
        self._ws = None
        self._events = None

    def close(self):
        if getattr(self, "handle", None):
            self._lib.tri_mul_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, B: int, N: int, dtype: torch.dtype) -> int:
        return int(self._lib.tri_mul_workspace_bytes(self.handle, B, N, _dtype_code(dtype)))

    def bind_workspace(self, buf: torch.Tensor | None):
        """Attach a caller-allocated uint8 CUDA buffer (or None) as the workspace."""
        self._ws = buf
        ptr = None if buf is None else buf.data_ptr()
        nbytes = 0 if buf is None else buf.numel() * buf.element_size()
        _check(self._lib.tri_mul_layer_bind_workspace(self.handle, ptr, nbytes))

    def ensure_workspace(self, B: int, N: int, dtype: torch.dtype):
        need = self.workspace_bytes(B, N, dtype)
        if self._ws is None or self._ws.numel() < need:
            self.bind_workspace(torch.empty(need, dtype=torch.uint8, device=self.device))

    def set_mask_skipping(self, enable: bool = True):
        """Leave out wholly masked tiles (mask extents found by a first pass); off by default."""
        _check(self._lib.tri_mul_layer_set_mask_skipping(self.handle, 1 if enable else 0))

    def set_valid_lengths(self, lengths, N: int | None = None) -> bool:
        """Valid lengths of a left-aligned padding mask, one per batch element, for every later
        forward of len(lengths) x N problems (None clears). Returns whether skipping was chosen."""
        if lengths is None:
            _check(self._lib.tri_mul_layer_set_valid_lengths(self.handle, None, 0, 0, None))
            return False
        arr = (ctypes.c_int64 * len(lengths))(*[int(v) for v in lengths])
        chosen = ctypes.c_int32(0)
        _check(self._lib.tri_mul_layer_set_valid_lengths(self.handle, arr, len(lengths), N, ctypes.byref(chosen)))
        return bool(chosen.value)

    def forward_extents(self, z: torch.Tensor, mask: torch.Tensor, extents: torch.Tensor, direction="outgoing",
                        out: torch.Tensor | None = None, out_dtype: torch.dtype | None = None, stream=None):
        """The update with the mask's extents given (int32 [B, 2] CUDA tensor, e.g. mask_extents())."""
        B, N = z.shape[0], z.shape[1]
        self.ensure_workspace(B, N, z.dtype)
        if extents.dtype != torch.int32 or tuple(extents.shape) != (B, 2) or not extents.is_contiguous():
            raise ValueError("extents must be a contiguous int32 [B, 2] tensor")
        if out is None:
            out = torch.empty(z.shape, dtype=out_dtype or torch.float32, device=z.device)
        zp, op = _pair(z), _pair(out)
        _check(self._lib.tri_mul_forward_extents(ctypes.byref(zp), _mask_ptr(mask, z), extents.data_ptr(), self.handle,
                                                 _DIRS[direction], ctypes.byref(op), _stream_ptr(stream)))
        return out

    def set_timing_events(self, events):
        """events: four torch.cuda.Event(enable_timing=True) or None."""
        self._events = events
        if events is None:
            _check(self._lib.tri_mul_layer_set_timing_events(self.handle, None))
            return
        arr = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
        _check(self._lib.tri_mul_layer_set_timing_events(self.handle, arr))

    def forward(self, z: torch.Tensor, mask: torch.Tensor | None = None, direction="outgoing",
                out: torch.Tensor | None = None, out_dtype: torch.dtype | None = None, stream=None,
                residual: bool = False):
        """The update (residual=False) or z + update (residual=True) of one direction."""
        B, N = z.shape[0], z.shape[1]
        self.ensure_workspace(B, N, z.dtype)
        if out is None:
            out = torch.empty(z.shape, dtype=out_dtype or torch.float32, device=z.device)
        zp, op = _pair(z), _pair(out)
        fn = self._lib.tri_mul_forward_residual if residual else self._lib.tri_mul_forward
        _check(fn(ctypes.byref(zp), _mask_ptr(mask, z), self.handle, _DIRS[direction], ctypes.byref(op),
                  _stream_ptr(stream)))
        return out

    __call__ = forward

    def project(self, z: torch.Tensor, mask: torch.Tensor | None = None, stream=None,
                a: torch.Tensor | None = None, b: torch.Tensor | None = None):
        """K1 alone: a, b as [B, c_h, N, N] in the intermediate dtype (into `a`, `b` when given)."""
        B, N = z.shape[0], z.shape[1]
        shape, dt = (B, self.c_h, N, N), intermediate_dtype(z.dtype)
        for t in (a, b):
            if t is not None and (tuple(t.shape) != shape or t.dtype != dt or not t.is_contiguous()):
                raise ValueError(f"a and b must be contiguous {shape} tensors of {dt}")
        a = torch.empty(shape, dtype=dt, device=z.device) if a is None else a
        b = torch.empty_like(a) if b is None else b
        zp = _pair(z)
        _check(self._lib.tri_mul_project(ctypes.byref(zp), _mask_ptr(mask, z), self.handle,
                                         a.data_ptr(), b.data_ptr(), _stream_ptr(stream)))
        return a, b

    # ---- row-sharded update (one shard of the rows; see include/trimul.h) ----

    def ensure_shard_workspace(self, B: int, R: int, N: int):
        need = int(self._lib.tri_mul_shard_workspace_bytes(self.handle, B, R, N))
        if self._ws is None or self._ws.numel() < need:
            self.bind_workspace(torch.empty(need, dtype=torch.uint8, device=self.device))

    def shard_project(self, z_rows: torch.Tensor, mask_rows: torch.Tensor | None, row0: int, N: int, stream=None):
        """Phase 1 for rows [row0, row0 + R) of an N x N pair tensor: a, b as [B, c_h, R, N] float16."""
        B, R = z_rows.shape[0], z_rows.shape[1]
        self.ensure_shard_workspace(B, R, N)
        a = torch.empty((B, self.c_h, R, N), dtype=torch.float16, device=z_rows.device)
        b = torch.empty_like(a)
        zr = _rows(z_rows, row0, N)
        _check(self._lib.tri_mul_shard_project(ctypes.byref(zr), _mask_ptr(mask_rows, z_rows) if mask_rows is not None
                                               else None, self.handle, a.data_ptr(), b.data_ptr(), _stream_ptr(stream)))
        return a, b

    def shard_finish(self, z_rows: torch.Tensor, mask_rows: torch.Tensor | None, row0: int, N: int, direction,
                     bounds, a_shards, b_shards, out: torch.Tensor | None = None,
                     out_dtype: torch.dtype | None = None, stream=None):
        """Phase 2: this shard's rows of the update from every shard's phase-1 a and b (a list of
        G tensors each; entries of a_shards other than this shard's may be None for outgoing)."""
        G = len(bounds) - 1
        B, R = z_rows.shape[0], z_rows.shape[1]
        self.ensure_shard_workspace(B, R, N)
        if out is None:
            out = torch.empty(z_rows.shape, dtype=out_dtype or torch.float32, device=z_rows.device)
        row_arr = (ctypes.c_int64 * (G + 1))(*bounds)
        ptr = lambda t: None if t is None else t.data_ptr()
        a_arr = (ctypes.c_void_p * G)(*[ptr(t) for t in a_shards])
        b_arr = (ctypes.c_void_p * G)(*[ptr(t) for t in b_shards])
        zr, orow = _rows(z_rows, row0, N), _rows(out, row0, N)
        _check(self._lib.tri_mul_shard_finish(ctypes.byref(zr), _mask_ptr(mask_rows, z_rows) if mask_rows is not None
                                              else None, self.handle, _DIRS[direction], G, row_arr, a_arr, b_arr,
                                              ctypes.byref(orow), _stream_ptr(stream)))
        return out

    def output_gate(self, z: torch.Tensor, x: torch.Tensor, mask: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, out_dtype: torch.dtype | None = None, x_scale: float = 1.0,
                    stream=None):
        """K3 alone: out from z and x [B, c_h, N, N] (intermediate dtype, holding x_scale * x)."""
        if (x.dtype != intermediate_dtype(z.dtype) or not x.is_contiguous()
                or tuple(x.shape) != (z.shape[0], self.c_h, z.shape[1], z.shape[2])):
            raise ValueError("x must be a contiguous [B, c_h, N, N] tensor in the intermediate dtype")
        if out is None:
            out = torch.empty(z.shape, dtype=out_dtype or torch.float32, device=z.device)
        zp, op = _pair(z), _pair(out)
        _check(self._lib.tri_mul_output_gate(ctypes.byref(zp), _mask_ptr(mask, z), x.data_ptr(), x_scale,
                                             self.handle, ctypes.byref(op), _stream_ptr(stream)))
        return out


def contract(a: torch.Tensor, b: torch.Tensor, direction="outgoing", out: torch.Tensor | None = None,
             x_scale: float = 1.0, stream=None):
    """K2 alone on [B, C, N, N] tensors (float16 / bfloat16 on tensor cores, float32 on CUDA cores)."""
    lib = load_library()
    if a.shape != b.shape or a.dim() != 4 or a.shape[2] != a.shape[3] or a.dtype != b.dtype:
        raise ValueError("a and b must be [B, C, N, N] of one dtype")
    if not (a.is_contiguous() and b.is_contiguous()):
        raise ValueError("a and b must be contiguous")
    if out is None:
        out = torch.empty_like(a)
    B, C, N, _ = a.shape
    _check(lib.tri_mul_contract(a.data_ptr(), b.data_ptr(), out.data_ptr(), B, C, N, _dtype_code(a.dtype),
                                _DIRS[direction], x_scale, _stream_ptr(stream)))
    return out


class PairTransition:
    """The fused pair transition out = z + m * (relu(z W1^T + b1) W2^T + b2) (bf16, c = 128,
    hidden = 256). Weights: CUDA bf16 tensors W1 [256, 128], W2 [128, 256], biases or None."""

    def __init__(self, w1: torch.Tensor, w2: torch.Tensor, b1: torch.Tensor | None = None,
                 b2: torch.Tensor | None = None, stream=None):
        self._lib = load_library()
        hidden, c = w1.shape
        for t in (w1, w2, b1, b2):
            if t is not None and (t.dtype != torch.bfloat16 or not t.is_cuda):
                raise ValueError("pair transition weights must be bfloat16 CUDA tensors")
        keep = [t.contiguous() for t in (w1, w2) + tuple(x for x in (b1, b2) if x is not None)]
        w1c, w2c = keep[0], keep[1]
        b1c = b1.contiguous() if b1 is not None else None
        b2c = b2.contiguous() if b2 is not None else None
        handle = ctypes.c_void_p()
        _check(self._lib.tri_mul_transition_create(c, hidden, BF16, w1c.data_ptr(),
                                                   None if b1c is None else b1c.data_ptr(), w2c.data_ptr(),
                                                   None if b2c is None else b2c.data_ptr(), _stream_ptr(stream),
                                                   ctypes.byref(handle)))
        self.handle = handle
        self.c, self.hidden = c, hidden

    def forward(self, z: torch.Tensor, mask: torch.Tensor | None = None, out: torch.Tensor | None = None,
                out_dtype: torch.dtype | None = None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(z.shape, dtype=out_dtype or z.dtype, device=z.device)
        zp, op = _pair(z), _pair(out)
        _check(self._lib.tri_mul_transition_forward(ctypes.byref(zp), _mask_ptr(mask, z), self.handle,
                                                    ctypes.byref(op), _stream_ptr(stream)))
        return out

    __call__ = forward

    def close(self):
        if getattr(self, "handle", None):
            self._lib.tri_mul_transition_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def pair_update(z: torch.Tensor, mask: torch.Tensor | None, layer_out: TriMulLayer, layer_in: TriMulLayer,
                out: torch.Tensor | None = None, z_mid: torch.Tensor | None = None, out_dtype: torch.dtype | None = None,
                stream=None):
    """One pair update: z_mid = z + U_outgoing(z) (z's dtype), out = z_mid + U_incoming(z_mid)."""
    B, N = z.shape[0], z.shape[1]
    layer_out.ensure_workspace(B, N, z.dtype)
    layer_in.ensure_workspace(B, N, z.dtype)
    if z_mid is None:
        z_mid = torch.empty_like(z)
    if out is None:
        out = torch.empty(z.shape, dtype=out_dtype or z.dtype, device=z.device)
    zp, mp, op = _pair(z), _pair(z_mid), _pair(out)
    _check(load_library().tri_mul_pair_update(ctypes.byref(zp), _mask_ptr(mask, z), layer_out.handle, layer_in.handle,
                                              ctypes.byref(mp), ctypes.byref(op), _stream_ptr(stream)))
    return out


class PairUpdateGraph:
    """A CUDA graph of one pair_update on fixed tensors; launch() replays it.

    The tensors and both layers (with their workspaces) must stay alive, in place, for the
    graph's lifetime; write new inputs into `z` and `mask` between launches.
    """

    def __init__(self, z: torch.Tensor, mask: torch.Tensor | None, layer_out: TriMulLayer, layer_in: TriMulLayer,
                 out_dtype: torch.dtype | None = None):
        self._lib = load_library()
        B, N = z.shape[0], z.shape[1]
        layer_out.ensure_workspace(B, N, z.dtype)
        layer_in.ensure_workspace(B, N, z.dtype)
        self.z, self.mask, self.layers = z, mask, (layer_out, layer_in)
        self.z_mid = torch.empty_like(z)
        self.out = torch.empty(z.shape, dtype=out_dtype or z.dtype, device=z.device)
        zp, mp, op = _pair(z), _pair(self.z_mid), _pair(self.out)
        handle = ctypes.c_void_p()
        torch.cuda.synchronize(z.device)
        _check(self._lib.tri_mul_pair_update_graph_create(ctypes.byref(zp), _mask_ptr(mask, z), layer_out.handle,
                                                          layer_in.handle, ctypes.byref(mp), ctypes.byref(op),
                                                          ctypes.byref(handle)))
        self.handle = handle

    def launch(self, stream=None) -> torch.Tensor:
        _check(self._lib.tri_mul_graph_launch(self.handle, _stream_ptr(stream)))
        return self.out

    def close(self):
        if getattr(self, "handle", None):
            self._lib.tri_mul_graph_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def mask_extents(mask: torch.Tensor, stream=None) -> torch.Tensor:
    """{R_b, C_b} of a bfloat16 [B, N, N] mask: int32 [B, 2] on its device."""
    if mask.dtype != torch.bfloat16 or mask.dim() != 3 or not mask.is_contiguous():
        raise ValueError("mask must be a contiguous bfloat16 [B, N, N] tensor")
    ext = torch.empty((mask.shape[0], 2), dtype=torch.int32, device=mask.device)
    _check(load_library().tri_mul_mask_extents(mask.data_ptr(), mask.shape[0], mask.shape[1], BF16, ext.data_ptr(),
                                               _stream_ptr(stream)))
    return ext


def skip_saving(lengths, N: int, c_z: int = 128, c_h: int = 128) -> float:
    """The share of a layer's dense work that skipping by these valid lengths leaves out."""
    arr = (ctypes.c_int64 * len(lengths))(*[int(v) for v in lengths])
    return float(load_library().tri_mul_skip_saving(arr, len(lengths), N, c_z, c_h))


def check_device_status():
    _check(load_library().tri_mul_check_device_status())


def kernels_per_forward() -> int:
    return int(load_library().tri_mul_kernels_per_forward())
