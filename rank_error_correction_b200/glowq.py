"""Thin Python binding of libglowq (the C ABI declared in include/glowq.h).

Argument marshalling only: every step of the corrected linear layer runs in
the library's CUDA kernels.  PyTorch tensors provide device memory and the
current CUDA stream; their data pointers are handed to the C entry points.
There is no CPU fallback: if ``libglowq.so`` is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
import re
from typing import List, Optional, Sequence, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libglowq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "glowq.h")

GROUP_SIZE = 128
MAX_RANK = 256
MAX_MODULES = 8

FMT_INT4, FMT_MXFP4, FMT_NVFP4 = 0, 1, 2
FP4_BLOCK = {FMT_MXFP4: 32, FMT_NVFP4: 16}

STATUS = {0: "GLOWQ_OK", 1: "GLOWQ_ERR_ARG", 2: "GLOWQ_ERR_SHAPE", 3: "GLOWQ_ERR_ALIGN",
          4: "GLOWQ_ERR_CUDA", 5: "GLOWQ_ERR_TIMEOUT", 6: "GLOWQ_ERR_UNSUPPORTED", 7: "GLOWQ_ERR_NUMERIC"}


class GlowQError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_status_string(code)})")


class _FP4Module(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("tensor_scale", C.c_void_p),
                ("A", C.c_void_p), ("out_features", C.c_int64), ("Y", C.c_void_p), ("ldY", C.c_int64)]


class _SolveModule(C.Structure):
    _fields_ = [("W", C.c_void_p), ("qweight", C.c_void_p), ("scales", C.c_void_p), ("zeros", C.c_void_p),
                ("out_features", C.c_int64)]


class _Module(C.Structure):
    _fields_ = [("qweight", C.c_void_p), ("scales", C.c_void_p), ("zeros", C.c_void_p),
                ("A", C.c_void_p), ("out_features", C.c_int64), ("Y", C.c_void_p), ("ldY", C.c_int64)]


_lib = None


def lib() -> C.CDLL:
    """Load libglowq.so (build it first with rank_error_correction_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libglowq.so not built at {LIB_PATH}; run "
                               "`python -m rank_error_correction_b200.build`")
        L = C.CDLL(LIB_PATH)
        p, i64, i32, st = C.c_void_p, C.c_int64, C.c_int32, C.c_int
        L.glowq_pack_int4.argtypes = [p, i64, i64, i32, p, p, p, p]
        L.glowq_dequant_int4.argtypes = [p, p, p, i64, i64, i32, p, p]
        L.glowq_pack_fp4.argtypes = [st, p, i64, i64, p, p, p, p]
        L.glowq_dequant_fp4.argtypes = [st, p, p, p, i64, i64, p, p]
        L.glowq_workspace_bytes.argtypes = [i64, i32]
        L.glowq_workspace_bytes.restype = C.c_size_t
        L.glowq_workspace_bytes_for.argtypes = [i64, i32, i64, p, i32]
        L.glowq_workspace_bytes_for.restype = C.c_size_t
        L.glowq_group_forward.argtypes = [C.POINTER(_Module), i32, i64, p, i32, p, i64, p, p, C.c_size_t, p]
        L.glowq_solo_forward.argtypes = [C.POINTER(_Module), i64, p, i32, p, i64, p, C.c_size_t, p]
        L.glowq_solo_forward_noalloc.argtypes = [C.POINTER(_Module), i64, p, i32, p, i64, p]
        L.glowq_group_forward_fp4.argtypes = [st, C.POINTER(_FP4Module), i32, i64, p, i32, p, i64, p, p, C.c_size_t, p]
        L.glowq_solo_forward_fp4.argtypes = [st, C.POINTER(_FP4Module), i64, p, i32, p, i64, p, C.c_size_t, p]
        L.glowq_noalloc_scratch_bytes.restype = C.c_size_t
        L.glowq_select_restore.argtypes = [p, p, p, p, i32, i32, p, p, p]
        L.glowq_quantize_act_e4m3.argtypes = [p, i64, i64, p, p, p, p]
        L.glowq_w4a8_workspace_bytes.argtypes = [i64, i64, i32]
        L.glowq_w4a8_workspace_bytes.restype = C.c_size_t
        L.glowq_group_forward_w4a8.argtypes = [C.POINTER(_Module), i32, i64, p, i32, p, i64, p, p, C.c_size_t, p]
        L.glowq_solo_forward_w4a8.argtypes = [C.POINTER(_Module), i64, p, i32, p, i64, p, C.c_size_t, p]
        L.glowq_solve_workspace_bytes.argtypes = [i64, i64, i32, i32]
        L.glowq_solve_workspace_bytes.restype = C.c_size_t
        L.glowq_group_solve.argtypes = [C.POINTER(_SolveModule), i32, i64, p, p, i32, i32, i32, p, p, p, p, p, p, p,
                                        p, C.c_size_t, p]
        L.glowq_select_restore_scores.argtypes = [p, p, p, i32, i32, p, p, p]
        L.glowq_error_norms.argtypes = [p, p, p, p, i64, i64, p, p]
        L.glowq_get_device_status.argtypes = [p]
        L.glowq_selftest_wait_timeout.argtypes = [C.c_uint32, p]
        L.glowq_status_string.argtypes = [st]
        L.glowq_status_string.restype = C.c_char_p
        L.glowq_version.restype = C.c_char_p
        for f in ("glowq_pack_int4", "glowq_dequant_int4", "glowq_pack_fp4", "glowq_dequant_fp4", "glowq_group_forward", "glowq_solo_forward",
                  "glowq_solo_forward_noalloc", "glowq_group_forward_fp4", "glowq_solo_forward_fp4",
                  "glowq_select_restore", "glowq_select_restore_scores", "glowq_error_norms", "glowq_group_solve",
                  "glowq_quantize_act_e4m3", "glowq_group_forward_w4a8", "glowq_solo_forward_w4a8",
                  "glowq_get_device_status",
                  "glowq_selftest_wait_timeout"):
            getattr(L, f).restype = st
        _lib = L
    return _lib


def declared_symbols() -> List[str]:
    """Entry points declared in include/glowq.h."""
    txt = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"GLOWQ_API\s+[\w\s\*]+?\b(glowq_\w+)\s*\(", txt)))


def _status_string(code: int) -> str:
    try:
        return lib().glowq_status_string(code).decode()
    except Exception:  # pragma: no cover - only while reporting another error
        return "?"


def _check(code: int, what: str) -> None:
    if code != 0:
        raise GlowQError(code, what)


def version() -> str:
    return lib().glowq_version().decode()


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libglowq operates on CUDA tensors only")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


# ---------------------------------------------------------------- packing ----

def pack_int4(W, stream=None):
    """W (O x d fp32, CUDA) -> (qweight int32 [O, d/8], scales fp16 [O, d/128], zeros uint8 [O, d/128]).
    qweight holds O * d/8 words in the library's block layout (16-row x 64-k
    blocks of 512 B; see tile_int4), not row by row."""
    import torch
    _require_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    O, d = W.shape
    q = torch.empty((O, d // 8), dtype=torch.int32, device=W.device)
    s = torch.empty((O, d // GROUP_SIZE), dtype=torch.float16, device=W.device)
    z = torch.empty((O, d // GROUP_SIZE), dtype=torch.uint8, device=W.device)
    _check(lib().glowq_pack_int4(_ptr(W), O, d, GROUP_SIZE, _ptr(q), _ptr(s), _ptr(z), _stream(stream)),
           "glowq_pack_int4")
    return q, s, z


def tile_int4(q):
    """Row-major INT4 words (int32 [O, d/8], code k of row o in word k/8) ->
    the library's block layout: blocks of 16 rows x 64 k (16 x 8 words),
    blocks along k within a 16-row tile, tiles in row order.  Same shape and
    dtype; O % 16 == 0.  For codes packed elsewhere."""
    O, w = q.shape
    return q.reshape(O // 16, 16, w // 8, 8).permute(0, 2, 1, 3).contiguous().reshape(O, w)


def untile_int4(q):
    """Inverse of tile_int4: the library's block layout -> row-major words."""
    O, w = q.shape
    return q.reshape(O // 16, w // 8, 16, 8).permute(0, 2, 1, 3).contiguous().reshape(O, w)


def dequant_int4(q, s, z, d: int, stream=None):
    import torch
    _require_cuda(q, s, z)
    O = q.shape[0]
    out = torch.empty((O, d), dtype=torch.float16, device=q.device)
    _check(lib().glowq_dequant_int4(_ptr(q), _ptr(s), _ptr(z), O, d, GROUP_SIZE, _ptr(out), _stream(stream)),
           "glowq_dequant_int4")
    return out


def pack_fp4(W, fmt: int, stream=None):
    """W (O x d fp32, CUDA) -> (codes int32 [O, d/8], scales uint8 [O, d/block], tensor_scale
    float32 [1] for NVFP4 else None) in MXFP4 (fmt 1) or NVFP4 (fmt 2)."""
    import torch
    _require_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    if fmt not in FP4_BLOCK:
        raise ValueError("fmt must be FMT_MXFP4 or FMT_NVFP4")
    O, d = W.shape
    q = torch.empty((O, d // 8), dtype=torch.int32, device=W.device)
    sc = torch.empty((O, d // FP4_BLOCK[fmt]), dtype=torch.uint8, device=W.device)
    ts = torch.empty(1, dtype=torch.float32, device=W.device) if fmt == FMT_NVFP4 else None
    _check(lib().glowq_pack_fp4(fmt, _ptr(W), O, d, _ptr(q), _ptr(sc), _ptr(ts), _stream(stream)), "glowq_pack_fp4")
    return q, sc, ts


def dequant_fp4(codes, scales, tensor_scale, d: int, fmt: int, stream=None):
    import torch
    _require_cuda(codes, scales, tensor_scale)
    O = codes.shape[0]
    out = torch.empty((O, d), dtype=torch.float16, device=codes.device)
    _check(lib().glowq_dequant_fp4(fmt, _ptr(codes), _ptr(scales), _ptr(tensor_scale), O, d, _ptr(out),
                                   _stream(stream)), "glowq_dequant_fp4")
    return out


def error_norms(W, q, s, z, stream=None):
    """Per-row (||W - w_hat||^2, ||W||^2) as a float64 CUDA tensor [O, 2]."""
    import torch
    _require_cuda(W, q, s, z)
    O, d = W.shape
    out = torch.empty((O, 2), dtype=torch.float64, device=W.device)
    _check(lib().glowq_error_norms(_ptr(W), _ptr(q), _ptr(s), _ptr(z), O, d, _ptr(out), _stream(stream)),
           "glowq_error_norms")
    return out


# ---------------------------------------------------------------- forward ----

@dataclasses.dataclass
class QModule:
    """One INT4 g128 module: packed weight, scales, zeros and (optional) left factor A (O x r fp16)."""
    qweight: "object"
    scales: "object"
    zeros: "object"
    A: Optional["object"] = None
    # validated device pointers (qweight, scales, zeros, A, out_features),
    # computed on first use and dropped whenever a field is reassigned
    _ptrs: Optional[tuple] = dataclasses.field(default=None, init=False, repr=False, compare=False)

    def __setattr__(self, name, value):
        object.__setattr__(self, name, value)
        if name != "_ptrs":
            object.__setattr__(self, "_ptrs", None)

    def pointers(self) -> tuple:
        if self._ptrs is None:
            _require_cuda(self.qweight, self.scales, self.zeros, self.A)
            object.__setattr__(self, "_ptrs", (self.qweight.data_ptr(), self.scales.data_ptr(), self.zeros.data_ptr(),
                                               _ptr(self.A), int(self.qweight.shape[0])))
        return self._ptrs

    @property
    def out_features(self) -> int:
        return int(self.qweight.shape[0])

    @property
    def in_features(self) -> int:
        return int(self.qweight.shape[1]) * 8


def workspace_bytes(T: int, r: int) -> int:
    return int(lib().glowq_workspace_bytes(T, r))


def workspace_bytes_for(T: int, r: int, d: int, out_features: Sequence[int]) -> int:
    """Workspace that also enables the k-split of a call of this shape."""
    outs = (C.c_int64 * len(out_features))(*[int(o) for o in out_features])
    return int(lib().glowq_workspace_bytes_for(T, r, d, outs, len(out_features)))


def alloc_workspace(T: int, r: int, device="cuda", d: int = 0, out_features: Sequence[int] = ()):
    # zero-filled: the first 4096 bytes (decode hand-off flags, k-split
    # tickets) must start at zero (every call leaves them zero)
    import torch
    n = workspace_bytes_for(T, r, d, out_features) if d and out_features else workspace_bytes(T, r)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def _auto_workspace(T: int, r: int, d: int, out_features: Sequence[int], device):
    """The workspace a call allocates for itself (None when it needs none)."""
    if workspace_bytes_for(T, r, d, out_features) == 0:
        return None
    return alloc_workspace(T, r, device, d, out_features)


def _module_structs(mods: Sequence[QModule], Ys, use_A: bool):
    items = []
    for m, Y in zip(mods, Ys):
        q, s, z, a, o = m.pointers()
        items.append(_Module(q, s, z, a if use_A else None, o, Y.data_ptr(), Y.stride(0)))
    return (_Module * len(items))(*items)


def group_forward(mods: Sequence[QModule], B, X, Ys=None, R_out=None, workspace=None, stream=None):
    """Input-sharing group: R = X B^T once, Y_i = X w_hat_i^T + R A_i^T.

    B (r x d fp16) may be None (correction off for the whole group).  Ys are
    optional preallocated outputs (T x ldY fp16 views, e.g. column slices of one
    T x sum(O_i) buffer).  Returns (Ys, R).
    """
    import torch
    _require_cuda(B, X)
    T, d = X.shape
    r = 0 if B is None else int(B.shape[0])
    if Ys is None:
        Ys = [torch.empty((T, m.out_features), dtype=torch.float16, device=X.device) for m in mods]
    for Y in Ys:
        if Y.stride(1) != 1:
            raise ValueError("outputs must have unit column stride")
    if r > 0 and R_out is None:
        R_out = torch.empty((T, r), dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = _auto_workspace(T, r, d, [m.out_features for m in mods], X.device)
    arr = _module_structs(mods, Ys, r > 0)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().glowq_group_forward(arr, len(mods), d, _ptr(B), r, _ptr(X), T, _ptr(R_out), _ptr(workspace),
                                     ws_n, _stream(stream)), "glowq_group_forward")
    return Ys, R_out


def solo_forward(mod: QModule, B, X, Y=None, workspace=None, stream=None):
    """Solo module: Y = X w_hat^T + (X B^T) A^T, R computed inline (nothing cached)."""
    import torch
    _require_cuda(B, X)
    T, d = X.shape
    r = 0 if B is None else int(B.shape[0])
    if Y is None:
        Y = torch.empty((T, mod.out_features), dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = _auto_workspace(T, r, d, [mod.out_features], X.device)
    arr = _module_structs([mod], [Y], r > 0)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().glowq_solo_forward(arr, d, _ptr(B), r, _ptr(X), T, _ptr(workspace), ws_n, _stream(stream)),
           "glowq_solo_forward")
    return Y


@dataclasses.dataclass
class FP4Module:
    """One MXFP4 / NVFP4 module: codes (int32 [O, d/8]), block scales (uint8),
    tensor scale (float32 [1], NVFP4) and optional left factor A (O x r fp16)."""
    fmt: int
    codes: "object"
    scales: "object"
    tensor_scale: Optional["object"] = None
    A: Optional["object"] = None

    @property
    def out_features(self) -> int:
        return int(self.codes.shape[0])


def _fp4_structs(mods: Sequence[FP4Module], Ys, use_A: bool):
    items = []
    for m, Y in zip(mods, Ys):
        _require_cuda(m.codes, m.scales, m.tensor_scale, m.A)
        items.append(_FP4Module(m.codes.data_ptr(), m.scales.data_ptr(), _ptr(m.tensor_scale),
                                _ptr(m.A) if use_A else None, m.out_features, Y.data_ptr(), Y.stride(0)))
    return (_FP4Module * len(items))(*items)


def group_forward_fp4(mods: Sequence[FP4Module], B, X, Ys=None, R_out=None, workspace=None, stream=None):
    """group_forward with MXFP4 / NVFP4 base weights (all modules of one format)."""
    import torch
    _require_cuda(B, X)
    T, d = X.shape
    r = 0 if B is None else int(B.shape[0])
    fmt = mods[0].fmt
    if any(m.fmt != fmt for m in mods):
        raise ValueError("all modules of a group share one format")
    if Ys is None:
        Ys = [torch.empty((T, m.out_features), dtype=torch.float16, device=X.device) for m in mods]
    if r > 0 and R_out is None:
        R_out = torch.empty((T, r), dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = _auto_workspace(T, r, d, [m.out_features for m in mods], X.device)
    arr = _fp4_structs(mods, Ys, r > 0)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().glowq_group_forward_fp4(fmt, arr, len(mods), d, _ptr(B), r, _ptr(X), T, _ptr(R_out),
                                         _ptr(workspace), ws_n, _stream(stream)), "glowq_group_forward_fp4")
    return Ys, R_out


def solo_forward_fp4(mod: FP4Module, B, X, Y=None, workspace=None, stream=None):
    import torch
    _require_cuda(B, X)
    T, d = X.shape
    r = 0 if B is None else int(B.shape[0])
    if Y is None:
        Y = torch.empty((T, mod.out_features), dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = _auto_workspace(T, r, d, [mod.out_features], X.device)
    arr = _fp4_structs([mod], [Y], r > 0)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().glowq_solo_forward_fp4(mod.fmt, arr, d, _ptr(B), r, _ptr(X), T, _ptr(workspace), ws_n,
                                        _stream(stream)), "glowq_solo_forward_fp4")
    return Y


class ForwardPlan:
    """A group or solo forward with its arguments marshalled once: calling the
    plan enqueues the kernels with a single C call (no per-call Python
    marshalling), for callers that repeat one call on fixed buffers, e.g. a
    decode loop that refills X in place.  The tensors must stay alive and at
    the same addresses while the plan is used."""

    def __init__(self, mods, B, X, Ys, R_out=None, workspace=None, solo: bool = False, stream=None):
        import torch
        _require_cuda(B, X)
        T, d = X.shape
        r = 0 if B is None else int(B.shape[0])
        if workspace is None:
            workspace = _auto_workspace(T, r, d, [m.out_features for m in mods], X.device)
        if not solo and r > 0 and R_out is None:
            R_out = torch.empty((T, r), dtype=torch.float16, device=X.device)
        self._keep = (mods, B, X, Ys, R_out, workspace)
        arr = _module_structs(mods, Ys, r > 0)
        ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
        L = lib()
        if solo:
            self._fn = L.glowq_solo_forward
            self._args = (arr, d, _ptr(B), r, _ptr(X), T, _ptr(workspace), ws_n)
        else:
            self._fn = L.glowq_group_forward
            self._args = (arr, len(mods), d, _ptr(B), r, _ptr(X), T, _ptr(R_out), _ptr(workspace), ws_n)
        self._stream = _stream(stream)
        self.Ys, self.R = Ys, R_out

    def __call__(self, stream=None):
        rc = self._fn(*self._args, self._stream if stream is None else _stream(stream))
        if rc != 0:
            raise GlowQError(rc, "ForwardPlan")
        return self.Ys


def solo_forward_noalloc(mod: QModule, B, X, Y=None, stream=None):
    """Solo module forward with no workspace argument: the library's fixed
    scratch array is used, so the call allocates no device memory.  For callers
    that cannot allocate at call time (e.g. inside another runtime's enqueue).
    Only the output Y is allocated here when not given."""
    import torch
    _require_cuda(B, X)
    T, d = X.shape
    r = 0 if B is None else int(B.shape[0])
    if Y is None:
        Y = torch.empty((T, mod.out_features), dtype=torch.float16, device=X.device)
    arr = _module_structs([mod], [Y], r > 0)
    _check(lib().glowq_solo_forward_noalloc(arr, d, _ptr(B), r, _ptr(X), T, _stream(stream)),
           "glowq_solo_forward_noalloc")
    return Y


def noalloc_scratch_bytes() -> int:
    return int(lib().glowq_noalloc_scratch_bytes())


def device_status(stream=None) -> int:
    """Reads and clears the device status word (0 = ok, 5 = a bounded wait ran out)."""
    return int(lib().glowq_get_device_status(_stream(stream)))


def selftest_wait_timeout(polls: int = 4096, stream=None) -> None:
    """Enqueues the failure-path self-test (a bounded wait that must run out)."""
    _check(lib().glowq_selftest_wait_timeout(int(polls), _stream(stream)), "glowq_selftest_wait_timeout")


# ------------------------------------------------------------------- W4A8 ----

def quantize_act_e4m3(X, stream=None):
    """Per-token FP8 E4M3 activations: X (T x d fp16, CUDA) -> (codes uint8 [T, d],
    scales float32 [T], X_q fp16 [T, d] exact code values; x_hat = scales[:, None] * X_q)."""
    import torch
    _require_cuda(X)
    T, d = X.shape
    codes = torch.empty((T, d), dtype=torch.uint8, device=X.device)
    scales = torch.empty(T, dtype=torch.float32, device=X.device)
    Xq = torch.empty((T, d), dtype=torch.float16, device=X.device)
    _check(lib().glowq_quantize_act_e4m3(_ptr(X), T, d, _ptr(codes), _ptr(scales), _ptr(Xq), _stream(stream)),
           "glowq_quantize_act_e4m3")
    return codes, scales, Xq


def w4a8_workspace(T: int, d: int, r: int, device="cuda"):
    import torch
    n = max(int(lib().glowq_w4a8_workspace_bytes(T, d, r)), 16)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def group_forward_w4a8(mods: Sequence[QModule], B, X, Ys=None, R_out=None, workspace=None, stream=None):
    """group_forward with FP8 (E4M3, per-token scale) activations; X is fp16 and
    is quantised inside the call."""
    import torch
    _require_cuda(B, X)
    T, d = X.shape
    r = 0 if B is None else int(B.shape[0])
    if Ys is None:
        Ys = [torch.empty((T, m.out_features), dtype=torch.float16, device=X.device) for m in mods]
    if r > 0 and R_out is None:
        R_out = torch.empty((T, r), dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = w4a8_workspace(T, d, r, X.device)
    arr = _module_structs(mods, Ys, r > 0)
    ws_n = workspace.numel() * workspace.element_size()
    _check(lib().glowq_group_forward_w4a8(arr, len(mods), d, _ptr(B), r, _ptr(X), T, _ptr(R_out), _ptr(workspace),
                                          ws_n, _stream(stream)), "glowq_group_forward_w4a8")
    return Ys, R_out


def solo_forward_w4a8(mod: QModule, B, X, Y=None, workspace=None, stream=None):
    import torch
    _require_cuda(B, X)
    T, d = X.shape
    r = 0 if B is None else int(B.shape[0])
    if Y is None:
        Y = torch.empty((T, mod.out_features), dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = w4a8_workspace(T, d, r, X.device)
    arr = _module_structs([mod], [Y], r > 0)
    ws_n = workspace.numel() * workspace.element_size()
    _check(lib().glowq_solo_forward_w4a8(arr, d, _ptr(B), r, _ptr(X), T, _ptr(workspace), ws_n, _stream(stream)),
           "glowq_solo_forward_w4a8")
    return Y


# ---------------------------------------------------------- offline solve ----

def solve_workspace_bytes(rows: int, d: int, r: int, p: int) -> int:
    return int(lib().glowq_solve_workspace_bytes(rows, d, r, p))


def group_solve(Ws, packs, Sx_half, Sx_half_pinv, r: int, p: int, q: int, Omega, fp16=True, stream=None):
    """Whitened shared-B solve on the GPU for one group.  Ws: fp32 weights
    (O_i x d); packs: (qweight, scales, zeros) of each; Sx_half, Sx_half_pinv:
    d x d float64; Omega: d x (r+p) float64.  All CUDA tensors.  Returns
    (A float64 [M, r], B float64 [r, d], sing float64 [r], g_ec float64 [1],
    A16, B16 fp16 or None)."""
    import torch
    d = int(Ws[0].shape[1])
    M = sum(int(W.shape[0]) for W in Ws)
    dev = Ws[0].device
    for t in (*Ws, Sx_half, Sx_half_pinv, Omega):
        _require_cuda(t)
    items = [_SolveModule(W.data_ptr(), q_.data_ptr(), s_.data_ptr(), z_.data_ptr(), int(W.shape[0]))
             for W, (q_, s_, z_) in zip(Ws, packs)]
    arr = (_SolveModule * len(items))(*items)
    A = torch.empty((M, r), dtype=torch.float64, device=dev)
    B = torch.empty((r, d), dtype=torch.float64, device=dev)
    sing = torch.empty(r, dtype=torch.float64, device=dev)
    gec = torch.empty(1, dtype=torch.float64, device=dev)
    A16 = torch.empty((M, r), dtype=torch.float16, device=dev) if fp16 else None
    B16 = torch.empty((r, d), dtype=torch.float16, device=dev) if fp16 else None
    nws = max(solve_workspace_bytes(M, d, r, p), 16)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    _check(lib().glowq_group_solve(arr, len(items), d, _ptr(Sx_half), _ptr(Sx_half_pinv), r, p, q, _ptr(Omega),
                                   _ptr(A), _ptr(B), _ptr(sing), _ptr(gec), _ptr(A16), _ptr(B16), _ptr(ws), nws,
                                   _stream(stream)), "glowq_group_solve")
    return A, B, sing, gec, A16, B16


# ---------------------------------------------------------------- GlowQ-S ----

def select_restore(err_fro2, w_fro2, layer_idx, kind, k: int) -> Tuple["object", "object", bool]:
    """Host-only ranking by g_ner = err/w; returns (mask uint8[n], order int32[n], used_fallback)."""
    import numpy as np
    e = np.ascontiguousarray(err_fro2, dtype=np.float64)
    w = np.ascontiguousarray(w_fro2, dtype=np.float64)
    la = np.ascontiguousarray(layer_idx, dtype=np.int32)
    ki = np.ascontiguousarray(kind, dtype=np.int32)
    n = e.size
    mask = np.zeros(n, np.uint8)
    order = np.zeros(n, np.int32)
    fb = C.c_int32(0)
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    _check(lib().glowq_select_restore(p(e), p(w), p(la), p(ki), n, int(k), p(mask), p(order), C.byref(fb)),
           "glowq_select_restore")
    return mask, order, bool(fb.value)


def select_restore_scores(score, layer_idx, kind, k: int) -> Tuple["object", "object", bool]:
    """Host-only ranking by a caller-computed score (e.g. g_ec from the offline
    solve); returns (mask uint8[n], order int32[n], used_fallback)."""
    import numpy as np
    sc = np.ascontiguousarray(score, dtype=np.float64)
    la = np.ascontiguousarray(layer_idx, dtype=np.int32)
    ki = np.ascontiguousarray(kind, dtype=np.int32)
    n = sc.size
    mask = np.zeros(n, np.uint8)
    order = np.zeros(n, np.int32)
    fb = C.c_int32(0)
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    _check(lib().glowq_select_restore_scores(p(sc), p(la), p(ki), n, int(k), p(mask), p(order), C.byref(fb)),
           "glowq_select_restore_scores")
    return mask, order, bool(fb.value)
