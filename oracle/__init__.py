"""CPU oracle for the GlowQ corrected quantised linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product path
(``rank_error_correction_b200``) never does, and the two share no code.

All arithmetic lives in ``glowq_oracle.c`` (plain C, float64 except the fp32
quantiser decisions); this module only builds it with gcc and marshals numpy
arrays through ctypes.  See the C file's header for the passages of the GlowQ
pages each function follows and for the readings taken where they are silent.

Parity status: every exported function is pinned by tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "glowq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libglowq_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, strict IEEE)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _declare(_lib)
    return _lib


_p = C.c_void_p
_i64 = C.c_int64
_i32 = C.c_int32


def _declare(L):
    L.ora_f16_to_f64.argtypes = [C.c_uint16]
    L.ora_f16_to_f64.restype = C.c_double
    L.ora_f64_to_f16.argtypes = [C.c_double]
    L.ora_f64_to_f16.restype = C.c_uint16
    L.ora_f32_to_f16.argtypes = [C.c_float]
    L.ora_f32_to_f16.restype = C.c_uint16
    L.ora_quantize_int4.argtypes = [_p, _i64, _i64, _i32, _p, _p, _p]
    L.ora_unpack_int4.argtypes = [_p, _i64, _i64, _p]
    L.ora_dequant_int4.argtypes = [_p, _p, _p, _i64, _i64, _i32, _p]
    L.ora_quant_error.argtypes = [_p, _p, _p, _p, _i64, _i64, _i32, _p, _p, _p]
    L.ora_anchor_project.argtypes = [_p, _p, _i64, _i64, _i32, _p]
    L.ora_module_forward.argtypes = [_p, _p, _p, _i64, _i64, _i32, _p, _i32, _p, _p, _i64, _p]
    L.ora_solo_forward.argtypes = [_p, _p, _p, _i64, _i64, _i32, _p, _p, _i32, _p, _i64, _p]
    L.ora_module_forward_sampled.argtypes = [_p, _p, _p, _i64, _i64, _i32, _p, _p, _i32, _p,
                                             _i64, _i64, _p, _p, _p]
    L.ora_matmul.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i32, _i32]
    L.ora_householder_qr.argtypes = [_p, _i64, _i64, _p, _p]
    L.ora_jacobi_svd.argtypes = [_p, _i64, _i64, _p, _p, _p]
    L.ora_rsvd.argtypes = [_p, _i64, _i64, _i32, _i32, _i32, _p, _p, _p, _p]
    L.ora_group_solve.argtypes = [_p, _i64, _i64, _p, _p, _i32, _i32, _i32, _p, _p, _p, _p]
    L.ora_select_restore.argtypes = [_p, _p, _p, _p, _i32, _i32, _p, _p, _p]
    L.ora_select_by_score.argtypes = [_p, _p, _p, _i32, _i32, _p, _p]
    L.ora_set_threads.argtypes = [_i32]
    L.ora_set_threads.restype = C.c_int
    L.ora_e2m1_decode.argtypes = [C.c_uint8]
    L.ora_e2m1_decode.restype = C.c_double
    L.ora_e2m1_encode.argtypes = [C.c_float]
    L.ora_e2m1_encode.restype = C.c_uint8
    L.ora_e4m3_decode.argtypes = [C.c_uint8]
    L.ora_e4m3_decode.restype = C.c_double
    L.ora_e4m3_encode.argtypes = [C.c_float]
    L.ora_e4m3_encode.restype = C.c_uint8
    L.ora_e8m0_decode.argtypes = [C.c_uint8]
    L.ora_e8m0_decode.restype = C.c_double
    L.ora_quantize_mxfp4.argtypes = [_p, _i64, _i64, _p, _p]
    L.ora_dequant_mxfp4.argtypes = [_p, _p, _i64, _i64, _p]
    L.ora_quantize_nvfp4.argtypes = [_p, _i64, _i64, _p, _p, _p]
    L.ora_dequant_nvfp4.argtypes = [_p, _p, C.c_float, _i64, _i64, _p]
    L.ora_quantize_act_e4m3.argtypes = [_p, _i64, _i64, _p, _p]
    L.ora_dequant_act_e4m3.argtypes = [_p, _p, _i64, _i64, _p]
    for name in ("ora_quantize_int4", "ora_unpack_int4", "ora_dequant_int4", "ora_quant_error",
                 "ora_anchor_project", "ora_module_forward", "ora_solo_forward",
                 "ora_module_forward_sampled", "ora_matmul", "ora_householder_qr",
                 "ora_jacobi_svd", "ora_rsvd", "ora_group_solve", "ora_select_restore",
                 "ora_select_by_score", "ora_quantize_mxfp4", "ora_dequant_mxfp4", "ora_quantize_nvfp4",
                 "ora_dequant_nvfp4", "ora_quantize_act_e4m3", "ora_dequant_act_e4m3"):
        getattr(L, name).restype = C.c_int


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc < 0:
        raise ValueError(f"oracle {what} failed with code {rc}")
    return rc


# -- fp16 -------------------------------------------------------------------

def f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    out = np.fromiter((L.ora_f16_to_f64(int(b)) for b in flat), dtype=np.float64, count=flat.size)
    return out.reshape(np.shape(bits))


def f64_to_f16_bits(x: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(x, dtype=np.float64).ravel()
    out = np.fromiter((L.ora_f64_to_f16(float(v)) for v in flat), dtype=np.uint16, count=flat.size)
    return out.reshape(np.shape(x))


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(x, dtype=np.float32).ravel()
    out = np.fromiter((L.ora_f32_to_f16(float(v)) for v in flat), dtype=np.uint16, count=flat.size)
    return out.reshape(np.shape(x))


# -- quantisation -------------------------------------------------------------

def quantize_int4(W: np.ndarray, group_size: int = 128):
    """W (O x d fp32) -> (q [O, d/8] uint32, s [O, d/gs] fp16 bits, z [O, d/gs] uint8)."""
    W = _c(W, np.float32)
    O, d = W.shape
    q = np.zeros((O, d // 8), np.uint32)
    s = np.zeros((O, d // group_size), np.uint16)
    z = np.zeros((O, d // group_size), np.uint8)
    _check(lib().ora_quantize_int4(_ptr(W), O, d, group_size, _ptr(q), _ptr(s), _ptr(z)), "quantize")
    return q, s, z


def unpack_int4(q: np.ndarray, d: int) -> np.ndarray:
    q = _c(q, np.uint32)
    O = q.shape[0]
    out = np.zeros((O, d), np.uint8)
    _check(lib().ora_unpack_int4(_ptr(q), O, d, _ptr(out)), "unpack")
    return out


def dequant_int4(q, s, z, d: int, group_size: int = 128) -> np.ndarray:
    """-> fp16 bit patterns [O, d]."""
    q, s, z = _c(q, np.uint32), _c(s, np.uint16), _c(z, np.uint8)
    O = q.shape[0]
    out = np.zeros((O, d), np.uint16)
    _check(lib().ora_dequant_int4(_ptr(q), _ptr(s), _ptr(z), O, d, group_size, _ptr(out)), "dequant")
    return out


def quant_error(W, q, s, z, group_size: int = 128, want_matrix: bool = True):
    W = _c(W, np.float32)
    q, s, z = _c(q, np.uint32), _c(s, np.uint16), _c(z, np.uint8)
    O, d = W.shape
    E = np.zeros((O, d), np.float64) if want_matrix else None
    e2 = C.c_double()
    w2 = C.c_double()
    _check(lib().ora_quant_error(_ptr(W), _ptr(q), _ptr(s), _ptr(z), O, d, group_size, _ptr(E),
                                 C.byref(e2), C.byref(w2)), "quant_error")
    return E, e2.value, w2.value


# -- forward -------------------------------------------------------------------

def anchor_project(X_bits, B_bits) -> np.ndarray:
    X, B = _c(X_bits, np.uint16), _c(B_bits, np.uint16)
    T, d = X.shape
    r = B.shape[0]
    R = np.zeros((T, r), np.float64)
    _check(lib().ora_anchor_project(_ptr(X), _ptr(B), T, d, r, _ptr(R)), "anchor_project")
    return R


def module_forward(q, s, z, A_bits, R, X_bits, group_size: int = 128) -> np.ndarray:
    """One module of a group, given the group's shared R (float64, T x r) or None."""
    q, s, z = _c(q, np.uint32), _c(s, np.uint16), _c(z, np.uint8)
    X = _c(X_bits, np.uint16)
    T, d = X.shape
    O = q.shape[0]
    A = None if A_bits is None else _c(A_bits, np.uint16)
    Rm = None if R is None else _c(R, np.float64)
    r = 0 if (A is None or Rm is None) else A.shape[1]
    Y = np.zeros((T, O), np.float64)
    _check(lib().ora_module_forward(_ptr(q), _ptr(s), _ptr(z), O, d, group_size, _ptr(A), r,
                                    _ptr(Rm), _ptr(X), T, _ptr(Y)), "module_forward")
    return Y


def group_forward(mods, B_bits, X_bits, group_size: int = 128):
    """mods: list of (q, s, z, A_bits or None).  R = X B^T once, reused by all."""
    R = None if B_bits is None else anchor_project(X_bits, B_bits)
    return [module_forward(q, s, z, A, R, X_bits, group_size) for (q, s, z, A) in mods], R


def solo_forward(q, s, z, A_bits, B_bits, X_bits, group_size: int = 128) -> np.ndarray:
    q, s, z = _c(q, np.uint32), _c(s, np.uint16), _c(z, np.uint8)
    X = _c(X_bits, np.uint16)
    T, d = X.shape
    O = q.shape[0]
    A = None if A_bits is None else _c(A_bits, np.uint16)
    B = None if B_bits is None else _c(B_bits, np.uint16)
    r = 0 if (A is None or B is None) else B.shape[0]
    Y = np.zeros((T, O), np.float64)
    _check(lib().ora_solo_forward(_ptr(q), _ptr(s), _ptr(z), O, d, group_size, _ptr(A), _ptr(B), r,
                                  _ptr(X), T, _ptr(Y)), "solo_forward")
    return Y


def module_forward_sampled(q, s, z, A_bits, B_bits, X_bits, t_idx, o_idx, group_size: int = 128):
    q, s, z = _c(q, np.uint32), _c(s, np.uint16), _c(z, np.uint8)
    X = _c(X_bits, np.uint16)
    T, d = X.shape
    O = q.shape[0]
    A = None if A_bits is None else _c(A_bits, np.uint16)
    B = None if B_bits is None else _c(B_bits, np.uint16)
    r = 0 if (A is None or B is None) else B.shape[0]
    ti, oi = _c(t_idx, np.int64), _c(o_idx, np.int64)
    out = np.zeros(ti.size, np.float64)
    _check(lib().ora_module_forward_sampled(_ptr(q), _ptr(s), _ptr(z), O, d, group_size, _ptr(A),
                                            _ptr(B), r, _ptr(X), T, ti.size, _ptr(ti), _ptr(oi),
                                            _ptr(out)), "forward_sampled")
    return out


# -- offline solve -----------------------------------------------------------------

def set_threads(n: int = 0) -> int:
    """OpenMP threads of the forward loops (n >= 1 sets it; 0 only queries).
    Results do not depend on it: each output is one sequential sum."""
    return int(lib().ora_set_threads(int(n)))


def matmul(A, B, ta=False, tb=False):
    A, B = _c(A, np.float64), _c(B, np.float64)
    m = A.shape[1] if ta else A.shape[0]
    k = A.shape[0] if ta else A.shape[1]
    n = B.shape[0] if tb else B.shape[1]
    Cm = np.zeros((m, n), np.float64)
    lib().ora_matmul(_ptr(A), _ptr(B), _ptr(Cm), m, n, k, int(ta), int(tb))
    return Cm


def householder_qr(A):
    A = _c(A, np.float64)
    m, n = A.shape
    k = min(m, n)
    Q = np.zeros((m, k))
    R = np.zeros((k, n))
    _check(lib().ora_householder_qr(_ptr(A), m, n, _ptr(Q), _ptr(R)), "qr")
    return Q, R


def jacobi_svd(A):
    A = _c(A, np.float64)
    m, n = A.shape
    k = min(m, n)
    U = np.zeros((m, k))
    S = np.zeros(k)
    V = np.zeros((n, k))
    _check(lib().ora_jacobi_svd(_ptr(A), m, n, _ptr(U), _ptr(S), _ptr(V)), "svd")
    return U, S, V


def rsvd(M, rank, p, q, Omega):
    M, Om = _c(M, np.float64), _c(Omega, np.float64)
    m, n = M.shape
    U = np.zeros((m, rank))
    S = np.zeros(rank)
    V = np.zeros((n, rank))
    _check(lib().ora_rsvd(_ptr(M), m, n, rank, p, q, _ptr(Om), _ptr(U), _ptr(S), _ptr(V)), "rsvd")
    return U, S, V


def group_solve(E_cat, Sh, Shp, r, p=16, q=2, Omega=None):
    """Whitened shared-B solve: returns (A m x r, B r x d, singular values of M)."""
    E, Sh, Shp = _c(E_cat, np.float64), _c(Sh, np.float64), _c(Shp, np.float64)
    m, d = E.shape
    Om = None if Omega is None else _c(Omega, np.float64)
    A = np.zeros((m, r))
    B = np.zeros((r, d))
    sing = np.zeros(r)
    _check(lib().ora_group_solve(_ptr(E), m, d, _ptr(Sh), _ptr(Shp), r, p, q, _ptr(Om), _ptr(A),
                                 _ptr(B), _ptr(sing)), "group_solve")
    return A, B, sing


# -- narrow floating-point base weights (Table 13: MXFP4, NVFP4) ------------------

def e2m1_decode(code: int) -> float:
    return float(lib().ora_e2m1_decode(int(code)))


def e2m1_encode(v: float) -> int:
    return int(lib().ora_e2m1_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return float(lib().ora_e4m3_decode(int(code)))


def e4m3_encode(v: float) -> int:
    return int(lib().ora_e4m3_encode(float(v)))


def e8m0_decode(code: int) -> float:
    return float(lib().ora_e8m0_decode(int(code)))


def quantize_mxfp4(W):
    """W (O x d fp32, d % 32 == 0) -> (codes uint8 [O, d/2], scales uint8 E8M0 [O, d/32])."""
    W = _c(W, np.float32)
    O, d = W.shape
    codes = np.zeros((O, d // 2), np.uint8)
    scales = np.zeros((O, d // 32), np.uint8)
    _check(lib().ora_quantize_mxfp4(_ptr(W), O, d, _ptr(codes), _ptr(scales)), "quantize_mxfp4")
    return codes, scales


def dequant_mxfp4(codes, scales, d):
    """-> w_hat fp16 bits [O, d] (uint16)."""
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    O = codes.shape[0]
    out = np.zeros((O, d), np.uint16)
    _check(lib().ora_dequant_mxfp4(_ptr(codes), _ptr(scales), O, d, _ptr(out)), "dequant_mxfp4")
    return out


def quantize_nvfp4(W):
    """W (O x d fp32, d % 16 == 0) -> (codes uint8 [O, d/2], scales uint8 E4M3 [O, d/16], tensor scale)."""
    W = _c(W, np.float32)
    O, d = W.shape
    codes = np.zeros((O, d // 2), np.uint8)
    scales = np.zeros((O, d // 16), np.uint8)
    ts = np.zeros(1, np.float32)
    _check(lib().ora_quantize_nvfp4(_ptr(W), O, d, _ptr(codes), _ptr(scales), _ptr(ts)), "quantize_nvfp4")
    return codes, scales, float(ts[0])


def dequant_nvfp4(codes, scales, tensor_scale, d):
    """-> w_hat fp16 bits [O, d] (uint16)."""
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    O = codes.shape[0]
    out = np.zeros((O, d), np.uint16)
    _check(lib().ora_dequant_nvfp4(_ptr(codes), _ptr(scales), C.c_float(tensor_scale), O, d, _ptr(out)),
           "dequant_nvfp4")
    return out


def fp4_group_forward(fmt, mods, B_bits, X_bits):
    """W4A16 group forward with MXFP4 / NVFP4 base weights, float64: R = X B^T
    once, Y_i = X w_hat_i^T + R A_i^T with w_hat_i the format's dequantised
    fp16 weight.  fmt: "mx" or "nv"; mods: (codes uint8 [O, d/2], scales,
    tensor_scale or None, A_bits or None).  Returns ([Y_i], R)."""
    X = _c(X_bits, np.uint16)
    d = X.shape[1]
    R = None if B_bits is None else anchor_project(X, B_bits)
    Xd = f16_bits_to_f64(X)
    outs = []
    for (codes, scales, ts, A) in mods:
        Wb = dequant_mxfp4(codes, scales, d) if fmt == "mx" else dequant_nvfp4(codes, scales, ts, d)
        Y = matmul(Xd, f16_bits_to_f64(Wb), tb=True)
        if A is not None and R is not None:
            Y = Y + matmul(R, f16_bits_to_f64(A), tb=True)
        outs.append(Y)
    return outs, R


def quantize_act_e4m3(X_bits):
    """Per-token FP8 E4M3 activations: X (T x d fp16 bits) -> (codes uint8 [T, d], scales fp32 [T])."""
    X = _c(X_bits, np.uint16)
    T, d = X.shape
    codes = np.zeros((T, d), np.uint8)
    scales = np.zeros(T, np.float32)
    _check(lib().ora_quantize_act_e4m3(_ptr(X), T, d, _ptr(codes), _ptr(scales)), "quantize_act_e4m3")
    return codes, scales


def dequant_act_e4m3(codes, scales):
    codes, scales = _c(codes, np.uint8), _c(scales, np.float32)
    T, d = codes.shape
    out = np.zeros((T, d), np.float64)
    _check(lib().ora_dequant_act_e4m3(_ptr(codes), _ptr(scales), T, d, _ptr(out)), "dequant_act_e4m3")
    return out


def w4a8_group_forward(mods, B_bits, X_bits, group_size: int = 128):
    """W4A8 group forward (reading): the layer consumes the per-token FP8
    activations X_hat; R = X_hat B^T and Y_i = X_hat w_hat_i^T + R A_i^T, float64.
    mods: (q, s, z, A_bits or None).  Returns ([Y_i], R, X_hat)."""
    Xh = dequant_act_e4m3(*quantize_act_e4m3(X_bits))
    d = Xh.shape[1]
    R = None if B_bits is None else matmul(Xh, f16_bits_to_f64(B_bits), tb=True)
    outs = []
    for (q, s, z, A) in mods:
        What = f16_bits_to_f64(dequant_int4(q, s, z, d, group_size))
        Y = matmul(Xh, What, tb=True)
        if A is not None and R is not None:
            Y = Y + matmul(R, f16_bits_to_f64(A), tb=True)
        outs.append(Y)
    return outs, R, Xh


def energy_capture(E_cat, Sh, r):
    """GSVD energy-capture score of a unit (GlowQ pages, papernotes.org summary,
    key design 4): g_ec(u) = sum_{j<=r} sigma_j(M_u)^2 / ||M_u||_F^2, with M_u the
    covariance-aligned core of the unit's stacked error, M = R_e Sx^{1/2}
    (R_e from the thin QR of E_cat, key design 3).  Exact singular values of
    the core (one-sided Jacobi), so for small and mid sizes only; since
    ||M||_F^2 = sum_j sigma_j^2, 1 - g_ec is the best rank-r fit's relative
    residual of the covariance-weighted error."""
    _, Re = householder_qr(E_cat)
    M = matmul(Re, Sh)
    _, S, _ = jacobi_svd(M)
    s2 = S * S
    tot = float(np.sum(s2))
    return float(np.sum(s2[:r]) / tot) if tot > 0 else float("nan")


# -- GlowQ-S ---------------------------------------------------------------------

def select_by_score(score, layer, kind, k):
    """Rank units by any importance score (g_ec or g_ner), descending; exact
    ties and the weak-signal fallback as in select_restore.  Returns
    (mask, order, used_fallback)."""
    sc = _c(score, np.float64)
    la, ki = _c(layer, np.int32), _c(kind, np.int32)
    n = sc.size
    mask = np.zeros(n, np.uint8)
    order = np.zeros(n, np.int32)
    rc = _check(lib().ora_select_by_score(_ptr(sc), _ptr(la), _ptr(ki), n, k, _ptr(mask), _ptr(order)),
                "select_by_score")
    return mask, order, bool(rc == 1)


def select_restore(err_fro2, w_fro2, layer, kind, k):
    e, w = _c(err_fro2, np.float64), _c(w_fro2, np.float64)
    la, ki = _c(layer, np.int32), _c(kind, np.int32)
    n = e.size
    mask = np.zeros(n, np.uint8)
    order = np.zeros(n, np.int32)
    score = np.zeros(n, np.float64)
    rc = _check(lib().ora_select_restore(_ptr(e), _ptr(w), _ptr(la), _ptr(ki), n, k, _ptr(mask),
                                         _ptr(order), _ptr(score)), "select_restore")
    return mask, order, score, bool(rc == 1)
