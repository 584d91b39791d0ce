"""Shared builders for the GPU parity tests: seeded inputs, oracle-side packing
and references, and the normwise comparison used as the parity bar."""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

import oracle
from rank_error_correction_b200 import synth

# Normwise relative error bar for fp16 outputs with fp32 accumulation: the
# output rounding alone contributes up to 2^-11 ~ 4.9e-4 per element; R's fp16
# rounding enters only through the ~1-2% correction term.
TOL = 2e-3

# Per-element bound beside the normwise bar:
#   |y_gpu - y_ora| <= ELEM_REL * |y_ora| + ELEM_ABS * max|y_ora|
# ELEM_REL = 2^-10 covers the fp16 rounding of y (2^-11 relative) twice over;
# ELEM_ABS = 2^-10 of the output's largest magnitude covers what does not scale
# with the element itself: fp32 accumulation over d <= 14336 terms, the decode
# kernel's exact (q - z) s weights against the oracle's fp16-rounded w_hat
# (<= 2^-12 per weight, random in sign), and R rounded to fp16 in the
# correction term.  Near-zero outputs are held to the absolute part only.
ELEM_REL = 2.0 ** -10
ELEM_ABS = 2.0 ** -10


@dataclasses.dataclass
class HostModule:
    W: np.ndarray            # fp32 O x d
    q: np.ndarray
    s: np.ndarray
    z: np.ndarray
    A: Optional[np.ndarray]  # fp16 O x r or None


def make_modules(d: int, outs: List[int], seed: int, sub0: int = 0, outlier_cols: int = 0) -> List[HostModule]:
    mods = []
    for i, O in enumerate(outs):
        W = synth.weights(O, d, seed=seed, stream_sub=sub0 + i, outlier_cols=outlier_cols)
        q, s, z = oracle.quantize_int4(W)
        mods.append(HostModule(W, q, s, z, None))
    return mods


def attach_random_factors(mods: List[HostModule], d: int, r: int, seed: int, sub: int = 0):
    As, B = synth.random_factors([m.W.shape[0] for m in mods], d, r, seed=seed, sub=sub)
    for m, A in zip(mods, As):
        m.A = A
    return B


def attach_solved_factors(mods: List[HostModule], d: int, r: int, alpha: float, seed: int,
                          basis=None, p: int = 16, q: int = 2):
    """Whitened stacked solve (oracle) with the population covariance; returns B fp16."""
    E = np.vstack([oracle.quant_error(m.W, m.q, m.s, m.z)[0] for m in mods])
    basis = basis if basis is not None else synth.orthogonal_basis(d, seed=seed)
    lam = synth.power_law_spectrum(d, alpha)
    Sh, Shp = synth.covariance_half(basis, lam)
    A, B, _ = oracle.group_solve(E, Sh, Shp, r, p=p, q=q,
                                 Omega=synth.gaussian_test_matrix(d, r + p, seed=seed))
    row = 0
    for m in mods:
        O = m.W.shape[0]
        m.A = A[row:row + O].astype(np.float16)
        row += O
    return B.astype(np.float16)


def normwise(y_gpu: np.ndarray, y_ref: np.ndarray) -> float:
    den = np.linalg.norm(y_ref)
    return float(np.linalg.norm(y_gpu.astype(np.float64) - y_ref) / (den if den > 0 else 1.0))


def elementwise_excess(y_gpu: np.ndarray, y_ref: np.ndarray, ymax: Optional[float] = None) -> float:
    """Largest |y_gpu - y_ref| / (ELEM_REL |y_ref| + ELEM_ABS ymax); <= 1 passes."""
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if y_ref.size == 0:
        return 0.0
    ymax = float(np.max(np.abs(y_ref))) if ymax is None else float(ymax)
    bound = ELEM_REL * np.abs(y_ref) + ELEM_ABS * max(ymax, 1e-30)
    return float(np.max(np.abs(np.asarray(y_gpu, dtype=np.float64) - y_ref) / bound))


def check(y_gpu: np.ndarray, y_ref: np.ndarray, ymax: Optional[float] = None, tol: float = TOL) -> None:
    """The parity bar of a module's output: normwise relative error <= tol and
    every element inside the per-element bound."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    assert y_gpu.shape == np.shape(y_ref), (y_gpu.shape, np.shape(y_ref))
    assert np.all(np.isfinite(y_gpu)), "non-finite output"
    nw = normwise(y_gpu, y_ref)
    assert nw < tol, f"normwise {nw:.3e} >= {tol:.1e}"
    ex = elementwise_excess(y_gpu, y_ref, ymax)
    assert ex <= 1.0, f"per-element bound exceeded by {ex:.2f}x"


def tile_int4(q: np.ndarray) -> np.ndarray:
    """Row-major INT4 words [O][d/8] (the oracle's layout) -> the library's
    block layout: 16-row x 64-k blocks of 16 x 8 words, blocks along k within
    a 16-row tile, tiles in row order (returned with shape [O, d/8])."""
    O, w = q.shape
    return np.ascontiguousarray(q.reshape(O // 16, 16, w // 8, 8).transpose(0, 2, 1, 3)).reshape(O, w)


def untile_int4(q: np.ndarray) -> np.ndarray:
    """Inverse of tile_int4."""
    O, w = q.shape
    return np.ascontiguousarray(q.reshape(O // 16, w // 8, 16, 8).transpose(0, 2, 1, 3)).reshape(O, w)


def to_dev(mods: List[HostModule], device="cuda", with_A: bool = True):
    import torch
    from rank_error_correction_b200 import glowq
    out = []
    for m in mods:
        out.append(glowq.QModule(
            torch.from_numpy(tile_int4(m.q).view(np.int32)).to(device),
            torch.from_numpy(m.s.view(np.float16)).to(device),
            torch.from_numpy(m.z).to(device),
            None if (m.A is None or not with_A) else torch.from_numpy(m.A).to(device)))
    return out
