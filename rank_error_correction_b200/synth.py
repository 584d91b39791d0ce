"""Seeded synthetic inputs for the GlowQ corrected linear layer.

This module only draws random numbers and arranges them into the shapes of the
workloads; it holds none of the method's arithmetic (no quantisation, no
factor solve, no forward).  Both the CUDA path's tests/benchmark and the CPU
oracle's tests take their inputs from here.

Recipe (the GlowQ pages' set-up: LLaMA-shaped W4A16 layers, rank 64,
heavy-tailed input spectra with power-law exponents alpha_QKV ~ 1.19 and
alpha_MLP ~ 0.77 -- papernotes.org key design 2 and the Figure 2 caption):

* weights W ~ N(0, 0.02^2) in fp32; the tiny QKV case also scales 4 seeded
  input columns by 10 (outlier channels);
* input covariance Sx = Q diag(lam) Q^T with lam_k proportional to k^-alpha,
  scaled to mean 1; Q is Haar-distributed (QR of a Gaussian, sign-fixed) for
  d <= 2048 and, above that, a product of 8 random Householder reflections
  applied to a random signed permutation (applied implicitly, O(T d) per
  reflection) so that large-d inputs stay cheap to draw;
* activations x_t = Q (sqrt(lam) * g_t), g_t ~ N(0, I), rounded to fp16;
* correction factors, where the offline solve is too slow for the CPU, are
  seeded Gaussians of the solve's typical magnitude: A ~ N(0, 0.005^2),
  B ~ N(0, 0.01^2), both rounded to fp16.

Every tensor draws from its own counter-based Philox stream keyed by
(seed, stream id), so any tensor can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

ALPHA_QKV = 1.19
ALPHA_MLP = 0.77

# stream ids (one per tensor role)
S_W, S_OUTLIER, S_BASIS, S_X, S_A, S_B, S_OMEGA = 1, 2, 3, 4, 5, 6, 7


def rng(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    """Philox4x64 keyed by (seed, stream, sub)."""
    key = (int(seed) & 0xFFFFFFFFFFFFFFFF) | ((int(stream) * 1000003 + int(sub)) << 64)
    return np.random.Generator(np.random.Philox(key=key))


def weights(O: int, d: int, seed: int = 0, stream_sub: int = 0, std: float = 0.02,
            outlier_cols: int = 0, outlier_scale: float = 10.0) -> np.ndarray:
    """W ~ N(0, std^2) (O x d fp32); optionally `outlier_cols` seeded input columns x scale."""
    g = rng(seed, S_W, stream_sub)
    W = (g.standard_normal((O, d), dtype=np.float32) * np.float32(std)).astype(np.float32)
    if outlier_cols:
        cols = outlier_columns(d, outlier_cols, seed)
        W[:, cols] *= np.float32(outlier_scale)
    return W


def outlier_columns(d: int, n: int, seed: int = 0) -> np.ndarray:
    return np.sort(rng(seed, S_OUTLIER).choice(d, size=n, replace=False))


def power_law_spectrum(d: int, alpha: float) -> np.ndarray:
    """lam_k = k^-alpha, k = 1..d, scaled to mean 1."""
    lam = np.arange(1, d + 1, dtype=np.float64) ** (-float(alpha))
    return lam * (d / lam.sum())


@dataclasses.dataclass
class Basis:
    """Random orthogonal Q: either an explicit matrix or an implicit product."""
    d: int
    matrix: Optional[np.ndarray] = None          # explicit Q (d x d)
    perm: Optional[np.ndarray] = None            # implicit: signed permutation ...
    signs: Optional[np.ndarray] = None
    reflectors: Optional[List[np.ndarray]] = None  # ... then H_k ... H_1 (unit vectors)

    def apply(self, Z: np.ndarray) -> np.ndarray:
        """Rows z_t -> rows (Q z_t); Z is T x d float64."""
        if self.matrix is not None:
            return Z @ self.matrix.T
        Y = Z[:, self.perm] * self.signs
        for v in self.reflectors:
            Y = Y - 2.0 * np.outer(Y @ v, v)
        return Y

    def dense(self) -> np.ndarray:
        if self.matrix is not None:
            return self.matrix
        return self.apply(np.eye(self.d)).T


def orthogonal_basis(d: int, seed: int = 0, sub: int = 0, haar_max: int = 2048) -> Basis:
    g = rng(seed, S_BASIS, sub)
    if d <= haar_max:
        Gm = g.standard_normal((d, d))
        Q, R = np.linalg.qr(Gm)
        Q = Q * np.sign(np.diag(R))[None, :]
        return Basis(d=d, matrix=Q)
    perm = g.permutation(d)
    signs = np.where(g.random(d) < 0.5, -1.0, 1.0)
    refl = []
    for _ in range(8):
        v = g.standard_normal(d)
        refl.append(v / np.linalg.norm(v))
    return Basis(d=d, perm=perm, signs=signs, reflectors=refl)


def activations(T: int, d: int, alpha: float, seed: int = 0, sub: int = 0,
                basis: Optional[Basis] = None) -> np.ndarray:
    """X (T x d) ~ N(0, Sx) rounded to fp16; returned as np.float16."""
    lam = power_law_spectrum(d, alpha)
    Q = basis if basis is not None else orthogonal_basis(d, seed, sub)
    Gz = rng(seed, S_X, sub).standard_normal((T, d))
    X = Q.apply(Gz * np.sqrt(lam)[None, :])
    return X.astype(np.float16)


def covariance_half(basis: Basis, lam: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Population Sx^{1/2} = Q diag(sqrt lam) Q^T and its pseudo-inverse (by construction)."""
    Q = basis.dense()
    sq = np.sqrt(lam)
    inv = np.where(sq > 0, 1.0 / np.where(sq > 0, sq, 1.0), 0.0)
    return (Q * sq[None, :]) @ Q.T, (Q * inv[None, :]) @ Q.T


def random_factors(out_features: List[int], d: int, r: int, seed: int = 0, sub: int = 0,
                   a_std: float = 0.005, b_std: float = 0.01):
    """Seeded stand-in factors: ([A_i (O_i x r) fp16], B (r x d) fp16)."""
    As = []
    for i, O in enumerate(out_features):
        As.append((rng(seed, S_A, sub * 64 + i).standard_normal((O, r)) * a_std).astype(np.float16))
    B = (rng(seed, S_B, sub).standard_normal((r, d)) * b_std).astype(np.float16)
    return As, B


def gaussian_test_matrix(n: int, l: int, seed: int = 0, sub: int = 0) -> np.ndarray:
    """Omega (n x l) for the randomised SVD."""
    return rng(seed, S_OMEGA, sub).standard_normal((n, l))


def bits(a: np.ndarray) -> np.ndarray:
    """fp16 array -> uint16 bit patterns (a view)."""
    return np.ascontiguousarray(a, dtype=np.float16).view(np.uint16)


# ----------------------------------------------------------------------------
# The workloads: LLaMA-shaped input-sharing groups and solo modules.
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class GroupSpec:
    name: str
    d: int
    outs: List[int]          # out_features per module; anchor first
    alpha: float
    r: int


@dataclasses.dataclass
class Workload:
    name: str
    groups: List[GroupSpec]  # input-sharing groups (m >= 2) and solos (m == 1)
    tokens: List[int]
    layers: int = 1
    restore_fraction: float = 1.0


WORKLOADS: Dict[str, Workload] = {
    "tiny_qkv": Workload(
        "tiny QKV group d=256, r=16, T=8",
        [GroupSpec("qkv", 256, [256, 256, 256], ALPHA_QKV, 16)], [8]),
    "llama2_7b_attn_decode": Workload(
        "LLaMA-2-7B attention: QKV group 3x4096x4096 + o_proj 4096x4096, r=64",
        [GroupSpec("qkv", 4096, [4096, 4096, 4096], ALPHA_QKV, 64),
         GroupSpec("o_proj", 4096, [4096], ALPHA_QKV, 64)], [1, 4, 16]),
    "llama2_7b_mlp_prefill": Workload(
        "LLaMA-2-7B MLP: gate/up group 2x11008x4096 + down_proj 4096x11008, r=64",
        [GroupSpec("gate_up", 4096, [11008, 11008], ALPHA_MLP, 64),
         GroupSpec("down_proj", 11008, [4096], ALPHA_MLP, 64)], [2048]),
    "llama31_8b_layer": Workload(
        "LLaMA-3.1-8B GQA layer: QKV 4096+1024+1024, gate/up 2x14336, o 4096, down 14336->4096, r=64",
        [GroupSpec("qkv", 4096, [4096, 1024, 1024], ALPHA_QKV, 64),
         GroupSpec("o_proj", 4096, [4096], ALPHA_QKV, 64),
         GroupSpec("gate_up", 4096, [14336, 14336], ALPHA_MLP, 64),
         GroupSpec("down_proj", 14336, [4096], ALPHA_MLP, 64)], [1, 4096]),
    "llama2_13b_stack": Workload(
        "LLaMA-2-13B 40-layer linear stack d=5120 ffn 13824, r=64, GlowQ-S 50%",
        [GroupSpec("qkv", 5120, [5120, 5120, 5120], ALPHA_QKV, 64),
         GroupSpec("o_proj", 5120, [5120], ALPHA_QKV, 64),
         GroupSpec("gate_up", 5120, [13824, 13824], ALPHA_MLP, 64),
         GroupSpec("down_proj", 13824, [5120], ALPHA_MLP, 64)], [1, 16, 64, 2048],
        layers=40, restore_fraction=0.5),
}


# ----------------------------------------------------------------------------
# Device-side draws for the benchmark (same distributions, drawn on the GPU so
# that hundreds of MB of weights need no host round trip).
# ----------------------------------------------------------------------------

def _torch_seed(seed: int, stream: int, sub: int) -> int:
    return (int(seed) * 0x9E3779B1 + int(stream) * 0x85EBCA77 + int(sub) * 0xC2B2AE3D) & 0x7FFFFFFFFFFFFFFF


def device_weights(O: int, d: int, seed: int, sub: int, device="cuda", std: float = 0.02):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(_torch_seed(seed, S_W, sub))
    return torch.randn((O, d), generator=g, device=device, dtype=torch.float32) * std


def device_factors(out_features: List[int], d: int, r: int, seed: int, sub: int, device="cuda",
                   a_std: float = 0.005, b_std: float = 0.01):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(_torch_seed(seed, S_A, sub))
    As = [(torch.randn((O, r), generator=g, device=device) * a_std).half() for O in out_features]
    g.manual_seed(_torch_seed(seed, S_B, sub))
    B = (torch.randn((r, d), generator=g, device=device) * b_std).half()
    return As, B


def device_activations(T: int, d: int, seed: int, sub: int, device="cuda"):
    """Timing-only stand-in for X on the device: iid N(0, 1) rounded to fp16, the
    same mean power per coordinate as the unit-mean power-law inputs (their
    correlation structure matters for the solve and the parity tests, not for
    the kernels' speed)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(_torch_seed(seed, S_X, sub))
    return torch.randn((T, d), generator=g, device=device, dtype=torch.float32).half()

