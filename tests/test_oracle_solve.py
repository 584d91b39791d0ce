"""Pins for the oracle's offline group solve (QR core, Jacobi SVD, Halko rSVD).

Pages: papernotes.org GlowQ summary, key designs 1-3 (Proposition 1: the shared
B spans the top-r right singular subspace of E_cat by Eckart-Young-Mirsky;
Propositions 2/3: covariance-aligned risk ||(E - AB) Sx^{1/2}||_F^2, isotropic
case = plain stacked SVD; thin QR core M = R_e Sx^{1/2}, randomised SVD with
oversampling p and q power iterations, balanced split lifted back with the
pseudo-inverse); thelatestinai.com GlowQ page, Table 6 (shapes) and the
Table 11/12 captions (Halko rSVD, p = 16 and q = 2 as the sweeps' fixed values).
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import synth


def _stacked_error(d, outs, seed):
    Es = []
    for i, O in enumerate(outs):
        W = synth.weights(O, d, seed=seed, stream_sub=i, outlier_cols=2)
        q, s, z = oracle.quantize_int4(W, group_size=min(128, d))
        Es.append(oracle.quant_error(W, q, s, z, group_size=min(128, d))[0])
    return np.vstack(Es)


def test_householder_qr():
    g = np.random.default_rng(0)
    for m, n in [(40, 12), (12, 40), (16, 16)]:
        A = g.standard_normal((m, n))
        Q, R = oracle.householder_qr(A)
        k = min(m, n)
        assert np.allclose(Q.T @ Q, np.eye(k), atol=1e-13)
        assert np.allclose(Q @ R, A, atol=1e-12)
        assert np.allclose(np.tril(R, -1), 0.0)
        assert np.allclose(np.abs(np.diag(R)), np.abs(np.diag(np.linalg.qr(A)[1])), rtol=1e-10)


@pytest.mark.parametrize("shape", [(30, 10), (10, 30), (25, 25)])
def test_jacobi_svd_matches_library(shape):
    A = np.random.default_rng(1).standard_normal(shape)
    U, S, V = oracle.jacobi_svd(A)
    assert np.allclose(S, np.linalg.svd(A, compute_uv=False), rtol=1e-12)
    assert np.allclose((U * S) @ V.T, A, atol=1e-12)
    assert np.allclose(U.T @ U, np.eye(min(shape)), atol=1e-12)
    assert np.allclose(V.T @ V, np.eye(min(shape)), atol=1e-12)


def test_jacobi_svd_rank_deficient():
    g = np.random.default_rng(2)
    A = g.standard_normal((20, 3)) @ g.standard_normal((3, 8))
    U, S, V = oracle.jacobi_svd(A)
    assert np.allclose(S[3:], 0.0, atol=1e-12)
    assert np.allclose(U.T @ U, np.eye(8), atol=1e-8)
    assert np.allclose((U * S) @ V.T, A, atol=1e-12)


def _principal_cosines(B1, B2):
    Q1 = np.linalg.qr(B1.T)[0]
    Q2 = np.linalg.qr(B2.T)[0]
    return np.linalg.svd(Q1.T @ Q2, compute_uv=False)


def test_prop1_shared_B_is_top_right_subspace_of_stack():
    """Sx = I: ||E - AB||_F^2 equals the tail energy; rows(B) = span of top-r right vectors."""
    d, r = 32, 6
    E = _stacked_error(d, [32, 32, 32], seed=3) * 100.0
    I = np.eye(d)
    A, B, sing = oracle.group_solve(E, I, I, r, Omega=None)
    sv = np.linalg.svd(E, compute_uv=False)
    resid = np.linalg.norm(E - A @ B) ** 2
    assert resid == pytest.approx(np.sum(sv[r:] ** 2), rel=1e-10)
    assert np.allclose(sing, sv[:r], rtol=1e-11)
    Vt = np.linalg.svd(E)[2]
    assert np.allclose(_principal_cosines(B, Vt[:r]), 1.0, atol=1e-10)
    # balanced split: A^T A = B B^T = diag(sigma)
    assert np.allclose(A.T @ A, np.diag(sing), atol=1e-10)
    assert np.allclose(B @ B.T, np.diag(sing), atol=1e-10)


def test_isotropic_whitening_reduces_to_stacked_svd():
    d, r = 24, 5
    E = _stacked_error(d, [24, 16], seed=4) * 100.0
    c = 2.5                                          # Sx = c I -> Sx^{1/2} = sqrt(c) I
    A, B, _ = oracle.group_solve(E, np.sqrt(c) * np.eye(d), np.eye(d) / np.sqrt(c), r)
    U, S, Vt = np.linalg.svd(E)
    assert np.allclose(A @ B, (U[:, :r] * S[:r]) @ Vt[:r], atol=1e-12)


def test_whitened_solve_minimises_covariance_weighted_risk():
    d, r, N = 32, 4, 4000
    E = _stacked_error(d, [32, 32, 32], seed=6) * 100.0
    basis = synth.orthogonal_basis(d, seed=6)
    lam = synth.power_law_spectrum(d, synth.ALPHA_QKV)
    Sh, Shp = synth.covariance_half(basis, lam)
    A, B, sing = oracle.group_solve(E, Sh, Shp, r)
    risk = np.linalg.norm((E - A @ B) @ Sh) ** 2
    # closed-form optimum: tail energy of E Sx^{1/2}
    sv = np.linalg.svd(E @ Sh, compute_uv=False)
    assert risk == pytest.approx(np.sum(sv[r:] ** 2), rel=1e-9)
    assert np.allclose(sing, sv[:r], rtol=1e-10)            # QR core keeps the spectrum
    # usage-weighted risk identity with the empirical second moment
    X = basis.apply(np.random.default_rng(7).standard_normal((N, d)) * np.sqrt(lam))
    Se = X.T @ X / N
    w, V = np.linalg.eigh(Se)
    Se_h = (V * np.sqrt(np.clip(w, 0, None))) @ V.T
    M = E - A @ B
    assert np.mean(np.sum((X @ M.T) ** 2, axis=1)) == pytest.approx(np.linalg.norm(M @ Se_h) ** 2, rel=1e-10)
    # unwhitened solve and random competitors never beat it on the weighted risk
    Au, Bu, _ = oracle.group_solve(E, np.eye(d), np.eye(d), r)
    assert np.linalg.norm((E - Au @ Bu) @ Sh) ** 2 >= risk * (1 - 1e-12)
    g = np.random.default_rng(8)
    for _ in range(20):
        Bc = g.standard_normal((r, d))
        Ac = E @ Sh @ np.linalg.pinv(Bc @ Sh)       # best A for that B
        assert np.linalg.norm((E - Ac @ Bc) @ Sh) ** 2 >= risk * (1 - 1e-12)


def test_full_rank_reconstructs_error_exactly():
    """r = d (m >= d), invertible Sx: w_hat + A B = W, so the correction is lossless."""
    d = 16
    outs = [16, 16, 16]
    Ws, Es = [], []
    for i, O in enumerate(outs):
        W = synth.weights(O, d, seed=9, stream_sub=i)
        q, s, z = oracle.quantize_int4(W, group_size=16)
        Ws.append((W, q, s, z))
        Es.append(oracle.quant_error(W, q, s, z, group_size=16)[0])
    E = np.vstack(Es)
    basis = synth.orthogonal_basis(d, seed=9)
    Sh, Shp = synth.covariance_half(basis, synth.power_law_spectrum(d, 1.19))
    A, B, _ = oracle.group_solve(E, Sh, Shp, d)
    row = 0
    for (W, q, s, z) in Ws:
        what = oracle.dequant_int4(q, s, z, d, group_size=16).view(np.float16).astype(np.float64)
        rec = what + A[row:row + W.shape[0]] @ B
        row += W.shape[0]
        assert np.allclose(rec, W.astype(np.float64), atol=1e-12)


def test_wide_stack_core_is_m_by_d():
    """m < d (a solo module with fewer outputs than inputs): the core is m x d."""
    d, r = 48, 5
    E = _stacked_error(d, [20], seed=10) * 100.0
    A, B, sing = oracle.group_solve(E, np.eye(d), np.eye(d), r)
    sv = np.linalg.svd(E, compute_uv=False)
    assert np.linalg.norm(E - A @ B) ** 2 == pytest.approx(np.sum(sv[r:] ** 2), rel=1e-10)


def test_rsvd_exact_on_low_rank_and_converges_with_power_steps():
    g = np.random.default_rng(11)
    m, n, r, p = 60, 50, 6, 4
    L = g.standard_normal((m, r)) @ g.standard_normal((r, n))
    Om = g.standard_normal((n, r + p))
    U, S, V = oracle.rsvd(L, r, p, 0, Om)
    assert np.allclose((U * S) @ V.T, L, atol=1e-10)
    # decaying spectrum: error of the top-r approximation shrinks with q
    Uo = np.linalg.qr(g.standard_normal((m, n)))[0]
    Vo = np.linalg.qr(g.standard_normal((n, n)))[0]
    sv = np.arange(1, n + 1) ** -0.8
    M = (Uo * sv) @ Vo.T
    best = np.sqrt(np.sum(sv[r:] ** 2))
    errs = []
    for q in [0, 1, 2, 4]:
        U, S, V = oracle.rsvd(M, r, p, q, Om)
        errs.append(np.linalg.norm(M - (U * S) @ V.T))
        assert np.allclose(U.T @ U, np.eye(r), atol=1e-10)
    assert errs[-1] <= errs[0] + 1e-12
    assert errs[2] <= best * 1.05          # q = 2 is near-optimal
    assert all(e >= best * (1 - 1e-12) for e in errs)


def test_rsvd_solve_close_to_exact_solve():
    d, r, p, q = 64, 8, 16, 2
    E = _stacked_error(d, [64, 64], seed=12) * 100.0
    basis = synth.orthogonal_basis(d, seed=12)
    Sh, Shp = synth.covariance_half(basis, synth.power_law_spectrum(d, 0.77))
    Ae, Be, se = oracle.group_solve(E, Sh, Shp, r)
    Ar, Br, sr = oracle.group_solve(E, Sh, Shp, r, p=p, q=q,
                                    Omega=synth.gaussian_test_matrix(d, r + p, seed=12))
    re = np.linalg.norm((E - Ae @ Be) @ Sh)
    rr = np.linalg.norm((E - Ar @ Br) @ Sh)
    assert re <= rr * (1 + 1e-12)
    assert rr <= re * 1.02
    assert np.allclose(sr, se, rtol=2e-2)


# -- GSVD energy-capture score g_ec (key design 4) ------------------------------

def test_energy_capture_closed_form_on_known_spectrum():
    """E = U diag(sv) V^T with known singular values and Sx = I: the core's
    singular values are sv, so g_ec = sum of the top-r squares / sum of all."""
    g = np.random.default_rng(20)
    m, d = 18, 7
    U, _ = np.linalg.qr(g.standard_normal((m, d)))
    V, _ = np.linalg.qr(g.standard_normal((d, d)))
    sv = np.array([5.0, 3.0, 2.0, 1.0, 0.5, 0.25, 0.125])
    E = U @ np.diag(sv) @ V.T
    for r in range(1, d + 1):
        want = np.sum(sv[:r] ** 2) / np.sum(sv ** 2)
        assert oracle.energy_capture(E, np.eye(d), r) == pytest.approx(want, rel=1e-12)


def test_energy_capture_is_the_best_fit_share_of_the_solve():
    """Eckart-Young-Mirsky tie to the solve: with the exact core SVD,
    1 - g_ec = ||(E - A B) Sx^{1/2}||_F^2 / ||E Sx^{1/2}||_F^2 at the same rank."""
    d, r = 32, 6
    E = _stacked_error(d, [24, 16, 16], seed=21) * 100.0
    basis = synth.orthogonal_basis(d, seed=21)
    Sh, Shp = synth.covariance_half(basis, synth.power_law_spectrum(d, 0.77))
    A, B, _ = oracle.group_solve(E, Sh, Shp, r)          # exact (Jacobi) core SVD
    resid = np.linalg.norm((E - A @ B) @ Sh) ** 2 / np.linalg.norm(E @ Sh) ** 2
    assert 1.0 - oracle.energy_capture(E, Sh, r) == pytest.approx(resid, rel=1e-9)


def test_energy_capture_invariances_and_range():
    g = np.random.default_rng(22)
    m, d = 20, 9
    E = g.standard_normal((m, d)) * np.linspace(3.0, 0.1, d)
    Sh = np.diag(np.linspace(1.5, 0.5, d))
    base = [oracle.energy_capture(E, Sh, r) for r in range(1, d + 1)]
    assert all(0.0 < v <= 1.0 + 1e-12 for v in base)
    assert all(b >= a - 1e-12 for a, b in zip(base, base[1:]))    # non-decreasing in r
    assert base[-1] == pytest.approx(1.0, abs=1e-12)              # r = rank captures everything
    Q, _ = np.linalg.qr(g.standard_normal((m, m)))                # rows mixed orthogonally
    assert [oracle.energy_capture(Q @ E, Sh, r) for r in range(1, d + 1)] == pytest.approx(base, rel=1e-10)
    assert [oracle.energy_capture(7.0 * E, Sh, r) for r in range(1, d + 1)] == pytest.approx(base, rel=1e-10)


def test_qr_core_is_lossless_and_whitened_split_is_balanced():
    """Key design 3: the thin QR core keeps the singular values of E Sx^{1/2}
    (left-orthogonal invariance), and the lifted factors are balanced in the
    whitened metric: A^T A = (B Sx^{1/2})(B Sx^{1/2})^T = diag(sigma_1..r)."""
    d, r = 24, 5
    E = _stacked_error(d, [20, 12, 12], seed=23) * 100.0
    basis = synth.orthogonal_basis(d, seed=23)
    Sh, Shp = synth.covariance_half(basis, synth.power_law_spectrum(d, 1.19))
    _, Re = oracle.householder_qr(E)
    sv_core = oracle.jacobi_svd(oracle.matmul(Re, Sh))[1]
    sv_full = np.linalg.svd(E @ Sh, compute_uv=False)
    assert np.allclose(sv_core, sv_full[:sv_core.size], rtol=1e-11, atol=1e-12 * sv_full[0])
    A, B, sing = oracle.group_solve(E, Sh, Shp, r)
    assert np.allclose(sing, sv_full[:r], rtol=1e-11)
    assert np.allclose(A.T @ A, np.diag(sing), rtol=1e-9, atol=1e-9 * sing[0])
    BS = B @ Sh
    assert np.allclose(BS @ BS.T, np.diag(sing), rtol=1e-9, atol=1e-9 * sing[0])
