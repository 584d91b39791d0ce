"""Pins for the oracle's corrected forward y_i = w_hat_i X + A_i (B X).

Pages: papernotes.org GlowQ summary, key design 4 (R = X B_shared^T computed
once per input-sharing group, y_i = W_i^(q) X + A_i R; Q/gate anchors, K/V/up
consumers; o_proj/down_proj solo, computed inline).  Pins: the plain definition
evaluated with numpy's matmul in a different association order, cached-vs-
recomputed R, sampled entries, r = 0 and empty-token edge cases.
"""
import numpy as np

import oracle
from rank_error_correction_b200 import synth


def _module(O, d, r, seed, sub):
    W = synth.weights(O, d, seed=seed, stream_sub=sub)
    q, s, z = oracle.quantize_int4(W)
    A = (synth.rng(seed, synth.S_A, sub).standard_normal((O, r)) * 0.005).astype(np.float16)
    return W, q, s, z, A


def _dense(q, s, z, d):
    return oracle.dequant_int4(q, s, z, d).view(np.float16).astype(np.float64)


def test_module_forward_matches_definition_in_other_order():
    d, r, T = 384, 24, 5
    W, q, s, z, A = _module(200, d, r, 0, 0)
    B = (synth.rng(0, synth.S_B).standard_normal((r, d)) * 0.01).astype(np.float16)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=0)
    Y = oracle.solo_forward(q, s, z, synth.bits(A), synth.bits(B), synth.bits(X))
    # definition, associated as X (w_hat + A B)^T
    Wc = _dense(q, s, z, d) + A.astype(np.float64) @ B.astype(np.float64)
    ref = X.astype(np.float64) @ Wc.T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    # and a plausible transposition mistake would be far off
    assert not np.allclose(Y, X.astype(np.float64) @ _dense(q, s, z, d).T, atol=1e-6)


def test_group_cached_R_equals_recomputed_per_module():
    d, r, T = 256, 16, 8
    mods = [_module(O, d, r, 1, i) for i, O in enumerate([256, 128, 128])]
    B = (synth.rng(1, synth.S_B).standard_normal((r, d)) * 0.01).astype(np.float16)
    X = synth.bits(synth.activations(T, d, synth.ALPHA_QKV, seed=1))
    outs, R = oracle.group_forward([(q, s, z, synth.bits(A)) for (_, q, s, z, A) in mods],
                                   synth.bits(B), X)
    assert R.shape == (T, r)
    assert np.allclose(R, X.view(np.float16).astype(np.float64) @ B.astype(np.float64).T, rtol=1e-13)
    for (W, q, s, z, A), Y in zip(mods, outs):
        solo = oracle.solo_forward(q, s, z, synth.bits(A), synth.bits(B), X)
        assert np.array_equal(Y, solo)          # bit-identical in the oracle


def test_correction_disabled_is_plain_w4a16():
    d, T = 256, 3
    W, q, s, z, A = _module(64, d, 8, 2, 0)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=2)
    Y = oracle.solo_forward(q, s, z, None, None, synth.bits(X))
    assert np.allclose(Y, X.astype(np.float64) @ _dense(q, s, z, d).T, rtol=1e-12, atol=1e-14)


def test_sampled_entries_equal_full_forward():
    d, r, T = 512, 32, 7
    W, q, s, z, A = _module(96, d, r, 3, 0)
    B = (synth.rng(3, synth.S_B).standard_normal((r, d)) * 0.01).astype(np.float16)
    X = synth.bits(synth.activations(T, d, synth.ALPHA_QKV, seed=3))
    Y = oracle.solo_forward(q, s, z, synth.bits(A), synth.bits(B), X)
    g = np.random.default_rng(0)
    ti, oi = g.integers(0, T, 50), g.integers(0, 96, 50)
    samp = oracle.module_forward_sampled(q, s, z, synth.bits(A), synth.bits(B), X, ti, oi)
    assert np.array_equal(samp, Y[ti, oi])


def test_zero_tokens():
    d = 128
    W, q, s, z, A = _module(16, d, 8, 4, 0)
    B = np.zeros((8, d), np.float16)
    Y = oracle.solo_forward(q, s, z, synth.bits(A), synth.bits(B), np.zeros((0, d), np.uint16))
    assert Y.shape == (0, 16)


def test_corrected_output_closer_to_full_precision_with_solved_factors():
    """With factors from the whitened solve, y moves toward W X (the method's purpose)."""
    d, r, T = 128, 32, 64
    mods = [_module(O, d, r, 5, i) for i, O in enumerate([128, 128, 128])]
    E = np.vstack([oracle.quant_error(W, q, s, z)[0] for (W, q, s, z, _) in mods])
    basis = synth.orthogonal_basis(d, seed=5)
    lam = synth.power_law_spectrum(d, synth.ALPHA_QKV)
    Sh, Shp = synth.covariance_half(basis, lam)
    Af, Bf, _ = oracle.group_solve(E, Sh, Shp, r, Omega=None)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=5, basis=basis)
    Xb = synth.bits(X)
    row = 0
    for (W, q, s, z, _) in mods:
        A_i = Af[row:row + W.shape[0]].astype(np.float16)
        row += W.shape[0]
        y_q = oracle.solo_forward(q, s, z, None, None, Xb)
        y_c = oracle.solo_forward(q, s, z, synth.bits(A_i), synth.bits(Bf.astype(np.float16)), Xb)
        y_fp = X.astype(np.float64) @ W.astype(np.float64).T
        assert np.linalg.norm(y_c - y_fp) < 0.8 * np.linalg.norm(y_q - y_fp)
