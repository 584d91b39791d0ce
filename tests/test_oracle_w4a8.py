"""Pins for the oracle's W4A8 path: per-token FP8 E4M3 activations consumed by
the whole corrected layer (the GlowQ pages report W4A8 next to W4A16, Tables
14-15 of the thelatestinai.com GlowQ page, without defining the activation
format; the per-token scale amax / 448 and round-to-nearest-even are readings
stated in the oracle).  Pins: the codes against PyTorch's float8_e4m3fn
conversion (a library routine), losslessness on the format's own grid (then
the W4A8 outputs equal the W4A16 oracle's), the rounding bound and
power-of-two equivariance.
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import synth

from helpers import attach_random_factors, make_modules, normwise


def test_activation_codes_against_torch():
    torch = pytest.importorskip("torch")
    X = synth.activations(9, 512, synth.ALPHA_QKV, seed=4)
    codes, scales = oracle.quantize_act_e4m3(synth.bits(X))
    xt = torch.from_numpy(X.astype(np.float32))
    st = xt.abs().amax(dim=1) / 448.0
    assert np.array_equal(st.numpy(), scales)
    want = (xt / st[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    diff = codes != want
    assert np.all((codes[diff] == 0) & (want[diff] == 0x80))       # only the sign of zero differs
    assert codes.max() <= 0xfe


def test_lossless_on_own_grid_equals_w4a16():
    g = np.random.default_rng(5)
    T, d, r = 5, 256, 16
    grid = np.array([oracle.e4m3_decode(c) for c in range(0x7f)])    # non-negative finite E4M3 values
    grid = grid[grid >= 2.0 ** -6]                                     # normal values: fp16-exact after scaling
    X = np.zeros((T, d), np.float64)
    for t in range(T):
        k = int(g.integers(-8, -2))
        row = g.choice(grid, d) * g.choice([-1.0, 1.0], d)
        row[int(g.integers(0, d))] = 448.0                             # the row max sets s = 2^k
        X[t] = row * 2.0 ** k
    Xb = oracle.f64_to_f16_bits(X)
    assert np.array_equal(oracle.f16_bits_to_f64(Xb), X)
    codes, scales = oracle.quantize_act_e4m3(Xb)
    assert np.array_equal(oracle.dequant_act_e4m3(codes, scales), X)
    mods = make_modules(d, [64, 32], seed=6)
    B = attach_random_factors(mods, d, r, seed=6)
    mt = [(m.q, m.s, m.z, synth.bits(m.A)) for m in mods]
    y8, R8, _ = oracle.w4a8_group_forward(mt, synth.bits(B), Xb)
    y16, R16 = oracle.group_forward(mt, synth.bits(B), Xb)
    assert np.allclose(R8, R16, rtol=1e-12, atol=1e-12)
    for a, b in zip(y8, y16):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_rounding_bound_and_equivariance():
    X = synth.activations(7, 384, synth.ALPHA_MLP, seed=8)
    codes, scales = oracle.quantize_act_e4m3(synth.bits(X))
    Xh = oracle.dequant_act_e4m3(codes, scales)
    x = X.astype(np.float64)
    s = scales.astype(np.float64)[:, None]
    normal = np.abs(x) >= s * 2.0 ** -6
    err = np.abs(Xh - x)
    assert np.all(err[normal] <= np.abs(x[normal]) * 2.0 ** -4 * (1 + 1e-6))   # half an ulp, 3 mantissa bits
    sub_bound = np.broadcast_to(s * 2.0 ** -10 * (1 + 1e-6), x.shape)       # half the subnormal step 2^-9
    assert np.all(err[~normal] <= sub_bound[~normal])
    c2, s2 = oracle.quantize_act_e4m3(synth.bits(X * np.float16(0.25)))
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales * np.float32(0.25))


def test_w4a8_output_close_to_w4a16():
    T, d, r = 4, 512, 32
    mods = make_modules(d, [128, 64], seed=9)
    B = attach_random_factors(mods, d, r, seed=9)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=9)
    mt = [(m.q, m.s, m.z, synth.bits(m.A)) for m in mods]
    y8, _, _ = oracle.w4a8_group_forward(mt, synth.bits(B), synth.bits(X))
    y16, _ = oracle.group_forward(mt, synth.bits(B), synth.bits(X))
    for a, b in zip(y8, y16):
        assert 0 < normwise(a, b) < 0.05                               # FP8 activations: a few percent
