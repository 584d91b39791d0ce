"""Pins for the oracle's narrow floating-point base-weight formats (MXFP4,
NVFP4), the alternative datatypes of the GlowQ pages' Table 13
(thelatestinai.com GlowQ page).  The pages give only perplexities; the formats
follow their public definitions (E2M1 elements, E8M0 or E4M3 block scales),
each choice a reading stated in the oracle.  Pins: the scale encodings against
PyTorch's float8 conversions (a library routine), E2M1 rounding against a
brute-force nearest search, losslessness on the formats' own grids, error
bounds, power-of-two equivariance and the packing order.
"""
import numpy as np
import pytest

import oracle


def _e2m1_magnitudes():
    return np.array([oracle.e2m1_decode(c) for c in range(8)])


def test_e2m1_decode_structure():
    mags = _e2m1_magnitudes()
    assert mags[0] == 0.0 and np.all(np.diff(mags) > 0)            # codes 0..7 increasing
    assert mags[1] == 0.5 and mags[-1] == 6.0
    for c in range(8):                                               # sign bit negates
        assert oracle.e2m1_decode(c | 8) == -mags[c]
    for e in range(0, 3):                                            # two values per binade (1 mantissa bit)
        inb = [m for m in mags if 2.0 ** e <= m < 2.0 ** (e + 1)]
        assert len(inb) == 2 and inb[1] / inb[0] == 1.5


def test_e2m1_encode_is_nearest_with_ties_to_even_and_saturation():
    mags = _e2m1_magnitudes()
    vals = np.arange(-0x7bff, 0x7bff, dtype=np.int32)                 # every finite fp16 magnitude pattern
    vals = vals[np.abs(vals) <= 0x4c00]                               # |v| <= 16
    v16 = np.where(vals >= 0, vals, 0x8000 - vals).astype(np.uint16).view(np.float16).astype(np.float32)
    for v in v16[::7]:
        a = abs(float(v))
        d = np.abs(mags - min(a, 6.0))
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        if want == 0 or v == 0:
            assert oracle.e2m1_encode(v) == 0, v
        else:
            assert oracle.e2m1_encode(v) == (int(want) | (8 if v < 0 else 0)), v


def test_e4m3_against_torch():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    ours = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))
    # encode: every finite fp16 value with |v| <= 448, round to nearest even
    bits = np.arange(0, 0x7c00, dtype=np.uint16)
    pos = bits.view(np.float16).astype(np.float32)
    v = np.concatenate([pos, -pos])
    v = v[np.abs(v) <= 448.0]
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(x)) for x in v], dtype=np.uint8)
    # values that round to zero encode as +0 here; torch keeps the sign (-0 = 0x80)
    diff = got != want
    assert np.all((got[diff] == 0) & (want[diff] == 0x80)), v[diff][:5]
    assert diff.sum() < v.size // 4
    # overflow saturates to +-448 (a reading)
    assert oracle.e4m3_encode(1e6) == 0x7e and oracle.e4m3_encode(-500.0) == 0xfe


def test_e8m0_against_torch():
    torch = pytest.importorskip("torch")
    codes = np.arange(255, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).float().numpy().astype(np.float64)
    ours = np.array([oracle.e8m0_decode(int(c)) for c in codes])
    finite = ref > 0                                                   # float32 loses the smallest powers
    assert np.all(ours[finite] == ref[finite])
    assert ours[0] == 2.0 ** -127 and ours[254] == 2.0 ** 127


def _f16(bits):
    return bits.view(np.float16).astype(np.float64)


def test_mxfp4_lossless_on_its_own_grid():
    g = np.random.default_rng(0)
    mags = _e2m1_magnitudes()
    O, d = 6, 128
    W = np.zeros((O, d), np.float32)
    for o in range(O):
        for b in range(d // 32):
            k = int(g.integers(-10, 4))
            blk = g.choice(mags, 32) * g.choice([-1.0, 1.0], 32)
            blk[int(g.integers(0, 32))] = g.choice([4.0, 6.0])          # the block max sets X = 2^k
            W[o, 32 * b:32 * b + 32] = blk * 2.0 ** k
    codes, scales = oracle.quantize_mxfp4(W)
    assert np.array_equal(_f16(oracle.dequant_mxfp4(codes, scales, d)), W.astype(np.float64))


def test_mxfp4_error_bound_equivariance_and_layout():
    g = np.random.default_rng(1)
    O, d = 8, 256
    W = (g.standard_normal((O, d)) * 0.02).astype(np.float32)
    codes, scales = oracle.quantize_mxfp4(W)
    wh = _f16(oracle.dequant_mxfp4(codes, scales, d))
    X = np.repeat(2.0 ** (scales.astype(np.float64) - 127), 32, axis=1)
    a = np.abs(W.astype(np.float64))
    inside = a <= 6 * X
    assert np.all(np.abs(wh - W)[inside] <= X[inside] * (1 + 2 ** -10))        # half the largest gap (1) x X
    assert np.all(np.abs(wh - W)[~inside] < 2 * X[~inside])                     # [6X, 8X) saturates to 6X
    # power-of-two equivariance: codes unchanged, scales shifted
    c2, s2 = oracle.quantize_mxfp4(W * np.float32(2.0 ** -3))
    assert np.array_equal(c2, codes) and np.array_equal(s2.astype(int), scales.astype(int) - 3)
    # packing: even k in the low nibble
    for k in (0, 1, 2, 3, 37):
        c = (codes[:, k // 2] >> (4 * (k % 2))) & 0xF
        want = np.array([oracle.e2m1_encode(float(W[o, k] / X[o, k])) for o in range(O)])
        assert np.array_equal(c, want)
    # an all-zero block: code 0 everywhere, the smallest scale
    Wz = W.copy()
    Wz[:, :32] = 0.0
    cz, sz = oracle.quantize_mxfp4(Wz)
    assert np.all(cz[:, :16] == 0) and np.all(sz[:, 0] == 0)


def test_nvfp4_scales_error_bound_and_zero_tensor():
    g = np.random.default_rng(2)
    O, d = 8, 256
    W = (g.standard_normal((O, d)) * 0.02).astype(np.float32)
    W[3, 17] = 0.3                                                      # one outlier sets the tensor scale
    codes, scales, st = oracle.quantize_nvfp4(W)
    assert st == pytest.approx(float(np.float32(0.3) / np.float32(6.0 * 448.0)), rel=0)
    dec = np.array([[oracle.e4m3_decode(int(c)) for c in row] for row in scales])
    full = np.repeat(dec * st, 16, axis=1)
    wh = _f16(oracle.dequant_nvfp4(codes, scales, st, d))
    err = np.abs(wh - W.astype(np.float64))
    # half the largest element gap (1.0) or the saturation of a rounded-down scale (< 0.4), times the block
    # scale, plus the final fp16 rounding
    assert np.all(err <= full * 1.0 + np.abs(wh) * 2 ** -11 + 1e-30)
    # block scales: the largest block (the outlier's) maps to exactly 448 (6 * s_t * 448 = 0.3)
    assert scales[3, 1] == 0x7e
    cz, sz, stz = oracle.quantize_nvfp4(np.zeros((2, 32), np.float32))
    assert stz == 1.0 and np.all(cz == 0) and np.all(sz == 0)


def _grid_weights(O, d, seed):
    """Weights on the MXFP4 grid: every 32-block is E2M1 magnitudes times 2^k with
    a 4 or 6 in it, so the block scale is 2^k and dequantisation is lossless."""
    g = np.random.default_rng(seed)
    mags = _e2m1_magnitudes()
    W = np.zeros((O, d), np.float32)
    for o in range(O):
        for b in range(d // 32):
            k = int(g.integers(-9, -3))
            blk = g.choice(mags, 32) * g.choice([-1.0, 1.0], 32)
            blk[int(g.integers(0, 32))] = g.choice([4.0, 6.0])
            W[o, 32 * b:32 * b + 32] = blk * 2.0 ** k
    return W


def test_fp4_group_forward_is_the_definition():
    """On the MXFP4 grid w_hat == W exactly, so the forward must equal X W^T + R A^T
    computed directly from W (numpy float64, other association order), and the
    shared R must equal each module's own projection."""
    g = np.random.default_rng(5)
    d, T, r = 256, 3, 8
    Ws = [_grid_weights(O, d, 10 + i) for i, O in enumerate((64, 32))]
    X = (g.standard_normal((T, d)) * 0.5).astype(np.float16)
    B = (g.standard_normal((r, d)) * 0.05).astype(np.float16)
    As = [(g.standard_normal((W.shape[0], r)) * 0.05).astype(np.float16) for W in Ws]
    mods = []
    for W, A in zip(Ws, As):
        codes, scales = oracle.quantize_mxfp4(W)
        mods.append((codes, scales, None, A.view(np.uint16)))
    outs, R = oracle.fp4_group_forward("mx", mods, B.view(np.uint16), X.view(np.uint16))
    Xd, Bd = X.astype(np.float64), B.astype(np.float64)
    Rn = (Bd @ Xd.T).T
    assert np.allclose(R, Rn, rtol=1e-13, atol=1e-15)
    for W, A, Y in zip(Ws, As, outs):
        want = (W.astype(np.float64) @ Xd.T).T + (A.astype(np.float64) @ Rn.T).T
        assert np.allclose(Y, want, rtol=1e-12, atol=1e-14)
    # NVFP4: the forward uses the NVFP4 dequantised weight (a different w_hat)
    mods_nv = []
    for W, A in zip(Ws, As):
        codes, scales, st = oracle.quantize_nvfp4(W)
        mods_nv.append((codes, scales, st, A.view(np.uint16)))
    outs_nv, _ = oracle.fp4_group_forward("nv", mods_nv, B.view(np.uint16), X.view(np.uint16))
    for (codes, scales, st, A), Y in zip(mods_nv, outs_nv):
        Wh = _f16(oracle.dequant_nvfp4(codes, scales, st, d))
        want = (Wh @ Xd.T).T + (A.view(np.float16).astype(np.float64) @ Rn.T).T
        assert np.allclose(Y, want, rtol=1e-12, atol=1e-14)
