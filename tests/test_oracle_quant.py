"""Pins for the oracle's fp16 conversions, INT4 g128 quantiser, packing and dequant.

Pages: papernotes.org GlowQ summary, experimental set-up paragraph (W4A16,
INT4 weights, group size 128).  Pins: exhaustive/library conversions, hand-worked
examples (tests/golden/int4_hand_examples.txt), brute-force nearest-code search,
lossless quantisation of values on the quantiser's own grid, exact zero.
"""
import os

import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "int4_hand_examples.txt")


# ---------------------------------------------------------------- fp16 ----

def test_f16_to_f64_exhaustive_matches_numpy():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_bits_to_f64(allbits)
    ref = allbits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zero preserved
    assert np.signbit(ours[0x8000]) and not np.signbit(ours[0])


def test_f64_to_f16_matches_numpy_rounding():
    g = np.random.default_rng(1)
    vals = [g.standard_normal(4000) * 10.0 ** g.integers(-9, 6, 4000)]
    # exact midpoints between adjacent fp16 values (ties-to-even cases)
    h = np.arange(0, 0x7BFF, 7, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    vals.append((lo + hi) / 2)
    vals.append(-(lo + hi) / 2)
    vals.append(np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e30, -1e30,
                          2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -14,
                          2.0 ** -14 - 2.0 ** -25, np.inf, -np.inf]))
    v = np.concatenate(vals)
    ours = oracle.f64_to_f16_bits(v)
    ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    assert oracle.f64_to_f16_bits(np.array([np.nan]))[0] & 0x7C00 == 0x7C00


def test_f32_to_f16_matches_numpy():
    g = np.random.default_rng(2)
    v = (g.standard_normal(3000) * 10.0 ** g.integers(-8, 5, 3000)).astype(np.float32)
    assert np.array_equal(oracle.f32_to_f16_bits(v), v.astype(np.float16).view(np.uint16))


# ---------------------------------------------------------- quantiser ----

def _golden_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, lead, sb, z, w0, wr, wh = line.split()
        rows.append((name, [float(x) for x in lead.split(",")], int(sb, 16), int(z),
                     int(w0, 16), int(wr, 16), [float(x) for x in wh.split(",")]))
    return rows


@pytest.mark.parametrize("case", _golden_rows(), ids=lambda c: c[0])
def test_hand_worked_examples(case):
    name, lead, sbits, zero, word0, word_rest, what = case
    W = np.zeros((1, 128), np.float32)
    W[0, :len(lead)] = lead
    q, s, z = oracle.quantize_int4(W)
    assert s[0, 0] == sbits
    assert z[0, 0] == zero
    assert q[0, 0] == word0
    assert np.all(q[0, 1:] == word_rest)
    deq = oracle.dequant_int4(q, s, z, 128).view(np.float16).astype(np.float64)
    assert np.array_equal(deq[0, :len(what)], np.array(what))
    assert np.all(deq[0, len(what):] == 0.0)


def _grid_group(g, s0, z0):
    """128 values that lie exactly on the grid (k - z0) * s0, k = 0..15, every code used."""
    codes = np.concatenate([np.arange(16), g.integers(0, 16, 112)])
    g.shuffle(codes)
    return ((codes - z0) * np.float64(s0)).astype(np.float32), codes


def test_lossless_on_own_grid():
    """Values on the quantiser's own grid (range spanning all 16 codes) come back exactly."""
    g = np.random.default_rng(3)
    O, d = 6, 512
    W = np.zeros((O, d), np.float32)
    want_codes = np.zeros((O, d), np.int64)
    want_s = np.zeros((O, d // 128), np.uint16)
    want_z = np.zeros((O, d // 128), np.int64)
    s_choices = np.array([2.0 ** -7, 0.01171875, 0.0013427734375, 0.25, 3.0, 2.0 ** -12], np.float16)
    for o in range(O):
        for j in range(d // 128):
            s0 = s_choices[(o + j) % len(s_choices)]
            z0 = int(g.integers(0, 16))
            vals, codes = _grid_group(g, s0, z0)
            W[o, j * 128:(j + 1) * 128] = vals
            want_codes[o, j * 128:(j + 1) * 128] = codes
            want_s[o, j] = s0.view(np.uint16)
            want_z[o, j] = z0
    q, s, z = oracle.quantize_int4(W)
    assert np.array_equal(s, want_s)
    assert np.array_equal(z.astype(np.int64), want_z)
    assert np.array_equal(oracle.unpack_int4(q, d).astype(np.int64), want_codes)
    deq = oracle.dequant_int4(q, s, z, d).view(np.float16).astype(np.float32)
    assert np.array_equal(deq, W)


def test_packing_layout_low_nibble_first():
    """Code k of a row sits in nibble k%8 of word k/8 (lowest nibble = lowest k)."""
    codes = (np.arange(2 * 256) * 7 % 16).reshape(2, 256).astype(np.uint32)
    words = np.zeros((2, 32), np.uint32)
    for k in range(256):
        words[:, k // 8] |= codes[:, k] << np.uint32(4 * (k % 8))
    assert np.array_equal(oracle.unpack_int4(words, 256), codes.astype(np.uint8))


def test_codes_are_nearest_grid_point():
    """Brute force over all 16 codes: q minimises |w/s - (q - z)| (ties excluded)."""
    W = synth.weights(16, 1024, seed=5, outlier_cols=4)
    q, s, z = oracle.quantize_int4(W)
    codes = oracle.unpack_int4(q, 1024).astype(np.float64)
    sf = s.view(np.float16).astype(np.float32)
    for o in range(16):
        for j in range(8):
            w = W[o, j * 128:(j + 1) * 128].astype(np.float32)
            t = (w / sf[o, j]).astype(np.float64)           # fp32 division, as defined
            grid = np.arange(16)[None, :] - float(z[o, j])
            dist = np.abs(t[:, None] - grid)
            best = np.argmin(dist, axis=1)
            srt = np.sort(dist, axis=1)
            clear = (srt[:, 1] - srt[:, 0]) > 1e-6
            assert np.array_equal(codes[o, j * 128:(j + 1) * 128][clear], best[clear])


def test_zero_maps_to_zero_and_error_bound():
    W = synth.weights(32, 768, seed=7)
    W[:, ::37] = 0.0
    q, s, z = oracle.quantize_int4(W)
    deq = oracle.dequant_int4(q, s, z, 768).view(np.float16).astype(np.float64)
    assert np.all(deq[:, ::37] == 0.0)
    sf = np.repeat(s.view(np.float16).astype(np.float64), 128, axis=1)
    err = np.abs(deq - W.astype(np.float64))
    # every weight within one step; the vast majority within half a step (+fp16 rounding)
    assert np.all(err <= sf * 1.0 + 1e-3 * sf)
    half = err <= 0.5 * sf + np.abs(deq) * 2.0 ** -11 + 1e-12
    assert half.mean() > 0.99


def test_degenerate_groups():
    W = np.zeros((3, 256), np.float32)
    W[1, :128] = 1e-30           # below fp16 range: s underflows -> 1.0
    W[2, :128] = -2.5            # all negative, constant
    q, s, z = oracle.quantize_int4(W)
    assert s[0, 0] == 0x3C00 and z[0, 0] == 0 and np.all(q[0] == 0)
    assert s[1, 0] == 0x3C00
    deq = oracle.dequant_int4(q, s, z, 256).view(np.float16).astype(np.float64)
    assert np.all(deq[0] == 0)
    # constant -2.5 group: mn=-2.5, mx=0, s=fp16(2.5/15), code 0 -> -z*s
    s2 = float(s[2, 0:1].view(np.float16)[0])
    assert z[2, 0] == 15
    assert abs(deq[2, 0] + 2.5) <= s2 / 2 + 1e-3


def test_scaling_by_power_of_two_is_equivariant():
    W = synth.weights(8, 512, seed=9)
    q1, s1, z1 = oracle.quantize_int4(W)
    q2, s2, z2 = oracle.quantize_int4(W * np.float32(4.0))
    assert np.array_equal(q1, q2) and np.array_equal(z1, z2)
    assert np.array_equal(s2.view(np.float16).astype(np.float64), 4 * s1.view(np.float16).astype(np.float64))


def test_dequant_exhaustive_codes_zeros_scales():
    """All 16 codes x 16 zeros x a grid of fp16 scales vs numpy's float64->float16 rounding."""
    g = np.random.default_rng(11)
    scales = np.concatenate([g.integers(0x0001, 0x7BFF, 200), [0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF]])
    rows = len(scales)
    d = 256                                   # two groups per row; each group covers all (q, z)
    codes = np.tile(np.arange(16), 16)        # 256 entries: q = k % 16
    q = np.zeros((rows, d // 8), np.uint32)
    for k in range(d):
        q[:, k // 8] |= np.uint32(codes[k]) << np.uint32(4 * (k % 8))
    s = np.stack([scales, scales[::-1]], axis=1).astype(np.uint16)
    z = np.zeros((rows, 2), np.uint8)
    outs = []
    for zz in range(16):
        z[:] = zz
        deq = oracle.dequant_int4(q, s, z, d)
        sf = np.repeat(s.view(np.float16).astype(np.float64), 128, axis=1)
        ref = ((codes[None, :] - zz) * sf).astype(np.float16).view(np.uint16)
        outs.append(np.array_equal(deq, ref))
    assert all(outs)
