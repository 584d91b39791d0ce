"""The C ABI library builds, loads and exports every entry point glowq.h declares.

No GPU needed: only host-side calls run here (argument validation that returns
before anything is enqueued, the workspace-size query, and the host-only
GlowQ-S ranking, checked against the oracle).
"""
import ctypes as C
import subprocess

import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq


@pytest.fixture(scope="module")
def L():
    build.build()
    return glowq.lib()


def test_exports_every_declared_symbol(L):
    declared = glowq.declared_symbols()
    assert len(declared) >= 10
    out = subprocess.check_output(["nm", "-D", "--defined-only", glowq.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    assert all(s.startswith("glowq_") for s in exported)   # nothing else leaks out
    for s in declared:
        getattr(L, s)


def test_version_and_status_strings(L):
    assert glowq.version().count(".") == 2
    for code in range(7):
        assert L.glowq_status_string(code)


def test_workspace_bytes(L):
    assert glowq.workspace_bytes(0, 64) == 0
    assert glowq.workspace_bytes(16, 0) == 0
    small = glowq.workspace_bytes(16, 64)
    # zero region (hand-off flags, k-split tickets) + up to 16 d-slices of fp32
    # partial sums of R + solo R
    assert small == 4096 + 16 * 16 * 64 * 4 + 16 * 64 * 2
    assert glowq.workspace_bytes(1, 64) == 4096 + 16 * 64 * 4 + 256    # solo R rounded up to 256 B
    big = glowq.workspace_bytes(2048, 64)
    assert big >= 4096 + 8 * 2048 * 64 * 4 + 2048 * 64 * 2  # zero region + split-d fp32 partials of R + solo R
    assert small % 256 == 0 and big % 256 == 0


def test_workspace_bytes_for_the_k_split(L):
    """Sizing of the small-batch k-split (host arithmetic only): slots of
    2 x 128 rows x 64 tokens fp32 behind the other regions, S parts per tile."""
    slot = 2 * 128 * 64 * 4
    # no split outside 16 < T <= 64, or for bad arguments
    for T in (1, 16, 65, 2048):
        assert glowq.workspace_bytes_for(T, 64, 4096, [4096]) == glowq.workspace_bytes(T, 64)
    assert glowq.workspace_bytes_for(40, 64, 200, [4096]) == glowq.workspace_bytes(40, 64)
    assert glowq.workspace_bytes_for(40, 64, 4096, []) == glowq.workspace_bytes(40, 64)
    assert glowq.workspace_bytes_for(40, 64, 1 << 21, [4096]) == glowq.workspace_bytes(40, 64)   # d > 2^20
    assert glowq.workspace_bytes_for(40, 64, 4096, [0]) == glowq.workspace_bytes(40, 64)
    # LLaMA-2-13B down_proj at T = 64: 20 tiles of 256 rows, far fewer than the CTA pairs
    for T, r, d, outs in [(64, 64, 13824, [5120]), (17, 64, 4096, [1024]), (40, 32, 4096, [512, 256]),
                          (48, 0, 8192, [512])]:
        n = glowq.workspace_bytes_for(T, r, d, outs)
        base = (glowq.workspace_bytes(T, r) if r else 4096)
        assert n > base and (n - base) % slot == 0, (T, r, d, outs)
        tiles = sum(-(-o // 256) for o in outs)
        parts, rem = divmod((n - base) // slot, tiles)
        assert rem == 0 and 2 <= parts <= 8, (T, d, outs, parts)
        # every part holds at least 8 k-blocks of 64 (4 groups of 128)
        assert -(-(d // 64) // parts) >= 8
    # enough tiles to fill the GPU: whole tiles
    assert glowq.workspace_bytes_for(64, 64, 4096, [4096] * 8) == glowq.workspace_bytes(64, 64)


def _parts(T, r, d, outs):
    """Parts per tile the k-split planner picks (1: whole tiles)."""
    n, base = glowq.workspace_bytes_for(T, r, d, outs), glowq.workspace_bytes(T, r)
    if n <= base:
        return 1
    return (n - base) // (2 * 128 * 64 * 4) // sum(-(-o // 256) for o in outs)


@pytest.mark.parametrize("outs,d,S", [
    ([4096] * 3, 4096, 1),        # LLaMA-2-7B Q/K/V: 48 tiles, whole tiles measured fastest
    ([4096], 4096, 4),            # o_proj 4096 x 4096: 16 tiles
    ([11008] * 2, 4096, 2),       # LLaMA-2-7B gate/up: 86 tiles
    ([4096], 11008, 4),           # LLaMA-2-7B down_proj
    ([14336] * 2, 4096, 1),       # LLaMA-3.1-8B gate/up: 112 tiles
    ([4096], 14336, 4),           # LLaMA-3.1-8B down_proj
    ([5120] * 3, 5120, 1),        # LLaMA-2-13B Q/K/V: 60 tiles
    ([5120], 5120, 3),            # LLaMA-2-13B o_proj: 20 tiles
    ([13824] * 2, 5120, 2),       # LLaMA-2-13B gate/up: 108 tiles
    ([5120], 13824, 3),           # LLaMA-2-13B down_proj
])
def test_split_planner_matches_the_measured_choice(L, outs, d, S):
    """The planner's part count for the LLaMA units at T = 32 and 64 (148 SMs,
    74 CTA pairs) equals the one a sweep of S = 1..8 on a B200 measured
    fastest for each unit (host arithmetic only).  The one unit of that sweep
    left out, the LLaMA-3.1-8B Q/K/V group, gets 3 parts where 2 measured
    6 % faster."""
    for T in (32, 64):
        assert _parts(T, 64, d, outs) == S, (outs, d, T)


def _mods(n, O=128, q=0x1000, Y=0x2000, ldY=128, A=0x3000):
    arr = (glowq._Module * n)()
    for i in range(n):
        arr[i].qweight, arr[i].scales, arr[i].zeros = q, q + 0x100, q + 0x200
        arr[i].A, arr[i].out_features, arr[i].Y, arr[i].ldY = A, O, Y, ldY
    return arr


def _gf(L, mods, m=1, d=256, B=0x4000, r=16, X=0x5000, T=4, R=0x6000, ws=0x7000, wsb=1 << 20):
    return L.glowq_group_forward(mods, m, d, B, r, X, T, R, ws, wsb, None)


def test_host_validation_errors(L):
    # Each call is rejected on the host before any CUDA work (fake addresses).
    assert _gf(L, _mods(1), d=200) == 2                 # d % 128
    assert _gf(L, _mods(1), r=12) == 2                  # r % 8
    assert _gf(L, _mods(1), r=512) == 2                 # r > 256
    assert _gf(L, _mods(1, O=100)) == 2                 # out_features % 16
    assert _gf(L, _mods(1), m=0) == 1
    assert _gf(L, _mods(9), m=9) == 1                   # more than 8 modules
    assert _gf(L, _mods(1), X=0x5001) == 3              # misaligned X
    assert _gf(L, _mods(1, ldY=100)) == 3               # ldY < out_features
    assert _gf(L, _mods(1, ldY=132)) == 3               # ldY % 8
    assert _gf(L, _mods(1), B=None) == 1                # r > 0 needs B
    assert _gf(L, _mods(1), R=None) == 1                # ... and R_out
    assert _gf(L, _mods(1), T=64, wsb=16) == 1          # workspace too small (T > 16 splits R)
    assert _gf(L, _mods(1), T=4, ws=None, wsb=0) == 1   # decode with r > 0 needs the hand-off flags
    assert _gf(L, _mods(1), T=4, wsb=128) == 1          # ... the whole zero region
    assert _gf(L, _mods(1), T=4, ws=0x7008) == 3        # misaligned workspace
    assert _gf(L, _mods(1), T=-1) == 1
    assert _gf(L, _mods(1), T=0) == 0                   # empty batch: no-op
    assert L.glowq_solo_forward(_mods(1), 256, 0x4000, 16, 0x5000, 4, None, 0, None) == 1
    assert L.glowq_pack_int4(0x1000, 16, 256, 64, 0x2000, 0x3000, 0x4000, None) == 6
    assert L.glowq_pack_int4(0x1000, 16, 200, 128, 0x2000, 0x3000, 0x4000, None) == 2
    assert L.glowq_pack_int4(0x1000, 0, 256, 128, 0x2000, 0x3000, 0x4000, None) == 0
    # the codes are stored in 16-row blocks: row counts must be multiples of 16
    assert L.glowq_pack_int4(0x1000, 8, 256, 128, 0x2000, 0x3000, 0x4000, None) == 2
    assert L.glowq_dequant_int4(0x1000, 0x2000, 0x3000, 24, 256, 128, 0x4000, None) == 2
    assert L.glowq_dequant_int4(0x1000, 0x2000, 0x3000, 16, 256, 128, 0x4008, None) == 3


def test_select_restore_matches_oracle(L):
    g = np.random.default_rng(0)
    for trial in range(40):
        n = int(g.integers(1, 60))
        e = np.round(g.random(n) * 4, 1 if trial % 2 else 6)
        w = np.round(g.random(n) * 4 + 0.1, 1 if trial % 2 else 6)
        if trial % 7 == 3:
            e = w * 0.25                                 # flat scores -> layer order
        layer = g.integers(0, 12, n)
        kind = g.integers(0, 4, n)
        k = int(g.integers(0, n + 1))
        m1, o1, f1 = glowq.select_restore(e, w, layer, kind, k)
        m2, o2, _, f2 = oracle.select_restore(e, w, layer, kind, k)
        assert f1 == f2
        assert np.array_equal(o1, o2) and np.array_equal(m1, m2)


def test_select_restore_rejects_bad_k(L):
    with pytest.raises(glowq.GlowQError):
        glowq.select_restore([1.0], [1.0], [0], [0], 2)


def test_select_restore_scores_matches_oracle(L):
    """Host-only ranking by a caller-computed score (e.g. g_ec) against the oracle."""
    g = np.random.default_rng(5)
    for trial in range(40):
        n = int(g.integers(1, 60))
        sc = np.round(g.random(n) * 4, 1 if trial % 2 else 6)
        if trial % 7 == 3:
            sc = np.full(n, 0.25)                                # flat scores -> layer order
        if trial % 11 == 5:
            sc[int(g.integers(0, n))] = np.nan                   # NaN -> layer order
        layer = g.integers(0, 12, n)
        kind = g.integers(0, 4, n)
        k = int(g.integers(0, n + 1))
        m_g, o_g, fb_g = glowq.select_restore_scores(sc, layer, kind, k)
        m_o, o_o, fb_o = oracle.select_by_score(sc, layer, kind, k)
        assert fb_g == fb_o
        assert np.array_equal(m_g, m_o) and np.array_equal(o_g, o_o)
    # argument errors are reported before anything is written
    assert L.glowq_select_restore_scores(None, None, None, 3, 1, None, None, None) == 1
    assert L.glowq_select_restore_scores(None, None, None, 0, 0, None, None, None) == 0
    x = np.zeros(2)
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    assert L.glowq_select_restore_scores(p(x), p(np.zeros(2, np.int32)), p(np.zeros(2, np.int32)), 2, 3,
                                         p(np.zeros(2, np.uint8)), None, None) == 1     # k > n
