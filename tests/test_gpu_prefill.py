"""GPU parity of the large-T (prefill) corrected linear: tcgen05 kernels vs the oracle.

Shapes span several 128-row and 256-token tiles with ragged tails in both, the
r = 0 / disabled-module / multi-slab (r > 64) cases, and the full LLaMA-2-7B
MLP and LLaMA-3.1-8B prefill shapes checked on whole output tiles (every
element of four 256 x 256 tiles per module) and whole tokens.
Pages: papernotes.org GlowQ summary, key design 4 and the set-up paragraph.
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

from helpers import check, TOL, attach_random_factors, make_modules, normwise, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    glowq.lib()
    yield
    assert glowq.device_status() == 0


def _np(t):
    return t.detach().cpu().numpy()


def _run_group(mods, B, X):
    import torch
    Ys, R = glowq.group_forward(to_dev(mods), None if B is None else torch.from_numpy(B).cuda(),
                                torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    return [_np(Y).astype(np.float64) for Y in Ys], (None if R is None else _np(R).astype(np.float64))


def _oracle_group(mods, B, X):
    return oracle.group_forward([(m.q, m.s, m.z, None if m.A is None else synth.bits(m.A)) for m in mods],
                                None if B is None else synth.bits(B), synth.bits(X))


@pytest.mark.parametrize("T,r", [(17, 16), (100, 64), (256, 64), (300, 24), (513, 64)])
def test_prefill_group_ragged(T, r):
    d = 512
    mods = make_modules(d, [256, 48, 144], seed=50 + T)      # partial 128-row tiles
    B = attach_random_factors(mods, d, r, seed=50 + T)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=50 + T)
    ys, R = _run_group(mods, B, X)
    refs, R_ref = _oracle_group(mods, B, X)
    assert normwise(R, R_ref) < 1e-3
    for y, ref in zip(ys, refs):
        assert y.shape == ref.shape
        check(y, ref)


@pytest.mark.parametrize("r", [0, 128, 200, 256])
def test_prefill_rank_slabs(r):
    d, T = 384, 130
    mods = make_modules(d, [128, 128], seed=60 + r)
    B = attach_random_factors(mods, d, r, seed=60 + r) if r else None
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=60 + r)
    ys, _ = _run_group(mods, B, X)
    refs, _ = _oracle_group(mods, B, X)
    for y, ref in zip(ys, refs):
        check(y, ref)


def test_prefill_disabled_module_and_ldY_views():
    import torch
    d, r, T = 640, 64, 200
    outs = [128, 64]
    mods = make_modules(d, outs, seed=70)
    B = attach_random_factors(mods, d, r, seed=70)
    mods[1].A = None
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=70)
    buf = torch.full((T, sum(outs) + 8), float("nan"), dtype=torch.float16, device="cuda")
    views = [buf[:, :128], buf[:, 128:192]]
    glowq.group_forward(to_dev(mods), torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda(), Ys=views)
    host = _np(buf).astype(np.float64)
    refs, _ = _oracle_group(mods, B, X)
    check(host[:, :128], refs[0])
    check(host[:, 128:192], refs[1])
    assert np.all(np.isnan(host[:, 192:]))


def test_prefill_solo_wide_input():
    """down_proj-like solo module: d = 11008 (86 groups), O = 256, T = 300."""
    import torch
    d, r, T = 11008, 64, 300
    mods = make_modules(d, [256], seed=80)
    B = attach_random_factors(mods, d, r, seed=80)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=80)
    Y = _np(glowq.solo_forward(to_dev(mods)[0], torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda()))
    m = mods[0]
    ref = oracle.solo_forward(m.q, m.s, m.z, synth.bits(m.A), synth.bits(B), synth.bits(X))
    check(Y.astype(np.float64), ref)


def test_prefill_deterministic():
    import torch
    d, r, T = 1024, 64, 600
    mods = make_modules(d, [384, 128], seed=81)
    B = attach_random_factors(mods, d, r, seed=81)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=81)
    dm = to_dev(mods)
    Bt, Xt = torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda()
    a, Ra = glowq.group_forward(dm, Bt, Xt)
    b, Rb = glowq.group_forward(dm, Bt, Xt)
    assert torch.equal(Ra, Rb)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# Output tiles of the prefill kernel: 256 W rows x 256 tokens per CTA pair.
TILE_ROWS, TILE_TOKENS = 256, 256


def _tiles(O, T):
    """(rows, tokens) ranges of the first, the last and two interior output tiles."""
    nm, nn = -(-O // TILE_ROWS), -(-T // TILE_TOKENS)
    picks = [(0, 0), (nm - 1, nn - 1), (nm // 3, nn // 2), ((2 * nm) // 3, max(nn // 2 - 1, 0))]
    return [((bi * TILE_ROWS, min(O, (bi + 1) * TILE_ROWS)), (bj * TILE_TOKENS, min(T, (bj + 1) * TILE_TOKENS)))
            for bi, bj in picks]


def _tile_check(mods, B, X, Ys, whole_tokens=(0, -1)):
    """Every element of four whole output tiles per module (the first, the last
    and two interior ones) and every output feature of a few whole tokens,
    against the oracle evaluated on exactly those rows and tokens."""
    Xb, Bb = synth.bits(X), synth.bits(B)
    for m, Y in zip(mods, Ys):
        T, O = Y.shape
        Ab = synth.bits(m.A)
        pairs = []
        for (r0, r1), (t0, t1) in _tiles(O, T):
            Xt = Xb[t0:t1]
            R = oracle.anchor_project(Xt, Bb)
            ref = oracle.module_forward(m.q[r0:r1], m.s[r0:r1], m.z[r0:r1], Ab[r0:r1], R, Xt)
            pairs.append((Y[t0:t1, r0:r1], ref))
        for t in whole_tokens:
            t = t % T
            Xt = Xb[t:t + 1]
            ref = oracle.module_forward(m.q, m.s, m.z, Ab, oracle.anchor_project(Xt, Bb), Xt)
            pairs.append((Y[t:t + 1], ref))
        ymax = max(float(np.max(np.abs(ref))) for _, ref in pairs)
        for got, ref in pairs:
            check(got.astype(np.float64), ref, ymax)


def test_llama2_7b_mlp_prefill_tiles():
    """gate/up 2 x 11008x4096 group + down_proj 4096x11008 solo, r=64, T=2048 (whole tiles)."""
    import torch
    d, r, T = 4096, 64, 2048
    gu = make_modules(d, [11008, 11008], seed=0, sub0=30)
    Bg = attach_random_factors(gu, d, r, seed=0, sub=30)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=0)
    Ys, _ = glowq.group_forward(to_dev(gu), torch.from_numpy(Bg).cuda(), torch.from_numpy(X).cuda())
    _tile_check(gu, Bg, X, [_np(Y) for Y in Ys])
    down = make_modules(11008, [4096], seed=0, sub0=40)
    Bd = attach_random_factors(down, 11008, r, seed=0, sub=40)
    Xd = synth.activations(T, 11008, synth.ALPHA_MLP, seed=0, sub=1)
    Yd = glowq.solo_forward(to_dev(down)[0], torch.from_numpy(Bd).cuda(), torch.from_numpy(Xd).cuda())
    _tile_check(down, Bd, Xd, [_np(Yd)])


def test_llama31_8b_qkv_prefill_t4096_tiles():
    """GQA Q/K/V group 4096/1024/1024 x 4096, r=64, T=4096 (whole tiles)."""
    import torch
    d, r, T = 4096, 64, 4096
    qkv = make_modules(d, [4096, 1024, 1024], seed=1, sub0=50)
    B = attach_random_factors(qkv, d, r, seed=1, sub=50)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=1)
    Ys, _ = glowq.group_forward(to_dev(qkv), torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    _tile_check(qkv, B, X, [_np(Y) for Y in Ys])


def test_llama31_8b_mlp_prefill_t4096_tiles():
    """gate/up 2 x 14336x4096 group (shared B) and down_proj 4096x14336 solo, r=64,
    T=4096, alpha=0.77 (whole tiles)."""
    import torch
    d, ffn, r, T = 4096, 14336, 64, 4096
    gu = make_modules(d, [ffn, ffn], seed=1, sub0=60)
    Bg = attach_random_factors(gu, d, r, seed=1, sub=60)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=1, sub=2)
    Ys, _ = glowq.group_forward(to_dev(gu), torch.from_numpy(Bg).cuda(), torch.from_numpy(X).cuda())
    _tile_check(gu, Bg, X, [_np(Y) for Y in Ys])
    del Ys
    down = make_modules(ffn, [d], seed=1, sub0=70)
    Bd = attach_random_factors(down, ffn, r, seed=1, sub=70)
    Xd = synth.activations(T, ffn, synth.ALPHA_MLP, seed=1, sub=3)
    Yd = glowq.solo_forward(to_dev(down)[0], torch.from_numpy(Bd).cuda(), torch.from_numpy(Xd).cuda())
    _tile_check(down, Bd, Xd, [_np(Yd)])


def test_prefill_eight_modules_small_outputs():
    """Eight modules of 16..128 rows (the peer CTA of a 256-row pair tile holds
    no valid row), ragged T, r = 64."""
    d, r, T = 768, 64, 300
    mods = make_modules(d, [16, 32, 48, 64, 80, 96, 112, 128], seed=88)
    B = attach_random_factors(mods, d, r, seed=88)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=88)
    ys, R = _run_group(mods, B, X)
    refs, R_ref = _oracle_group(mods, B, X)
    assert normwise(R, R_ref) < 1e-3
    for y, ref in zip(ys, refs):
        assert y.shape == ref.shape
        check(y, ref)
