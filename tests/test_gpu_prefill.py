"""GPU parity of the large-T (prefill) corrected linear: tcgen05 kernels vs the oracle.

Shapes span several 128-row and 256-token tiles with ragged tails in both, the
r = 0 / disabled-module / multi-slab (r > 64) cases, and the full LLaMA-2-7B
MLP and LLaMA-3.1-8B prefill shapes checked on sampled outputs.
Pages: papernotes.org GlowQ summary, key design 4 and the set-up paragraph.
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

from helpers import TOL, attach_random_factors, make_modules, normwise, to_dev

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
        assert normwise(y, ref) < TOL


@pytest.mark.parametrize("r", [0, 128, 200, 256])
def test_prefill_rank_slabs(r):
    d, T = 384, 130
    mods = make_modules(d, [128, 128], seed=60 + r)
    B = attach_random_factors(mods, d, r, seed=60 + r) if r else None
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=60 + r)
    ys, _ = _run_group(mods, B, X)
    refs, _ = _oracle_group(mods, B, X)
    for y, ref in zip(ys, refs):
        assert normwise(y, ref) < TOL


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
    assert normwise(host[:, :128], refs[0]) < TOL
    assert normwise(host[:, 128:192], refs[1]) < TOL
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
    assert normwise(Y.astype(np.float64), ref) < TOL


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


def _sampled_check(mods, B, X, Ys, n=1500, seed=0):
    g = np.random.default_rng(seed)
    Xb, Bb = synth.bits(X), synth.bits(B)
    for m, Y in zip(mods, Ys):
        T, O = Y.shape
        ti, oi = g.integers(0, T, n), g.integers(0, O, n)
        ref = oracle.module_forward_sampled(m.q, m.s, m.z, synth.bits(m.A), Bb, Xb, ti, oi)
        got = Y[ti, oi].astype(np.float64)
        assert normwise(got, ref) < TOL


def test_llama2_7b_mlp_prefill_sampled():
    """gate/up 2 x 11008x4096 group + down_proj 4096x11008 solo, r=64, T=2048 (sampled outputs)."""
    import torch
    d, r, T = 4096, 64, 2048
    gu = make_modules(d, [11008, 11008], seed=0, sub0=30)
    Bg = attach_random_factors(gu, d, r, seed=0, sub=30)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=0)
    Ys, _ = glowq.group_forward(to_dev(gu), torch.from_numpy(Bg).cuda(), torch.from_numpy(X).cuda())
    _sampled_check(gu, Bg, X, [_np(Y) for Y in Ys])
    down = make_modules(11008, [4096], seed=0, sub0=40)
    Bd = attach_random_factors(down, 11008, r, seed=0, sub=40)
    Xd = synth.activations(T, 11008, synth.ALPHA_MLP, seed=0, sub=1)
    Yd = glowq.solo_forward(to_dev(down)[0], torch.from_numpy(Bd).cuda(), torch.from_numpy(Xd).cuda())
    _sampled_check(down, Bd, Xd, [_np(Yd)])


def test_llama31_8b_qkv_prefill_t4096_sampled():
    import torch
    d, r, T = 4096, 64, 4096
    qkv = make_modules(d, [4096, 1024, 1024], seed=1, sub0=50)
    B = attach_random_factors(qkv, d, r, seed=1, sub=50)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=1)
    Ys, _ = glowq.group_forward(to_dev(qkv), torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    _sampled_check(qkv, B, X, [_np(Y) for Y in Ys])


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
        assert normwise(y, ref) < TOL
