"""GPU parity of small batches (16 < T <= 64): the tcgen05 kernel on 64-token
pair tiles, with each tile's d range split across CTA pairs (fp32 partial sums
added in a fixed order by the part that counts last on the tile's ticket).

Shapes: an o_proj-like module whose 256-row tiles are far fewer than the CTA
pairs (the case the split exists for), a ragged Q/K/V-like group (partial
128-row tiles, 48- and 144-wide modules), plain W4A16 (r = 0), MXFP4 / NVFP4
base weights, and the LLaMA-2-13B o_proj / down_proj at decode batches 32 and
64 (d = 13824, every output element).  Every result is checked against the
oracle; split and whole-tile runs both pass the same bar, the split's result is
bit-identical across calls, and every call leaves the workspace's zero region
zero.  Pages: papernotes.org GlowQ summary, key design 4 and the set-up
paragraph (W4A16, g128, rank 64); decode batches of the 13B stack: the
thelatestinai.com GlowQ page, Table 3.
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

from helpers import attach_random_factors, check, make_modules, normwise, to_dev

pytestmark = pytest.mark.gpu

ZERO_REGION = 4096


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


def _splits(T, r, d, outs):
    """The call of this shape takes the k-split (its sizing adds slots)."""
    return glowq.workspace_bytes_for(T, r, d, outs) > glowq.workspace_bytes(T, r)


def _oracle_group(mods, B, X):
    return oracle.group_forward([(m.q, m.s, m.z, None if m.A is None else synth.bits(m.A)) for m in mods],
                                None if B is None else synth.bits(B), synth.bits(X))


def _group(mods, B, X, ws):
    import torch
    Ys, R = glowq.group_forward(mods, None if B is None else torch.from_numpy(B).cuda(),
                                torch.from_numpy(X).cuda(), workspace=ws)
    torch.cuda.synchronize()
    return Ys, R


@pytest.mark.parametrize("T,d,outs,r", [
    (17, 4096, [1024], 64),            # 4 tiles of 256 rows: split up to 8 ways
    (40, 4096, [1024], 64),
    (64, 4096, [1024], 64),
    (33, 2048, [256, 48, 144], 16),    # ragged rows in a group
    (48, 8192, [512], 0),              # plain W4A16, no correction
])
def test_split_matches_oracle(T, d, outs, r):
    import torch
    assert _splits(T, r, d, outs), "the shape is meant to take the k-split"
    mods = make_modules(d, outs, seed=900 + T)
    B = attach_random_factors(mods, d, r, seed=900 + T) if r else None
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=900 + T)
    ws = glowq.alloc_workspace(T, r, "cuda", d, outs)
    dm = to_dev(mods)
    Ys, R = _group(dm, B, X, ws)
    refs, R_ref = _oracle_group(mods, B, X)
    if r:
        assert normwise(_np(R).astype(np.float64), R_ref) < 1e-3
    for Y, ref in zip(Ys, refs):
        check(_np(Y).astype(np.float64), ref)
    assert int(ws[:ZERO_REGION].count_nonzero()) == 0, "tickets or flags left non-zero"
    # the sum order is fixed: a second call gives the same bits
    Ys2, _ = _group(dm, B, X, ws)
    for a, b in zip(Ys, Ys2):
        assert torch.equal(a, b)
    assert int(ws[:ZERO_REGION].count_nonzero()) == 0


def test_whole_tiles_when_the_workspace_has_no_room():
    """With only glowq_workspace_bytes(T, r) the call runs whole tiles; both
    decompositions meet the oracle bar."""
    T, d, outs, r = 40, 4096, [1024], 64
    mods = make_modules(d, outs, seed=940)
    B = attach_random_factors(mods, d, r, seed=940)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=940)
    refs, _ = _oracle_group(mods, B, X)
    dm = to_dev(mods)
    small = glowq.alloc_workspace(T, r, "cuda")
    big = glowq.alloc_workspace(T, r, "cuda", d, outs)
    assert big.numel() > small.numel()
    for ws in (small, big):
        Ys, _ = _group(dm, B, X, ws)
        check(_np(Ys[0]).astype(np.float64), refs[0])
        assert int(ws[:ZERO_REGION].count_nonzero()) == 0


def test_workspace_shared_across_decode_small_and_prefill_calls():
    """One workspace (sized for the largest use) across T = 1, 40, 300, 64 calls
    in order on one stream: every result matches the oracle and the zero
    region is zero after each call."""
    import torch
    d, outs, r = 2048, [512], 32
    mods = make_modules(d, outs, seed=950)
    B = attach_random_factors(mods, d, r, seed=950)
    dm = to_dev(mods)
    n = max(glowq.workspace_bytes_for(T, r, d, outs) for T in (1, 40, 64, 300))
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    for T in (1, 40, 300, 64):
        X = synth.activations(T, d, synth.ALPHA_MLP, seed=950 + T)
        Y = glowq.solo_forward(dm[0], torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda(), workspace=ws)
        torch.cuda.synchronize()
        m = mods[0]
        ref = oracle.solo_forward(m.q, m.s, m.z, synth.bits(m.A), synth.bits(B), synth.bits(X))
        check(_np(Y).astype(np.float64), ref)
        assert int(ws[:ZERO_REGION].count_nonzero()) == 0, T


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_fp4_split_matches_oracle(fmt):
    import torch
    from test_gpu_fp4 import _fp4_modules
    T, d, outs, r = 40, 4096, [512, 256], 32
    assert _splits(T, r, d, outs)
    host, dev, B = _fp4_modules(fmt, d, outs, 960, r)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=960)
    Ys, R = glowq.group_forward_fp4(dev, torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    refs, R_ref = oracle.fp4_group_forward(fmt, host, synth.bits(B), synth.bits(X))
    assert normwise(_np(R).astype(np.float64), R_ref) < 1e-3
    for Y, ref in zip(Ys, refs):
        check(_np(Y).astype(np.float64), ref)


@pytest.mark.parametrize("T,d,O", [(32, 5120, 5120), (64, 13824, 5120)])
def test_llama2_13b_solo_decode_batches(T, d, O):
    """LLaMA-2-13B o_proj (5120 -> 5120) at T = 32 and down_proj (13824 -> 5120)
    at T = 64, r = 64: 20 tiles of 256 rows split across the pairs; every
    output element against the oracle."""
    import torch
    r = 64
    assert _splits(T, r, d, [O])
    mods = make_modules(d, [O], seed=970 + T)
    B = attach_random_factors(mods, d, r, seed=970 + T)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=970 + T)
    Y = glowq.solo_forward(to_dev(mods)[0], torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    m = mods[0]
    ref = oracle.solo_forward(m.q, m.s, m.z, synth.bits(m.A), synth.bits(B), synth.bits(X))
    check(_np(Y).astype(np.float64), ref)
