"""The allocation-free solo forward matches the oracle.

glowq_solo_forward_noalloc is for callers that cannot allocate device memory
at call time (for example a custom op or plugin inside another runtime's
enqueue step, where that runtime owns every allocation): it takes no workspace
and uses a fixed scratch array compiled into the library.  Every call shares
that array, so each test makes two calls in a row with different inputs and
checks both against the CPU oracle.  This file runs last (pytest collects it
after the others) and passes alone or after the suite.
"""
import ctypes as C

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


def _noalloc(m, d, Bt, r, X, O):
    """One call through the C ABI; returns (status, Y on the host)."""
    import torch
    T = X.shape[0]
    Y = torch.full((T, O), float("nan"), dtype=torch.float16, device="cuda")
    arr = glowq._module_structs([m], [Y], True)
    rc = glowq.lib().glowq_solo_forward_noalloc(arr, d, Bt.data_ptr(), r, X.data_ptr(), T,
                                                 C.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, Y.cpu().numpy().astype(np.float64)


def _largest_T(r):
    cap = glowq.noalloc_scratch_bytes()
    T = 1
    while glowq.workspace_bytes(T + 1, r) <= cap:
        T += 1
    return T


@pytest.mark.parametrize("d,O,T", [(4096, 256, 1), (4096, 256, 16), (512, 144, 300)])
def test_noalloc_matches_oracle_twice(d, O, T):
    import torch
    r = 64
    mods = make_modules(d, [O], seed=90 + T)
    B = attach_random_factors(mods, d, r, seed=90 + T)
    m = to_dev(mods)[0]
    Bt = torch.from_numpy(B).cuda()
    h = mods[0]
    # two calls in a row, different inputs, one shared scratch array
    for seed in (1, 2):
        X = synth.activations(T, d, synth.ALPHA_QKV, seed=seed)
        rc, got = _noalloc(m, d, Bt, r, torch.from_numpy(X).cuda(), O)
        assert rc == 0
        assert np.all(np.isfinite(got))
        ref = oracle.solo_forward(h.q, h.s, h.z, synth.bits(h.A), synth.bits(B), synth.bits(X))
        check(got, ref)


def test_noalloc_size_boundary():
    """The largest T whose scratch need fits is accepted and correct; T + 1 is rejected."""
    import torch
    r, d, O = 64, 256, 64
    Tmax = _largest_T(r)
    assert Tmax == 480                       # 4096 + 8*T*r*4 + align256(T*r*2) <= 1 MiB
    mods = make_modules(d, [O], seed=97)
    B = attach_random_factors(mods, d, r, seed=97)
    m = to_dev(mods)[0]
    Bt = torch.from_numpy(B).cuda()
    h = mods[0]
    X = synth.activations(Tmax + 1, d, synth.ALPHA_QKV, seed=97)
    rc, got = _noalloc(m, d, Bt, r, torch.from_numpy(X[:Tmax]).cuda(), O)
    assert rc == 0
    ref = oracle.solo_forward(h.q, h.s, h.z, synth.bits(h.A), synth.bits(B), synth.bits(X[:Tmax]))
    check(got, ref)
    rc, got = _noalloc(m, d, Bt, r, torch.from_numpy(X).cuda(), O)
    assert rc == 2                           # GLOWQ_ERR_SHAPE, nothing enqueued
    assert np.all(np.isnan(got))             # output untouched


def test_noalloc_rejects_oversized_requests():
    import torch
    cap = glowq.noalloc_scratch_bytes()
    assert cap == 1 << 20
    T = 2 * cap // (64 * 2)          # R alone (T x 64 fp16) would need twice the scratch
    assert glowq.workspace_bytes(T, 64) > cap
    mods = make_modules(256, [64], seed=99)
    attach_random_factors(mods, 256, 64, seed=99)
    m = to_dev(mods)[0]
    B = torch.zeros((64, 256), dtype=torch.float16, device="cuda")
    X = torch.zeros((16, 256), dtype=torch.float16, device="cuda")
    Y = torch.empty((T, 64), dtype=torch.float16, device="cuda")
    arr = glowq._module_structs([m], [Y], True)
    rc = glowq.lib().glowq_solo_forward_noalloc(arr, 256, B.data_ptr(), 64, X.data_ptr(), T, None)
    assert rc == 2                   # GLOWQ_ERR_SHAPE, nothing enqueued


def test_noalloc_after_a_timed_out_wait():
    """A bounded wait that ran out (recorded in the device status word) leaves
    the next allocation-free decode calls correct: each call clears the zero
    region (hand-off flags, k-split tickets) of the shared array before its
    kernels."""
    import torch
    glowq.selftest_wait_timeout(polls=64)
    assert glowq.device_status() == 5        # GLOWQ_ERR_TIMEOUT, read and cleared
    d, O, r = 1024, 128, 32
    mods = make_modules(d, [O], seed=98)
    B = attach_random_factors(mods, d, r, seed=98)
    m = to_dev(mods)[0]
    Bt = torch.from_numpy(B).cuda()
    h = mods[0]
    for T in (1, 16):
        X = synth.activations(T, d, synth.ALPHA_MLP, seed=98 + T)
        rc, got = _noalloc(m, d, Bt, r, torch.from_numpy(X).cuda(), O)
        assert rc == 0
        ref = oracle.solo_forward(h.q, h.s, h.z, synth.bits(h.A), synth.bits(B), synth.bits(X))
        check(got, ref)


def test_noalloc_small_batch_split_twice():
    """A small batch (T = 40) whose 256-row tiles are too few for the GPU takes
    the k-split inside the fixed array (tickets in its zero region, partial
    tiles behind R): two calls in a row match the oracle, so the tickets the
    first call leaves are the zeros the second one needs."""
    import torch
    d, O, r, T = 4096, 1024, 64, 40
    assert glowq.workspace_bytes_for(T, r, d, [O]) > glowq.workspace_bytes(T, r)
    mods = make_modules(d, [O], seed=96)
    B = attach_random_factors(mods, d, r, seed=96)
    m = to_dev(mods)[0]
    Bt = torch.from_numpy(B).cuda()
    h = mods[0]
    for k in range(2):
        X = synth.activations(T, d, synth.ALPHA_MLP, seed=96 + k)
        rc, got = _noalloc(m, d, Bt, r, torch.from_numpy(X).cuda(), O)
        assert rc == 0
        ref = oracle.solo_forward(h.q, h.s, h.z, synth.bits(h.A), synth.bits(B), synth.bits(X))
        check(got, ref)
