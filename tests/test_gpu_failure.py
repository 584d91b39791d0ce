"""Failure detection on the device without a fault: a bounded wait that runs
out records GLOWQ_ERR_TIMEOUT in the status word, the kernel returns, and the
context stays usable for the next forward call."""
import numpy as np
import pytest
import ctypes as C

from rank_error_correction_b200 import glowq, synth

from helpers import check, TOL, attach_random_factors, make_modules, normwise, to_dev

import oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert glowq.device_status() == 0                  # clean start (reads and clears)
    glowq.selftest_wait_timeout(polls=2048)
    assert glowq.device_status() == 5                  # GLOWQ_ERR_TIMEOUT recorded
    assert glowq.device_status() == 0                  # ... and cleared by the read
    # the context is usable: a forward call runs and matches the oracle
    d, T, r = 512, 4, 32
    mods = make_modules(d, [128, 64], seed=77)
    B = attach_random_factors(mods, d, r, seed=77)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=77)
    Ys, R = glowq.group_forward(to_dev(mods), torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    Rr = oracle.anchor_project(synth.bits(X), synth.bits(B))
    for m, Y in zip(mods, Ys):
        ref = oracle.module_forward(m.q, m.s, m.z, synth.bits(m.A), Rr, synth.bits(X))
        check(Y.cpu().numpy().astype(np.float64), ref)
    assert glowq.device_status() == 0


def test_selftest_rejects_bad_limits():
    assert glowq.lib().glowq_selftest_wait_timeout(0, None) == 1
    assert glowq.lib().glowq_selftest_wait_timeout(1 << 20, None) == 1
