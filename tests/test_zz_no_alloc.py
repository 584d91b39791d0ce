"""The allocation-free solo forward matches the regular solo forward.

glowq_solo_forward_noalloc is for callers that cannot allocate device memory
at call time (for example a custom op or plugin inside another runtime's
enqueue step, where that runtime owns every allocation): it takes no workspace
and uses a fixed scratch array compiled into the library.  This file runs last
(pytest collects it after the others) and passes alone or after the suite.
"""
import ctypes as C

import numpy as np
import pytest

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


@pytest.mark.parametrize("d,O,T", [(1024, 256, 8), (4096, 256, 16), (512, 144, 300)])
def test_noalloc_matches_solo_forward_twice(d, O, T):
    import torch
    r = 64
    mods = make_modules(d, [O], seed=90 + T)
    B = attach_random_factors(mods, d, r, seed=90 + T)
    m = to_dev(mods)[0]
    Bt = torch.from_numpy(B).cuda()
    ref = glowq.solo_forward(m, Bt, torch.from_numpy(synth.activations(T, d, synth.ALPHA_QKV, seed=1)).cuda())
    ref2 = glowq.solo_forward(m, Bt, torch.from_numpy(synth.activations(T, d, synth.ALPHA_QKV, seed=2)).cuda())
    # two calls in a row through the C ABI, different inputs, shared scratch
    for seed, want in ((1, ref), (2, ref2)):
        X = torch.from_numpy(synth.activations(T, d, synth.ALPHA_QKV, seed=seed)).cuda()
        Y = torch.full((T, O), float("nan"), dtype=torch.float16, device="cuda")
        arr = glowq._module_structs([m], [Y], True)
        rc = glowq.lib().glowq_solo_forward_noalloc(arr, d, Bt.data_ptr(), r, X.data_ptr(), T,
                                                     C.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0
        torch.cuda.synchronize()
        got = Y.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got))
        assert normwise(got, want.cpu().numpy().astype(np.float64)) < TOL


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
