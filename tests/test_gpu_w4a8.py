"""GPU W4A8 path (thelatestinai.com GlowQ page, Tables 14-15: GlowQ with FP8
activations): the per-token E4M3 quantiser bit-exact against the oracle, and
the W4A8 group / solo forward against the oracle's W4A8 forward (decode and
tensor-core paths)."""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

from helpers import attach_random_factors, check, make_modules, normwise, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    glowq.lib()
    yield
    assert glowq.device_status() == 0


@pytest.mark.parametrize("T,d", [(1, 4096), (7, 640), (300, 1024)])
def test_quantize_act_bit_exact(T, d):
    import torch
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=80 + T)
    X[0, :5] = np.array([0.0, -0.0, 1e-7, -1e-7, 60000.0], dtype=np.float16)   # zeros, tiny, large
    if T > 1:
        X[1] = 0.0                                                            # all-zero token: s = 1
    codes_o, scales_o = oracle.quantize_act_e4m3(synth.bits(X))
    codes, scales, Xq = glowq.quantize_act_e4m3(torch.from_numpy(X).cuda())
    assert np.array_equal(scales.cpu().numpy(), scales_o)
    assert np.array_equal(codes.cpu().numpy(), codes_o)
    xh = oracle.dequant_act_e4m3(codes_o, scales_o)
    got = Xq.cpu().numpy().astype(np.float64) * scales_o.astype(np.float64)[:, None]
    assert np.array_equal(got, xh)


@pytest.mark.parametrize("T", [1, 5, 16, 17, 300])
def test_w4a8_group_and_solo_match_oracle(T):
    import torch
    d, r = 768, 32
    mods = make_modules(d, [256, 48, 144], seed=90 + T)
    B = attach_random_factors(mods, d, r, seed=90 + T)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=90 + T)
    dm = to_dev(mods)
    Bt, Xt = torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda()
    Ys, R = glowq.group_forward_w4a8(dm, Bt, Xt)
    torch.cuda.synchronize()
    refs, R_ref, _ = oracle.w4a8_group_forward([(m.q, m.s, m.z, synth.bits(m.A)) for m in mods], synth.bits(B),
                                               synth.bits(X))
    assert normwise(R.cpu().numpy().astype(np.float64), R_ref) < 1e-3
    for Y, ref in zip(Ys, refs):
        check(Y.cpu().numpy().astype(np.float64), ref)
    Y = glowq.solo_forward_w4a8(dm[2], Bt, Xt)
    check(Y.cpu().numpy().astype(np.float64), refs[2])


def test_w4a8_llama_shaped_decode_and_prefill():
    """LLaMA-2-7B Q/K/V-shaped group (3 x 4096 x 4096, r = 64) at T = 1 and a
    gate/up-shaped group (2 x 2048 x 4096) at T = 300 with FP8 activations."""
    import torch
    d, r = 4096, 64
    for outs, T in (([4096, 4096, 4096], 1), ([2048, 2048], 300)):
        mods = make_modules(d, outs, seed=95 + T)
        B = attach_random_factors(mods, d, r, seed=95 + T)
        X = synth.activations(T, d, synth.ALPHA_QKV, seed=95 + T)
        Ys, _ = glowq.group_forward_w4a8(to_dev(mods), torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
        refs, _, _ = oracle.w4a8_group_forward([(m.q, m.s, m.z, synth.bits(m.A)) for m in mods], synth.bits(B),
                                               synth.bits(X))
        for Y, ref in zip(Ys, refs):
            check(Y.cpu().numpy().astype(np.float64), ref)
