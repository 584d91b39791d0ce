"""GPU parity of the MXFP4 / NVFP4 base-weight path (thelatestinai.com GlowQ
page, Table 13): packing and dequantisation bit-exact against the oracle."""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

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


def _edge_weights(d):
    W = synth.weights(12, d, seed=31, outlier_cols=3)
    W[0, :128] = 0.0                                         # all-zero blocks
    W[1, :32] = 1e-30                                        # E8M0 clamps at 0, subnormal block scale
    W[2, 40] = np.nan                                        # NaN element -> code 0
    W[3, :64] = -2.5                                         # constant blocks
    W[4, 128:160] = np.float32(3e4)                          # large block
    W[5, :32] = np.linspace(-1, 1, 32, dtype=np.float32)     # E2M1 ties within the block grid
    W[6, :16] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, -0.25, -0.1, 0.0, -0.0, 1e-3, -5.0, 4.0],
                         dtype=np.float32)                   # midpoints of the E2M1 grid (block amax 7)
    W[7, 64:96] = -1e-6                                      # tiny negatives -> +0
    return W


@pytest.mark.parametrize("O,d", [(256, 256), (96, 1152), (1024, 4096)])
def test_mxfp4_pack_and_dequant_bit_exact(O, d):
    import torch
    W = synth.weights(O, d, seed=32, outlier_cols=4)
    codes_o, scales_o = oracle.quantize_mxfp4(W)
    q, sc, _ = glowq.pack_fp4(torch.from_numpy(W).cuda(), glowq.FMT_MXFP4)
    assert np.array_equal(_np(q).view(np.uint8).reshape(O, d // 2), codes_o)
    assert np.array_equal(_np(sc), scales_o)
    deq = _np(glowq.dequant_fp4(q, sc, None, d, glowq.FMT_MXFP4)).view(np.uint16)
    assert np.array_equal(deq, oracle.dequant_mxfp4(codes_o, scales_o, d))


@pytest.mark.parametrize("O,d", [(256, 256), (96, 1152), (1024, 4096)])
def test_nvfp4_pack_and_dequant_bit_exact(O, d):
    import torch
    W = synth.weights(O, d, seed=33, outlier_cols=4)
    codes_o, scales_o, ts_o = oracle.quantize_nvfp4(W)
    q, sc, ts = glowq.pack_fp4(torch.from_numpy(W).cuda(), glowq.FMT_NVFP4)
    assert np.float32(_np(ts)[0]) == np.float32(ts_o)
    assert np.array_equal(_np(sc), scales_o)
    assert np.array_equal(_np(q).view(np.uint8).reshape(O, d // 2), codes_o)
    deq = _np(glowq.dequant_fp4(q, sc, ts, d, glowq.FMT_NVFP4)).view(np.uint16)
    assert np.array_equal(deq, oracle.dequant_nvfp4(codes_o, scales_o, ts_o, d))


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_fp4_edge_values_bit_exact(fmt):
    import torch
    d = 256
    W = _edge_weights(d)
    Wd = torch.from_numpy(W).cuda()
    if fmt == "mx":
        codes_o, scales_o = oracle.quantize_mxfp4(W)
        q, sc, ts = glowq.pack_fp4(Wd, glowq.FMT_MXFP4)
        ref = oracle.dequant_mxfp4(codes_o, scales_o, d)
        f = glowq.FMT_MXFP4
    else:
        codes_o, scales_o, ts_o = oracle.quantize_nvfp4(W)
        q, sc, ts = glowq.pack_fp4(Wd, glowq.FMT_NVFP4)
        assert np.float32(_np(ts)[0]) == np.float32(ts_o)
        ref = oracle.dequant_nvfp4(codes_o, scales_o, ts_o, d)
        f = glowq.FMT_NVFP4
    assert np.array_equal(_np(sc), scales_o)
    assert np.array_equal(_np(q).view(np.uint8).reshape(W.shape[0], d // 2), codes_o)
    assert np.array_equal(_np(glowq.dequant_fp4(q, sc, ts, d, f)).view(np.uint16), ref)


# ------------------------------------------------------- forward with FP4 weights

def _fp4_modules(fmt, d, outs, seed, r):
    from helpers import attach_random_factors, make_modules
    import torch
    mods = make_modules(d, outs, seed=seed)
    B = attach_random_factors(mods, d, r, seed=seed) if r else None
    host, dev = [], []
    for m in mods:
        if fmt == "mx":
            codes, scales = oracle.quantize_mxfp4(m.W)
            ts = None
        else:
            codes, scales, ts = oracle.quantize_nvfp4(m.W)
        A = None if (m.A is None or not r) else m.A
        host.append((codes, scales, ts, None if A is None else synth.bits(A)))
        dev.append(glowq.FP4Module(glowq.FMT_MXFP4 if fmt == "mx" else glowq.FMT_NVFP4,
                                   torch.from_numpy(codes.view(np.int32)).cuda(), torch.from_numpy(scales).cuda(),
                                   None if ts is None else torch.tensor([ts], dtype=torch.float32, device="cuda"),
                                   None if A is None else torch.from_numpy(A).cuda()))
    return host, dev, B


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("T", [1, 5, 16, 17, 300])
def test_fp4_group_forward_matches_oracle(fmt, T):
    """Q/K/V-like group with MXFP4 / NVFP4 base weights, r = 32, decode (T <= 16)
    and tensor-core (T > 16) paths, ragged row tiles."""
    import torch
    from helpers import check, normwise
    d, r = 512, 32
    host, dev, B = _fp4_modules(fmt, d, [256, 48, 144], 40 + T, r)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=40 + T)
    Ys, R = glowq.group_forward_fp4(dev, torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    refs, R_ref = oracle.fp4_group_forward(fmt, host, synth.bits(B), synth.bits(X))
    assert normwise(_np(R).astype(np.float64), R_ref) < 1e-3
    for Y, ref in zip(Ys, refs):
        check(_np(Y).astype(np.float64), ref)


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("T", [1, 16, 512])
def test_fp4_llama_shaped_solo_and_group(fmt, T):
    """d = 4096: a two-module group (1024 + 512 rows) and an o_proj-like solo
    (512 x 4096), r = 64, at decode and prefill token counts."""
    import torch
    from helpers import check
    d, r = 4096, 64
    host, dev, B = _fp4_modules(fmt, d, [1024, 512], 50 + T, r)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=50 + T)
    Ys, _ = glowq.group_forward_fp4(dev, torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    refs, _ = oracle.fp4_group_forward(fmt, host, synth.bits(B), synth.bits(X))
    for Y, ref in zip(Ys, refs):
        check(_np(Y).astype(np.float64), ref)
    hs, ds, Bs = _fp4_modules(fmt, d, [512], 60 + T, r)
    Y = glowq.solo_forward_fp4(ds[0], torch.from_numpy(Bs).cuda(), torch.from_numpy(X).cuda())
    (ref,), _ = oracle.fp4_group_forward(fmt, hs, synth.bits(Bs), synth.bits(X))
    check(_np(Y).astype(np.float64), ref)


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_fp4_rank_zero(fmt):
    """r = 0 (a GlowQ-S unit that is not restored): plain W4A16 with FP4 weights."""
    import torch
    from helpers import check
    d = 1024
    host, dev, _ = _fp4_modules(fmt, d, [128, 64], 70, 0)
    for T in (3, 40):
        X = synth.activations(T, d, synth.ALPHA_QKV, seed=70 + T)
        Ys, R = glowq.group_forward_fp4(dev, None, torch.from_numpy(X).cuda())
        assert R is None
        refs, _ = oracle.fp4_group_forward(fmt, host, None, synth.bits(X))
        for Y, ref in zip(Ys, refs):
            check(_np(Y).astype(np.float64), ref)
