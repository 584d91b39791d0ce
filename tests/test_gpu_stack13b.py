"""LLaMA-2-13B-shaped linear stack with GlowQ-S (d = 5120, ffn = 13824, r = 64).

Per layer the units are the Q/K/V group, the o_proj solo, the gate/up group and
the down_proj solo (an input-sharing group or a solo module is one unit).  The
GPU computes every module's quantisation error norms, the host ranks the units
by g_ner = ||E_u||_F^2 / ||W_u||_F^2 and restores the top half (GlowQ pages,
papernotes.org summary, GlowQ-S), and every unit then runs through the
corrected path when restored and the plain INT4 path (r = 0) otherwise, at
decode batch sizes and at prefill.  The oracle repeats the packing, the norms,
the selection and the outputs from the same seeded inputs.

Inputs come from the seeded device generator (weights and factors) and the
host activation generator; the oracle receives host copies of those inputs,
never a result of the kernels under test.
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import glowq, synth

from helpers import TOL, check, normwise

pytestmark = pytest.mark.gpu

D, FFN, R = 5120, 13824, 64
LAYERS = 2
SEED = 13
# (name, output features of the unit's modules, input dimension, activation alpha)
UNITS = [("qkv", [D, D, D], D, synth.ALPHA_QKV),
         ("o_proj", [D], D, synth.ALPHA_QKV),
         ("gate_up", [FFN, FFN], D, synth.ALPHA_MLP),
         ("down_proj", [D], FFN, synth.ALPHA_MLP)]
# units given 4 outlier input columns (x10), so that their error ratio stands out
OUTLIER_UNITS = {(0, 0), (1, 1), (1, 3)}


@pytest.fixture(scope="module")
def stack():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    units = []
    for layer in range(LAYERS):
        for kind, (name, outs, d, alpha) in enumerate(UNITS):
            dev_mods, host_mods = [], []
            e_gpu = w_gpu = e_ora = w_ora = 0.0
            for i, O in enumerate(outs):
                W = synth.device_weights(O, d, SEED, sub=1000 * layer + 100 * kind + i)
                if (layer, kind) in OUTLIER_UNITS:
                    cols = torch.arange(4, device=W.device) * (d // 4) + 7 * kind + layer
                    W[:, cols] *= 10.0
                q, s, z = glowq.pack_int4(W)
                en = glowq.error_norms(W, q, s, z).sum(dim=0).cpu().numpy()
                e_gpu += float(en[0])
                w_gpu += float(en[1])
                Wh = W.cpu().numpy()
                qh, sh, zh = oracle.quantize_int4(Wh)
                _, e2, w2 = oracle.quant_error(Wh, qh, sh, zh, want_matrix=False)
                e_ora += e2
                w_ora += w2
                dev_mods.append(glowq.QModule(q, s, z))
                host_mods.append((qh, sh, zh))
                del W, Wh
            As, B = synth.device_factors(outs, d, R, SEED, sub=10 * layer + kind)
            units.append(dict(layer=layer, kind=kind, name=name, outs=outs, d=d, alpha=alpha,
                              dev=dev_mods, host=host_mods, As=As, B=B,
                              As_bits=[synth.bits(A.cpu().numpy()) for A in As],
                              B_bits=synth.bits(B.cpu().numpy()),
                              e_gpu=e_gpu, w_gpu=w_gpu, e_ora=e_ora, w_ora=w_ora))
    torch.cuda.synchronize()
    yield units
    assert glowq.device_status() == 0


def _selection(units, which):
    e = np.array([u["e_" + which] for u in units])
    w = np.array([u["w_" + which] for u in units])
    layer = np.array([u["layer"] for u in units], np.int32)
    kind = np.array([u["kind"] for u in units], np.int32)
    return e, w, layer, kind


def test_glowq_s_selection_matches_oracle(stack):
    e_g, w_g, layer, kind = _selection(stack, "gpu")
    e_o, w_o, _, _ = _selection(stack, "ora")
    # the device norms are fp64 sums in another order: equal to ~1e-12 relative
    assert np.allclose(e_g, e_o, rtol=1e-9, atol=0) and np.allclose(w_g, w_o, rtol=1e-9, atol=0)
    k = len(stack) // 2                                    # GlowQ-S: restore the top 50%
    m_g, o_g, fb_g = glowq.select_restore(e_g, w_g, layer, kind, k)
    m_o, o_o, _, fb_o = oracle.select_restore(e_o, w_o, layer, kind, k)
    assert fb_g == fb_o == 0
    assert np.array_equal(m_g, m_o) and np.array_equal(o_g, o_o)
    assert int(m_g.sum()) == k
    # the units with outlier columns have the largest error ratios
    top = {(int(layer[i]), int(kind[i])) for i in o_g[:len(OUTLIER_UNITS)]}
    assert top == OUTLIER_UNITS


_X_CACHE = {}
_BASES = {}


def _activations(T, d, alpha, layer):
    # one orthogonal basis per width (building it dominates the host time); the
    # Gaussian draws differ per layer at decode sizes, while the T = 2048
    # inputs are shared by the layers (same shape and spectrum)
    if d not in _BASES:
        _BASES[d] = synth.orthogonal_basis(d, SEED)
    key = (T, d, alpha, layer if T <= 64 else -1)
    if key not in _X_CACHE:
        _X_CACHE[key] = synth.activations(T, d, alpha, seed=SEED, sub=key[3] + 1, basis=_BASES[d])
    return _X_CACHE[key]


@pytest.mark.parametrize("T", [1, 16, 64, 2048])
def test_stack_forward_matches_oracle(stack, T):
    """Restored units run with their factors, the others with r = 0; sampled outputs."""
    import torch
    e_g, w_g, layer, kind = _selection(stack, "gpu")
    mask, _, _ = glowq.select_restore(e_g, w_g, layer, kind, len(stack) // 2)
    g = np.random.default_rng(T)
    for u, restore in zip(stack, mask):
        X = _activations(T, u["d"], u["alpha"], u["layer"])
        Xd = torch.from_numpy(X).cuda()
        mods = u["dev"]
        for m, A in zip(mods, u["As"]):
            m.A = A if restore else None
        B = u["B"] if restore else None
        if len(mods) > 1:
            Ys, _ = glowq.group_forward(mods, B, Xd)
        else:
            Ys = [glowq.solo_forward(mods[0], B, Xd)]
        torch.cuda.synchronize()
        Xb = synth.bits(X)
        for (qh, sh, zh), A_bits, Y in zip(u["host"], u["As_bits"], Ys):
            O = qh.shape[0]
            n = 512
            ti, oi = g.integers(0, T, n), g.integers(0, O, n)
            ref = oracle.module_forward_sampled(qh, sh, zh, A_bits if restore else None,
                                                u["B_bits"] if restore else None, Xb, ti, oi)
            got = Y.cpu().numpy()[ti, oi].astype(np.float64)
            assert np.all(np.isfinite(got))
            assert normwise(got, ref) < TOL, (u["name"], u["layer"], bool(restore), T)
            check(got, ref)


@pytest.mark.parametrize("T", [1, 64])
def test_layerwise_mode_matches_oracle(stack, T):
    """Layerwise baseline: every module of the layer-0 Q/K/V group with its own
    factors (A_i, B_i) through the solo path, R_i = X B_i^T per module."""
    import torch
    u = stack[0]
    X = _activations(T, u["d"], u["alpha"], u["layer"])
    Xd = torch.from_numpy(X).cuda()
    Xb = synth.bits(X)
    g = np.random.default_rng(100 + T)
    for i, ((qh, sh, zh), m) in enumerate(zip(u["host"], u["dev"])):
        As, B = synth.device_factors([qh.shape[0]], u["d"], R, SEED, sub=900 + i)
        m.A = As[0]
        Y = glowq.solo_forward(m, B, Xd)
        torch.cuda.synchronize()
        n = 512
        ti, oi = g.integers(0, T, n), g.integers(0, qh.shape[0], n)
        ref = oracle.module_forward_sampled(qh, sh, zh, synth.bits(As[0].cpu().numpy()), synth.bits(B.cpu().numpy()),
                                            Xb, ti, oi)
        check(Y.cpu().numpy()[ti, oi].astype(np.float64), ref)
