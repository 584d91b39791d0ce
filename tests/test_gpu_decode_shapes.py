"""GPU parity of the decode kernel at every work shape of the library's measured
shape table: the LLaMA-2-7B, LLaMA-3.1-8B and LLaMA-2-13B units (Q/K/V groups,
o_proj, gate/up groups, down_proj) at one token count of each of the table's
token classes (T = 1, 4, 7, 11, 16) with r = 64, each unit
checked on sampled outputs of every module against the oracle.  The table
replaces the cost model's work shape for these sizes, so each of its entries
must meet the same parity bar as the shapes the model picks.
Pages: papernotes.org GlowQ summary, key design 4 and the set-up paragraph
(W4A16, g128, rank 64); model shapes of the thelatestinai.com GlowQ page,
Tables 3 and 8.
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import glowq, synth

from helpers import check

pytestmark = pytest.mark.gpu

R = 64
SEED = 21
# unit: (module output features, input dimension)
UNITS = {
    "o_4096": ([4096], 4096),
    "qkv_7b": ([4096] * 3, 4096),
    "qkv_8b": ([4096, 1024, 1024], 4096),
    "gu_8b": ([14336] * 2, 4096),
    "down_7b": ([4096], 11008),
    "down_8b": ([4096], 14336),
    "o_13b": ([5120], 5120),
    "qkv_13b": ([5120] * 3, 5120),
    "gu_13b": ([13824] * 2, 5120),
    "down_13b": ([5120], 13824),
}
# the table's entries, one token count per class (T = 1; 2-5; 6-8; 9-12; 13-16)
CASES = [(1, u) for u in ("o_4096", "qkv_7b", "qkv_8b", "down_7b", "down_8b", "o_13b", "down_13b")] + \
        [(4, u) for u in ("o_4096", "qkv_8b", "gu_8b", "down_7b", "down_8b", "o_13b", "gu_13b")] + \
        [(7, u) for u in ("o_4096", "qkv_8b", "gu_8b", "down_7b", "down_8b", "o_13b", "gu_13b")] + \
        [(11, u) for u in ("o_4096", "qkv_8b", "gu_8b", "down_7b", "down_8b", "o_13b", "qkv_13b", "gu_13b",
                           "down_13b")] + \
        [(16, u) for u in ("o_4096", "qkv_8b", "gu_8b", "down_8b", "o_13b", "qkv_13b", "down_13b")]

_BUILT = {}


def _unit(name):
    """Device modules packed by the library, host codes packed by the oracle
    from the same seeded weights, and the seeded r = 64 factors."""
    import torch
    if name not in _BUILT:
        outs, d = UNITS[name]
        dev, host = [], []
        for i, O in enumerate(outs):
            W = synth.device_weights(O, d, SEED, sub=100 * len(_BUILT) + i)
            q, s, z = glowq.pack_int4(W)
            dev.append(glowq.QModule(q, s, z))
            host.append(oracle.quantize_int4(W.cpu().numpy()))
            del W
        As, B = synth.device_factors(outs, d, R, SEED, sub=len(_BUILT))
        for m, A in zip(dev, As):
            m.A = A
        torch.cuda.synchronize()
        _BUILT[name] = dict(outs=outs, d=d, dev=dev, host=host, As_bits=[synth.bits(A.cpu().numpy()) for A in As],
                            B=B, B_bits=synth.bits(B.cpu().numpy()))
    return _BUILT[name]


@pytest.fixture(scope="module", autouse=True)
def _done():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    _BUILT.clear()
    assert glowq.device_status() == 0


@pytest.mark.parametrize("T,name", CASES)
def test_measured_shape_matches_oracle(T, name):
    import torch
    u = _unit(name)
    X = synth.activations(T, u["d"], synth.ALPHA_QKV, seed=SEED + T)
    Xd = torch.from_numpy(X).cuda()
    if len(u["dev"]) > 1:
        Ys, _ = glowq.group_forward(u["dev"], u["B"], Xd)
    else:
        Ys = [glowq.solo_forward(u["dev"][0], u["B"], Xd)]
    torch.cuda.synchronize()
    Xb = synth.bits(X)
    g = np.random.default_rng(T * 1000 + len(name))
    for (qh, sh, zh), A_bits, Y in zip(u["host"], u["As_bits"], Ys):
        O = qh.shape[0]
        n = 512
        ti, oi = g.integers(0, T, n), g.integers(0, O, n)
        ref = oracle.module_forward_sampled(qh, sh, zh, A_bits, u["B_bits"], Xb, ti, oi)
        got = Y.cpu().numpy()[ti, oi].astype(np.float64)
        check(got, ref)


@pytest.mark.parametrize("T,name", [(1, "o_4096"), (4, "gu_8b"), (16, "qkv_13b")])
def test_measured_shape_without_correction(T, name):
    """The table's shapes also serve r = 0 (plain W4A16, e.g. units GlowQ-S
    leaves unrestored)."""
    import torch
    u = _unit(name)
    X = synth.activations(T, u["d"], synth.ALPHA_MLP, seed=SEED + 7 * T)
    Xd = torch.from_numpy(X).cuda()
    plain = [glowq.QModule(m.qweight, m.scales, m.zeros) for m in u["dev"]]
    if len(plain) > 1:
        Ys, _ = glowq.group_forward(plain, None, Xd)
    else:
        Ys = [glowq.solo_forward(plain[0], None, Xd)]
    torch.cuda.synchronize()
    Xb = synth.bits(X)
    g = np.random.default_rng(T * 77 + len(name))
    for (qh, sh, zh), Y in zip(u["host"], Ys):
        O = qh.shape[0]
        ti, oi = g.integers(0, T, 512), g.integers(0, O, 512)
        ref = oracle.module_forward_sampled(qh, sh, zh, None, None, Xb, ti, oi)
        check(Y.cpu().numpy()[ti, oi].astype(np.float64), ref)
