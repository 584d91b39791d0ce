"""GPU parity of the packing kernels and the small-T (decode) corrected linear.

Compares the CUDA path, called through the C ABI, with the CPU oracle on the
same seeded inputs: bit-exact for INT4 codes, scales, zeros and dequantised
weights; normwise relative error <= 2e-3 for fp16 outputs.
Pages: papernotes.org GlowQ summary, key design 4 and the set-up paragraph.
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

from helpers import (check, TOL, attach_random_factors, attach_solved_factors, make_modules, normwise, tile_int4,
                     to_dev, untile_int4)

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


# ------------------------------------------------------------- pack / dequant

@pytest.mark.parametrize("O,d,outliers", [(256, 256, 4), (144, 1152, 0), (4096, 4096, 0), (1024, 14336, 8)])
def test_pack_bit_exact(O, d, outliers):
    import torch
    W = synth.weights(O, d, seed=21, outlier_cols=outliers)
    q_o, s_o, z_o = oracle.quantize_int4(W)
    q, s, z = glowq.pack_int4(torch.from_numpy(W).cuda())
    assert np.array_equal(untile_int4(_np(q).view(np.uint32)), q_o)
    assert np.array_equal(_np(s).view(np.uint16), s_o)
    assert np.array_equal(_np(z), z_o)


def test_pack_edge_values_bit_exact():
    import torch
    d = 512
    W = synth.weights(16, d, seed=22)                  # one 16-row block
    W[0, :128] = 0.0                                  # all-zero group
    W[1, :128] = 1e-30                                # scale underflow -> 1.0
    W[2, 5] = np.nan                                  # NaN weight -> code 0
    W[3, :128] = -2.5                                 # constant negative group
    W[4, 128:256] = np.float32(1e6)                   # scale overflow -> 65504
    W[5, 300] = np.inf
    W[6, 256:384] = np.linspace(-1, 3, 128, dtype=np.float32)
    q_o, s_o, z_o = oracle.quantize_int4(W)
    q, s, z = glowq.pack_int4(torch.from_numpy(W).cuda())
    assert np.array_equal(untile_int4(_np(q).view(np.uint32)), q_o)
    assert np.array_equal(_np(s).view(np.uint16), s_o)
    assert np.array_equal(_np(z), z_o)


@pytest.mark.parametrize("O,d", [(256, 256), (4096, 11008)])
def test_dequant_bit_exact(O, d):
    import torch
    W = synth.weights(O, d, seed=23, outlier_cols=3)
    q_o, s_o, z_o = oracle.quantize_int4(W)
    ref = oracle.dequant_int4(q_o, s_o, z_o, d)
    out = glowq.dequant_int4(torch.from_numpy(tile_int4(q_o).view(np.int32)).cuda(),
                             torch.from_numpy(s_o.view(np.float16)).cuda(), torch.from_numpy(z_o).cuda(), d)
    assert np.array_equal(_np(out).view(np.uint16), ref)


def test_error_norms_match_oracle():
    import torch
    O, d = 512, 1024
    W = synth.weights(O, d, seed=24, outlier_cols=4)
    q, s, z = oracle.quantize_int4(W)
    rows = _np(glowq.error_norms(torch.from_numpy(W).cuda(), torch.from_numpy(tile_int4(q).view(np.int32)).cuda(),
                                 torch.from_numpy(s.view(np.float16)).cuda(), torch.from_numpy(z).cuda()))
    _, e2, w2 = oracle.quant_error(W, q, s, z, want_matrix=False)
    assert rows.sum(axis=0)[0] == pytest.approx(e2, rel=1e-12)
    assert rows.sum(axis=0)[1] == pytest.approx(w2, rel=1e-12)


# ------------------------------------------------------------- decode forward

def _run_group(mods, B, X, device="cuda"):
    import torch
    dm = to_dev(mods, device)
    Bt = None if B is None else torch.from_numpy(B).to(device)
    Xt = torch.from_numpy(X).to(device)
    Ys, R = glowq.group_forward(dm, Bt, Xt)
    torch.cuda.synchronize()
    return [_np(Y).astype(np.float64) for Y in Ys], (None if R is None else _np(R).astype(np.float64))


def _oracle_group(mods, B, X):
    Xb = synth.bits(X)
    outs, R = oracle.group_forward([(m.q, m.s, m.z, None if m.A is None else synth.bits(m.A)) for m in mods],
                                   None if B is None else synth.bits(B), Xb)
    return outs, R


def test_tiny_qkv_group_with_solved_factors():
    """d=256, Q/K/V 256 each, 4 outlier columns x10, r=16 whitened solve, T=8, alpha=1.19, seed 0."""
    d, r, T = 256, 16, 8
    mods = make_modules(d, [256, 256, 256], seed=0, outlier_cols=4)
    basis = synth.orthogonal_basis(d, seed=0)
    B = attach_solved_factors(mods, d, r, synth.ALPHA_QKV, seed=0, basis=basis)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=0, basis=basis)
    ys, R = _run_group(mods, B, X)
    refs, R_ref = _oracle_group(mods, B, X)
    assert normwise(R, R_ref) < 1e-3
    for y, ref in zip(ys, refs):
        check(y, ref)


@pytest.mark.parametrize("T", [1, 2, 3, 5, 7, 8, 9, 12, 15, 16])
def test_decode_token_counts(T):
    d, r = 640, 24                                   # 5 groups of 128: ragged split along d
    mods = make_modules(d, [128, 48, 80], seed=30 + T)
    B = attach_random_factors(mods, d, r, seed=30 + T)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=30 + T)
    ys, R = _run_group(mods, B, X)
    refs, R_ref = _oracle_group(mods, B, X)
    assert normwise(R, R_ref) < 1e-3
    for y, ref in zip(ys, refs):
        assert y.shape == ref.shape
        check(y, ref)


def test_rank_zero_and_disabled_module():
    d, T = 512, 4
    mods = make_modules(d, [64, 64], seed=40)
    B = attach_random_factors(mods, d, 16, seed=40)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=40)
    # r = 0 for the whole group: plain W4A16
    ys, R = _run_group(mods, None, X)
    assert R is None
    for y, m in zip(ys, mods):
        ref = oracle.solo_forward(m.q, m.s, m.z, None, None, synth.bits(X))
        check(y, ref)
    # one module with its correction switched off
    mods[1].A = None
    ys, _ = _run_group(mods, B, X)
    refs, _ = _oracle_group(mods, B, X)
    for y, ref in zip(ys, refs):
        check(y, ref)


def test_solo_equals_group_of_one_and_oracle():
    import torch
    d, r, T = 1024, 32, 6
    mods = make_modules(d, [256], seed=41)
    B = attach_random_factors(mods, d, r, seed=41)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=41)
    dm = to_dev(mods)[0]
    Xt, Bt = torch.from_numpy(X).cuda(), torch.from_numpy(B).cuda()
    Y = _np(glowq.solo_forward(dm, Bt, Xt)).astype(np.float64)
    (Yg,), _ = glowq.group_forward([dm], Bt, Xt)
    assert np.array_equal(Y, _np(Yg).astype(np.float64))
    ref = oracle.solo_forward(mods[0].q, mods[0].s, mods[0].z, synth.bits(mods[0].A), synth.bits(B), synth.bits(X))
    check(Y, ref)


def test_outputs_land_in_one_buffer_with_leading_dimension():
    """Q/K/V written as column blocks of one T x (sum O) buffer via ldY."""
    import torch
    d, r, T = 512, 16, 5
    outs = [128, 32, 32]
    mods = make_modules(d, outs, seed=42)
    B = attach_random_factors(mods, d, r, seed=42)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=42)
    buf = torch.full((T, sum(outs) + 8), float("nan"), dtype=torch.float16, device="cuda")
    views, c = [], 0
    for O in outs:
        views.append(buf[:, c:c + O])
        c += O
    glowq.group_forward(to_dev(mods), torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda(), Ys=views)
    host = _np(buf).astype(np.float64)
    refs, _ = _oracle_group(mods, B, X)
    c = 0
    for O, ref in zip(outs, refs):
        check(host[:, c:c + O], ref)
        c += O
    assert np.all(np.isnan(host[:, c:]))              # padding columns untouched


def test_decode_deterministic():
    import torch
    d, r, T = 2048, 64, 16
    mods = make_modules(d, [512, 256], seed=43)
    B = attach_random_factors(mods, d, r, seed=43)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=43)
    dm = to_dev(mods)
    Bt, Xt = torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda()
    a, Ra = glowq.group_forward(dm, Bt, Xt)
    b, Rb = glowq.group_forward(dm, Bt, Xt)
    assert torch.equal(Ra, Rb)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ------------------------------------------------------- full-size workloads

@pytest.mark.parametrize("T", [1, 4, 16])
def test_llama2_7b_attention_decode(T):
    """QKV group 3 x 4096x4096 + solo o_proj 4096x4096, r=64, alpha=1.19 (full compare)."""
    import torch
    d, r = 4096, 64
    qkv = make_modules(d, [4096, 4096, 4096], seed=0)
    Bq = attach_random_factors(qkv, d, r, seed=0, sub=0)
    o = make_modules(d, [4096], seed=0, sub0=10)
    Bo = attach_random_factors(o, d, r, seed=0, sub=1)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=0)
    ys, R = _run_group(qkv, Bq, X)
    refs, R_ref = _oracle_group(qkv, Bq, X)
    assert normwise(R, R_ref) < 1e-3
    for y, ref in zip(ys, refs):
        check(y, ref)
    X2 = synth.activations(T, d, synth.ALPHA_QKV, seed=0, sub=1)
    Yo = _np(glowq.solo_forward(to_dev(o)[0], torch.from_numpy(Bo).cuda(), torch.from_numpy(X2).cuda()))
    ref = oracle.solo_forward(o[0].q, o[0].s, o[0].z, synth.bits(o[0].A), synth.bits(Bo), synth.bits(X2))
    check(Yo.astype(np.float64), ref)


def test_llama31_8b_layer_decode_t1():
    """GQA QKV 4096/1024/1024, gate/up 2x14336, o 4096, down 14336->4096 at T=1."""
    import torch
    d, r, T = 4096, 64, 1
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=0)
    for outs, alpha, sub in [([4096, 1024, 1024], synth.ALPHA_QKV, 0), ([14336, 14336], synth.ALPHA_MLP, 10)]:
        mods = make_modules(d, outs, seed=1, sub0=sub)
        B = attach_random_factors(mods, d, r, seed=1, sub=sub)
        ys, _ = _run_group(mods, B, X)
        refs, _ = _oracle_group(mods, B, X)
        for y, ref in zip(ys, refs):
            check(y, ref)
    down = make_modules(14336, [4096], seed=1, sub0=20)
    Bd = attach_random_factors(down, 14336, r, seed=1, sub=20)
    Xd = synth.activations(T, 14336, synth.ALPHA_MLP, seed=1)
    Y = _np(glowq.solo_forward(to_dev(down)[0], torch.from_numpy(Bd).cuda(), torch.from_numpy(Xd).cuda()))
    ref = oracle.solo_forward(down[0].q, down[0].s, down[0].z, synth.bits(down[0].A), synth.bits(Bd),
                              synth.bits(Xd))
    check(Y.astype(np.float64), ref)


@pytest.mark.parametrize("T", [1, 16])
@pytest.mark.parametrize("r", [8, 256])
def test_decode_rank_extremes_and_eight_modules(T, r):
    """Smallest and largest rank with the largest group (8 modules, 16..128 rows)."""
    import torch
    d = 1024
    outs = [16, 32, 48, 64, 80, 96, 112, 128]
    mods = make_modules(d, outs, seed=60 + r + T)
    B = attach_random_factors(mods, d, r, seed=60 + r + T)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=60 + T)
    Ys, R = glowq.group_forward(to_dev(mods), torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    Rr = oracle.anchor_project(synth.bits(X), synth.bits(B))
    assert normwise(R.cpu().numpy().astype(np.float64), Rr) < 1e-3
    for m, Y in zip(mods, Ys):
        ref = oracle.module_forward(m.q, m.s, m.z, synth.bits(m.A), Rr, synth.bits(X))
        check(Y.cpu().numpy().astype(np.float64), ref)


def test_decode_wide_input_solo():
    """LLaMA-3.1-8B down_proj shape at T=1: 4096 x 14336 (R's B slice too wide to stage)."""
    import torch
    d, O, r, T = 14336, 4096, 64, 1
    mods = make_modules(d, [O], seed=65)
    B = attach_random_factors(mods, d, r, seed=65)
    X = synth.activations(T, d, synth.ALPHA_MLP, seed=65)
    Y = glowq.solo_forward(to_dev(mods)[0], torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    ref = oracle.solo_forward(mods[0].q, mods[0].s, mods[0].z, synth.bits(mods[0].A), synth.bits(B), synth.bits(X))
    check(Y.cpu().numpy().astype(np.float64), ref)


def test_workspace_flags_shared_by_decode_prefill_and_solo_calls():
    """One workspace serves decode group, prefill group and decode solo calls in
    turn (any T, one stream): the zero region at offset 0 (decode hand-off
    flags, k-split tickets) is zero after every call and the outputs match the oracle throughout."""
    import torch
    d, r = 512, 32
    mods = make_modules(d, [128, 64], seed=91)
    B = attach_random_factors(mods, d, r, seed=91)
    dev = to_dev(mods)
    Bd = torch.from_numpy(B).cuda()
    ws = glowq.alloc_workspace(64, r)
    for k, T in enumerate((1, 64, 3, 16, 1)):
        X = synth.activations(T, d, synth.ALPHA_QKV, seed=92 + k)
        Xd = torch.from_numpy(X).cuda()
        Ys, R = glowq.group_forward(dev, Bd, Xd, workspace=ws)
        Yo = glowq.solo_forward(dev[1], Bd, Xd, workspace=ws)
        torch.cuda.synchronize()
        assert int(ws[:4096].view(torch.int32).abs().sum()) == 0, (T, ws[:72].tolist())
        refs, R_ref = _oracle_group(mods, B, X)
        assert normwise(_np(R).astype(np.float64), R_ref) < 1e-3
        for y, ref in zip(Ys, refs):
            check(_np(y).astype(np.float64), ref)
        check(_np(Yo).astype(np.float64), refs[1])


@pytest.mark.parametrize("T", [1, 16])
def test_decode_activation_outliers(T):
    """Heavy-tailed activations: 6 seeded input columns scaled x100 (values in
    the hundreds), through the LLaMA-2-7B Q/K/V group and o_proj.  The decode
    GEMV finishes each 128-group as s (64 D_E + D_O - (1024 + z) S_E - (64 + z) S_O),
    which cancels terms ~100x larger than the result; the outlier columns make
    those terms largest."""
    import torch
    d, r = 4096, 64
    cols = synth.outlier_columns(d, 6, seed=7)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=7).astype(np.float32)
    X[:, cols] *= 100.0
    X = X.astype(np.float16)
    assert np.all(np.isfinite(X)) and np.abs(X).max() > 100.0
    qkv = make_modules(d, [4096, 4096, 4096], seed=7)
    Bq = attach_random_factors(qkv, d, r, seed=7, sub=0)
    ys, R = _run_group(qkv, Bq, X)
    refs, R_ref = _oracle_group(qkv, Bq, X)
    assert normwise(R, R_ref) < 1e-3
    for y, ref in zip(ys, refs):
        check(y, ref)
    o = make_modules(d, [4096], seed=7, sub0=10)
    Bo = attach_random_factors(o, d, r, seed=7, sub=1)
    Yo = _np(glowq.solo_forward(to_dev(o)[0], torch.from_numpy(Bo).cuda(), torch.from_numpy(X).cuda()))
    ref = oracle.solo_forward(o[0].q, o[0].s, o[0].z, synth.bits(o[0].A), synth.bits(Bo), synth.bits(X))
    check(Yo.astype(np.float64), ref)


@pytest.mark.parametrize("T", [1, 16, 100])
def test_forward_plan_repeats_with_refilled_input(T):
    """glowq.ForwardPlan marshals a call once; refilling X in place and calling
    the plan again gives the new input's outputs (group and solo plans)."""
    import torch
    d, r = 1024, 32
    mods = make_modules(d, [256, 128], seed=110 + T)
    B = attach_random_factors(mods, d, r, seed=110 + T)
    dev = to_dev(mods)
    Bt = torch.from_numpy(B).cuda()
    Xd = torch.empty((T, d), dtype=torch.float16, device="cuda")
    Ys = [torch.empty((T, m.out_features), dtype=torch.float16, device="cuda") for m in dev]
    Yo = torch.empty((T, 128), dtype=torch.float16, device="cuda")
    pg = glowq.ForwardPlan(dev, Bt, Xd, Ys)
    ps = glowq.ForwardPlan([dev[1]], Bt, Xd, [Yo], solo=True)
    for k in range(2):
        X = synth.activations(T, d, synth.ALPHA_QKV, seed=120 + 10 * T + k)
        Xd.copy_(torch.from_numpy(X))
        pg()
        ps()
        torch.cuda.synchronize()
        refs, _ = _oracle_group(mods, B, X)
        for Y, ref in zip(Ys, refs):
            check(_np(Y).astype(np.float64), ref)
        check(_np(Yo).astype(np.float64), refs[1])
