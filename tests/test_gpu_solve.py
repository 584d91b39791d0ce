"""GPU offline group solve (papernotes.org GlowQ summary, key designs 1-3;
thelatestinai.com GlowQ page, Tables 11-12) against the oracle's whitened
solve with the same test matrix Omega and covariance root.  Singular vectors
carry a free sign, so the checks are on sign-free quantities: the products
A_i B, the singular values, the weighted objective and the energy capture."""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

from helpers import make_modules, tile_int4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    glowq.lib()
    yield
    assert glowq.device_status() == 0


def _case(d, outs, r, p, alpha, seed, outlier_cols=0):
    import torch
    mods = make_modules(d, outs, seed=seed, outlier_cols=outlier_cols)
    basis = synth.orthogonal_basis(d, seed=seed)
    Sh, Shp = synth.covariance_half(basis, synth.power_law_spectrum(d, alpha))
    Om = synth.gaussian_test_matrix(d, r + p, seed=seed)
    E = np.vstack([oracle.quant_error(m.W, m.q, m.s, m.z)[0] for m in mods])
    dev = dict(Ws=[torch.from_numpy(m.W).cuda() for m in mods],
               packs=[(torch.from_numpy(tile_int4(m.q).view(np.int32)).cuda(), torch.from_numpy(m.s.view(np.float16)).cuda(),
                       torch.from_numpy(m.z).cuda()) for m in mods],
               Sh=torch.from_numpy(np.ascontiguousarray(Sh)).cuda(),
               Shp=torch.from_numpy(np.ascontiguousarray(Shp)).cuda(),
               Om=torch.from_numpy(np.ascontiguousarray(Om)).cuda())
    return mods, E, Sh, Shp, Om, dev


@pytest.mark.parametrize("d,outs,r,p,q,alpha", [(256, [256, 256, 256], 16, 16, 2, 1.19),
                                                 (1024, [1024, 512], 64, 16, 2, 0.77),
                                                 (512, [128, 128], 24, 8, 0, 1.19)])
def test_group_solve_matches_oracle(d, outs, r, p, q, alpha):
    mods, E, Sh, Shp, Om, dev = _case(d, outs, r, p, alpha, seed=7 + d, outlier_cols=2)
    A_o, B_o, s_o = oracle.group_solve(E, Sh, Shp, r, p=p, q=q, Omega=Om)
    A, B, sing, gec, A16, B16 = glowq.group_solve(dev["Ws"], dev["packs"], dev["Sh"], dev["Shp"], r, p, q, dev["Om"])
    A, B, sing = A.cpu().numpy(), B.cpu().numpy(), sing.cpu().numpy()
    # singular values of the covariance-aligned core (same randomised algorithm, same Omega)
    assert np.allclose(sing, s_o, rtol=1e-9, atol=1e-12 * s_o[0])
    # the shared correction of every module: A_i B (sign-free)
    row = 0
    for O in outs:
        P, P_o = A[row:row + O] @ B, A_o[row:row + O] @ B_o
        assert np.linalg.norm(P - P_o) <= 1e-8 * np.linalg.norm(P_o)
        row += O
    # the weighted objective it minimises is the oracle's
    obj = np.linalg.norm((E - A @ B) @ Sh) ** 2
    obj_o = np.linalg.norm((E - A_o @ B_o) @ Sh) ** 2
    assert obj == pytest.approx(obj_o, rel=1e-9)
    # energy capture: the captured fraction of ||E Sx^{1/2}||_F^2
    ew2 = np.linalg.norm(E @ Sh) ** 2
    assert float(gec.cpu()[0]) == pytest.approx(float(np.sum(s_o ** 2) / ew2), rel=1e-9)
    # fp16 factors are the float64 ones rounded once
    assert np.array_equal(A16.cpu().numpy(), A.astype(np.float16))
    assert np.array_equal(B16.cpu().numpy(), B.astype(np.float16))


def test_group_solve_factors_drive_the_forward():
    """The GPU-solved fp16 factors in the corrected forward (tiny Q/K/V config:
    d = 256, 4 outlier columns x10, r = 16, T = 8) match the oracle forward with
    the same factors, and the correction shrinks the covariance-weighted error."""
    import torch
    from helpers import check
    d, outs, r, p, q = 256, [256, 256, 256], 16, 16, 2
    mods, E, Sh, Shp, Om, dev = _case(d, outs, r, p, synth.ALPHA_QKV, seed=0, outlier_cols=4)
    _, _, _, _, A16, B16 = glowq.group_solve(dev["Ws"], dev["packs"], dev["Sh"], dev["Shp"], r, p, q, dev["Om"])
    As = torch.split(A16, outs)
    qm = [glowq.QModule(pk[0], pk[1], pk[2], A.contiguous()) for pk, A in zip(dev["packs"], As)]
    X = synth.activations(8, d, synth.ALPHA_QKV, seed=0, basis=synth.orthogonal_basis(d, seed=0))
    Ys, _ = glowq.group_forward(qm, B16, torch.from_numpy(X).cuda())
    Bb = synth.bits(B16.cpu().numpy())
    refs, _ = oracle.group_forward([(m.q, m.s, m.z, synth.bits(A.cpu().numpy())) for m, A in zip(mods, As)], Bb,
                                   synth.bits(X))
    for Y, ref in zip(Ys, refs):
        check(Y.cpu().numpy().astype(np.float64), ref)
    AB = np.vstack([A.cpu().numpy().astype(np.float64) for A in As]) @ B16.cpu().numpy().astype(np.float64)
    assert np.linalg.norm((E - AB) @ Sh) < 0.95 * np.linalg.norm(E @ Sh)


def test_group_solve_reports_a_rank_deficient_error():
    """Weights already on their INT4 grid give E_cat = 0: the orthonormalisation
    meets a zero pivot and the device status reports GLOWQ_ERR_NUMERIC."""
    import torch
    d, outs, r, p = 256, [128, 128], 8, 8
    mods, _, Sh, Shp, Om, dev = _case(d, outs, r, p, 1.19, seed=3)
    Ws = [torch.from_numpy(oracle.f16_bits_to_f64(oracle.dequant_int4(m.q, m.s, m.z, d)).astype(np.float32)).cuda()
          for m in mods]
    glowq.group_solve(Ws, dev["packs"], dev["Sh"], dev["Shp"], r, p, 1, dev["Om"])
    assert glowq.device_status() == 7
    assert glowq.device_status() == 0
