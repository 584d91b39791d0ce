"""Guard bands around every buffer the forward calls write: the workspace, R
and Y are carved out of larger allocations whose margins hold a byte pattern;
after decode (T = 1, 16), small-batch (T = 40, k-split) and prefill (T = 300)
calls, group and solo, the margins must be untouched and the results must
still match the oracle.  A kernel that writes past a buffer's end (or before
its start) fails here even when its own output looks right.
Pages: papernotes.org GlowQ summary, key design 4 (R = X B^T once per group,
y_i = W_i^(q) X + A_i R).
"""
import numpy as np
import pytest

import oracle
from rank_error_correction_b200 import build, glowq, synth

from helpers import attach_random_factors, check, make_modules, normwise, to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096            # bytes of margin on each side (keeps 256-byte alignment)
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    glowq.lib()
    yield
    assert glowq.device_status() == 0


def _guarded(nbytes, fill_body=None):
    """A uint8 device buffer of nbytes inside two GUARD-byte margins of PATTERN."""
    import torch
    buf = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    if fill_body is not None:
        buf[GUARD:GUARD + nbytes].fill_(fill_body)
    return buf, buf[GUARD:GUARD + nbytes]


def _margins_intact(buf, nbytes):
    import torch
    head, tail = buf[:GUARD], buf[GUARD + nbytes:]
    return bool(torch.all(head == PATTERN)) and bool(torch.all(tail == PATTERN))


@pytest.mark.parametrize("T", [1, 16, 40, 300])
def test_group_and_solo_write_inside_their_buffers(T):
    import torch
    d, outs, r = 2048, [256, 128], 32          # T = 40 takes the k-split at this d
    mods = make_modules(d, outs, seed=1200 + T)
    B = attach_random_factors(mods, d, r, seed=1200 + T)
    X = synth.activations(T, d, synth.ALPHA_QKV, seed=1200 + T)
    dm = to_dev(mods)
    Bd, Xd = torch.from_numpy(B).cuda(), torch.from_numpy(X).cuda()
    if T == 40:
        assert glowq.workspace_bytes_for(T, r, d, outs) > glowq.workspace_bytes(T, r)

    # workspace: zero region zero, the rest a pattern the kernels may overwrite
    wsn = max(glowq.workspace_bytes_for(T, r, d, outs), glowq.workspace_bytes_for(T, r, d, outs[1:]))
    wbuf, ws = _guarded(wsn, fill_body=0x5A)
    ws[:4096].zero_()
    # R and Y inside guarded allocations
    rbuf, rb = _guarded(T * r * 2)
    R = rb.view(torch.float16).view(T, r)
    ybufs, Ys = [], []
    for O in outs:
        yb, body = _guarded(T * O * 2)
        ybufs.append(yb)
        Ys.append(body.view(torch.float16).view(T, O))
    glowq.group_forward(dm, Bd, Xd, Ys=Ys, R_out=R, workspace=ws)
    sbuf, sb = _guarded(T * outs[1] * 2)
    Ysolo = sb.view(torch.float16).view(T, outs[1])
    glowq.solo_forward(dm[1], Bd, Xd, Y=Ysolo, workspace=ws)
    torch.cuda.synchronize()

    assert _margins_intact(wbuf, wsn), "workspace margin overwritten"
    assert _margins_intact(rbuf, T * r * 2), "R margin overwritten"
    for yb, O in zip(ybufs, outs):
        assert _margins_intact(yb, T * O * 2), "Y margin overwritten"
    assert _margins_intact(sbuf, T * outs[1] * 2), "solo Y margin overwritten"
    assert int(ws[:4096].count_nonzero()) == 0

    refs, R_ref = oracle.group_forward([(m.q, m.s, m.z, synth.bits(m.A)) for m in mods], synth.bits(B),
                                       synth.bits(X))
    assert normwise(R.cpu().numpy().astype(np.float64), R_ref) < 1e-3
    for Y, ref in zip(Ys, refs):
        check(Y.cpu().numpy().astype(np.float64), ref)
    check(Ysolo.cpu().numpy().astype(np.float64), refs[1])
