"""Measure work shapes for the decode kernel and part counts for the
small-batch k-split on the GPU at hand, for given module shapes.

The library picks a decode work shape (rt 16-row tiles and kw splits of d per
CTA, kc CTAs per cluster, ring depth) from a cost model, or from its measured
table for the LLaMA-family shapes; the small-batch path (16 < T <= 64) picks
its number of parts S from a fitted cost model.  This tool times every legal
choice through the library's tuning overrides (GLOWQ_DECODE_SHAPE,
GLOWQ_SPLIT_S) as the average call of a CUDA graph of back-to-back calls over
weight replicas larger than L2, and prints the best choices next to the
library's own.  A table line is printed for each decode case where the best
shape beats the library's pick by the margin, in the form of the library's
table entries (row tiles, d, token class, rt, kw, kc, stages).

    python -m rank_error_correction_b200.tune --outs 4096 --d 4096 --tokens 1,4,16
    python -m rank_error_correction_b200.tune --outs 4096,4096,4096 --d 4096 --tokens 32,64 --split

Weights, factors (r = 64 by default) and activations are seeded random draws
of the library's synthetic generators; timings do not depend on their values.
Needs a CUDA device.
"""
from __future__ import annotations

import argparse
import os

L2_BYTES = 126 * 1024 * 1024


def _unit(outs, d, r, sub, device):
    from rank_error_correction_b200 import glowq, synth
    mods = []
    for j, O in enumerate(outs):
        W = synth.device_weights(O, d, 0, sub=sub + j, device=device)
        q, s, z = glowq.pack_int4(W)
        del W
        mods.append(glowq.QModule(q, s, z))
    B = None
    if r > 0:
        As, B = synth.device_factors(outs, d, r, 0, sub=sub, device=device)
        for m, A in zip(mods, As):
            m.A = A
    return mods, B


def _chain_us(reps, X, T, r, d, outs, calls=48):
    """Average call of a graph of back-to-back calls over the replicas."""
    import torch
    from rank_error_correction_b200 import glowq
    dev = X.device
    Ys = [torch.empty((T, O), dtype=torch.float16, device=dev) for O in outs]
    R = torch.empty((T, max(r, 8)), dtype=torch.float16, device=dev) if r > 0 else None
    ws = torch.zeros(max(glowq.workspace_bytes_for(T, r, d, outs), 16), dtype=torch.uint8, device=dev)

    def call(i):
        mods, B = reps[i % len(reps)]
        if len(mods) > 1:
            glowq.group_forward(mods, B, X, Ys=Ys, R_out=R, workspace=ws)
        else:
            glowq.solo_forward(mods[0], B, X, Y=Ys[0], workspace=ws)

    st = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(st):
        for i in range(2):
            call(i)
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for i in range(calls):
            call(i)
    with torch.cuda.stream(st):
        g.replay()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(2):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            t0.record()
            g.replay()
            t1.record()
        torch.cuda.synchronize()
        best = min(best, t0.elapsed_time(t1) * 1e3 / calls)
    del g
    status = glowq.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    return best


def decode_shapes(d: int):
    """Every (rt, kw, kc, stages) the decode kernel accepts for input width d."""
    ngroups = d // 128
    out = []
    for stages in (4, 8):
        for rt in range(1, 16):
            for kw in range(1, 16 // rt + 1):
                if rt * kw <= 15 and ngroups >= kw:
                    out.append((rt, kw, 1, stages))
            for kc in range(2, 9):
                if rt <= 15 and kc <= ngroups:
                    out.append((rt, 1, kc, stages))
    return out


def token_class(T: int) -> int:
    return 0 if T == 1 else 1 if T <= 5 else 2 if T <= 8 else 3 if T <= 12 else 4


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--outs", required=True, help="output features of the unit's modules, comma separated")
    ap.add_argument("--d", type=int, required=True, help="input features")
    ap.add_argument("--tokens", default="1,4,16", help="token counts, comma separated")
    ap.add_argument("--rank", type=int, default=64)
    ap.add_argument("--split", action="store_true", help="sweep the k-split parts S (16 < T <= 64) instead")
    ap.add_argument("--margin", type=float, default=0.03, help="gain over the library's pick that prints a table line")
    args = ap.parse_args(argv)
    import torch
    from rank_error_correction_b200 import synth
    device = torch.device("cuda")
    outs = [int(o) for o in args.outs.split(",")]
    d, r = args.d, args.rank
    bytes_1 = sum(O * d // 2 + O * (d // 128) * 3 for O in outs)
    n_rep = max(2, min(8, -(-2 * L2_BYTES // bytes_1)))
    reps = [_unit(outs, d, r, 1000 * i, device) for i in range(n_rep)]
    tiles = sum(O // 16 for O in outs)
    for T in (int(t) for t in args.tokens.split(",")):
        X = synth.device_activations(T, d, 0, sub=700, device=device)
        key = "GLOWQ_SPLIT_S" if args.split else "GLOWQ_DECODE_SHAPE"
        os.environ.pop("GLOWQ_SPLIT_S", None)
        os.environ.pop("GLOWQ_DECODE_SHAPE", None)
        lib = _chain_us(reps, X, T, r, d, outs)
        cands = [(S,) for S in range(1, 9)] if args.split else decode_shapes(d)
        res = []
        for c in cands:
            os.environ[key] = ",".join(map(str, c))
            try:
                res.append((_chain_us(reps, X, T, r, d, outs), c))
            except RuntimeError as e:
                print(f"  {c}: {e}")
        os.environ.pop(key, None)
        res.sort()
        top = " ".join(f"{c}={us:.2f}" for us, c in res[:6])
        print(f"T={T}: library {lib:.2f} us; best {top}", flush=True)
        if not args.split and res and res[0][0] < (1.0 - args.margin) * lib:
            rt, kw, kc, st = res[0][1]
            print(f"    {{{tiles}, {d}, {token_class(T)}, {rt}, {kw}, {kc}, {st}}},")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
