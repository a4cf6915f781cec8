"""One small run of the whole path for profiler captures.

    python -m post_weight_quantization_guided_b200.profile_case --workload q_proj --rows 1024

builds the guided Fisher blocks, initialises the codebooks and runs `--iters` LNQ iterations plus
the objective on a named synthetic workload, optionally with fewer output rows (`--rows`, a
multiple of the group count) so that a capture stays small. It prints the objective's sum so that
a run can be checked to have completed.

With `--fisher-only` it stops after building the blocks twice (`--tokens` shortens n). With
`--lut N` it then packs the codes and runs the lookup-table GEMV N times on one activation
vector (the codes cycled through enough copies that they come from HBM). With `--diag N` it runs
N calls of LNQ with diagonal Fisher blocks (the diagonals of the blocks just built, `--iters`
iterations each, from the initial codebooks). With `--ganq N` it runs N calls of the GANQ-style
comparison solver (`--iters` iterations each, from the initial codebooks).
"""
from __future__ import annotations

import argparse

import torch

from . import binding as api
from . import workloads as wl

WORKLOADS = {"tiny": wl.TINY, "q_proj": wl.Q_PROJ, "down_proj": wl.DOWN_PROJ, "up_proj": wl.UP_PROJ,
             "block_q": wl.decoder_block(16)[0], "block_gate": wl.decoder_block(16)[4],
             "block_down": wl.decoder_block(16)[6]}


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="q_proj", choices=sorted(WORKLOADS))
    ap.add_argument("--rows", type=int, default=0, help="output rows (default: the workload's)")
    ap.add_argument("--iters", type=int, default=1)
    ap.add_argument("--lut", type=int, default=0, help="lookup-table GEMV calls after the run")
    ap.add_argument("--diag", type=int, default=0,
                    help="calls of LNQ with diagonal Fisher blocks after the run")
    ap.add_argument("--ganq", type=int, default=0,
                    help="calls of the GANQ-style comparison solver after the run")
    ap.add_argument("--fisher-only", action="store_true",
                    help="build the Fisher blocks (twice) and stop")
    ap.add_argument("--tokens", type=int, default=0, help="calibration tokens (default: the workload's)")
    ap.add_argument("--m", type=int, default=0, help="codewords per row (default: the workload's)")
    args = ap.parse_args(argv)
    layer = WORKLOADS[args.workload]
    if args.rows:
        if args.rows % layer.groups:
            raise SystemExit(f"--rows must be a multiple of {layer.groups}")
        layer = wl.scaled(layer, d_out=args.rows)
    if args.tokens:
        layer = wl.scaled(layer, n=args.tokens)
    if args.m:
        layer = wl.scaled(layer, m=args.m)
    dev = torch.device("cuda:0")
    X, G, W = wl.make_layer(layer, dev)
    F = api.lnq_build_fisher(X, G, layer.groups)
    if args.fisher_only:
        api.lnq_build_fisher(X, G, layer.groups, F=F)
        torch.cuda.synchronize()
        print(f"{layer.name} n={layer.n} fisher sum(diag)={float(torch.diagonal(F, dim1=1, dim2=2).sum()):.6e}")
        return
    C, Q = api.lnq_init_codebook(W, layer.m)
    J = torch.empty(layer.d_out, dtype=torch.float64, device=dev)
    st = torch.empty(layer.d_out, dtype=torch.int32, device=dev)
    api.lnq_quantize_rows(F, W, layer.m, args.iters, C, Q, J, st)
    torch.cuda.synchronize()
    print(f"{layer.name} rows={layer.d_out} iters={args.iters} sum(J)={float(J.sum()):.6e}")
    if args.lut:
        bits = layer.m.bit_length() - 1
        P = api.lnq_pack_codes(Q, bits)
        Ps = [P.clone() for _ in range(max(2, int(3 * 126e6 / (P.numel() * 4)) + 1))]
        x = torch.randn(1, layer.d_in, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
        y = torch.empty(1, layer.d_out, device=dev)
        for k in range(args.lut):
            api.lnq_lut_gemv(x, Ps[k % len(Ps)], C, layer.d_in, y=y)
        torch.cuda.synchronize()
        print(f"lut_gemv calls={args.lut} sum(y)={float(y.sum()):.6e}")
    if args.diag:
        Fd = torch.diagonal(F, dim1=1, dim2=2).contiguous()
        C0, Q0 = api.lnq_init_codebook(W, layer.m)
        for _ in range(args.diag):
            C.copy_(C0)
            Q.copy_(Q0)
            api.lnq_quantize_rows_diag(Fd, W, layer.m, args.iters, C, Q, J, st)
        torch.cuda.synchronize()
        print(f"lnq_diag calls={args.diag} iters={args.iters} sum(J)={float(J.sum()):.6e}")
    if args.ganq:
        C0, Q0 = api.lnq_init_codebook(W, layer.m)
        for _ in range(args.ganq):
            C.copy_(C0)
            Q.copy_(Q0)
            api.lnq_ganq_rows(F, W, layer.m, args.iters, C, Q, J, st)
        torch.cuda.synchronize()
        print(f"ganq calls={args.ganq} iters={args.iters} sum(J)={float(J.sum()):.6e}")


if __name__ == "__main__":
    main()
