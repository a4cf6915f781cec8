"""Several layers across ranks: every (linear, Fisher group) pair is one unit of independent work.

"GuidedQuant" (jinukkim.me blog), GuidedQuant section, third equation and the sentence after it:
the objective is a sum over layers l and output rows j of per-row terms, and rows share a Fisher
block only inside their group. So a unit needs X of its layer, the G columns and W rows of its
group, and nothing from any other unit: ranks run their units without a collective, and one
all-gather of the results (codebooks C and codes Q) ends the job.

  plan(layers, world)           units assigned to ranks, largest first to the least-loaded rank
                                (ties to the lower rank); every rank computes the same plan
  run(layers, rank, world, compute, group=None)
                                runs this rank's units through `compute`, then all-gathers every
                                unit's (C, Q) into whole-layer tensors on every rank
  gpu_compute(lnq, wl, device)  the unit computation on the GPU library: guided Fisher block of the
                                group (its G columns, one group), initial codebook, LNQ iterations
  token_range, reduce_fisher    the alternative for very large n: each rank builds the blocks
                                over its own tokens, one all-reduce (or reduce-scatter of the
                                groups) sums them
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Tuple

import torch
import torch.distributed as dist


@dataclasses.dataclass(frozen=True)
class Unit:
    layer: int        # index into the layer list
    group: int        # Fisher group within the layer
    row0: int         # first output row of the group
    row1: int         # one past the last
    cost: float       # flop estimate used for balancing


def unit_cost(layer) -> float:
    """Flops of one group: its Fisher block (n d_in (d_in + 1) unique-entry flops) plus the class-
    binned product of every LNQ iteration (2 d_in^2 m flops per row), which dominate the step."""
    R = layer.d_out // layer.groups
    return (float(layer.n) * layer.d_in * (layer.d_in + 1)
            + 2.0 * layer.d_in * layer.d_in * layer.m * R * layer.iters)


def units_of(layers) -> List[Unit]:
    out = []
    for li, layer in enumerate(layers):
        R = layer.d_out // layer.groups
        c = unit_cost(layer)
        for g in range(layer.groups):
            out.append(Unit(li, g, g * R, (g + 1) * R, c))
    return out


def plan(layers, world: int) -> List[List[Unit]]:
    """Longest-processing-time assignment: units by decreasing cost (then layer, group), each to
    the rank with the least load so far (the lowest rank among equals). Deterministic, so every
    rank derives the same plan without communication. Each rank's list is in assignment order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(units_of(layers), key=lambda u: (-u.cost, u.layer, u.group))
    load = [0.0] * world
    out: List[List[Unit]] = [[] for _ in range(world)]
    for u in order:
        r = min(range(world), key=lambda k: (load[k], k))
        out[r].append(u)
        load[r] += u.cost
    return out


def _unit_bytes(layers, u: Unit) -> int:
    layer = layers[u.layer]
    return (u.row1 - u.row0) * (4 * layer.m + layer.d_in)


def _pack(layers, units, results, device) -> torch.Tensor:
    parts = []
    for u in units:
        C, Q = results[(u.layer, u.group)]
        parts.append(C.contiguous().view(torch.uint8).reshape(-1).to(device))
        parts.append(Q.contiguous().reshape(-1).to(device))
    if not parts:
        return torch.empty(0, dtype=torch.uint8, device=device)
    return torch.cat(parts)


def gather(layers, assignment, results, device, group=None):
    """All-gathers the units' (C, Q) of every rank. Returns, for every layer, (C [d_out][m] fp32,
    Q [d_out][d_in] uint8) on `device`. Buffer sizes follow from the plan, so one all_gather of
    equal-length byte buffers (padded to the largest rank) is the only exchange."""
    world = len(assignment)
    sizes = [sum(_unit_bytes(layers, u) for u in units) for units in assignment]
    mx = max(sizes) if sizes else 0
    rank = dist.get_rank(group) if world > 1 else 0
    mine = _pack(layers, assignment[rank], results, device)
    buf = torch.zeros(mx, dtype=torch.uint8, device=device)
    buf[:mine.numel()] = mine
    if world > 1:
        bufs = [torch.empty(mx, dtype=torch.uint8, device=device) for _ in range(world)]
        dist.all_gather(bufs, buf, group=group)
    else:
        bufs = [buf]
    out = {li: (torch.empty((layer.d_out, layer.m), dtype=torch.float32, device=device),
                torch.empty((layer.d_out, layer.d_in), dtype=torch.uint8, device=device))
           for li, layer in enumerate(layers)}
    for r, units in enumerate(assignment):
        off = 0
        for u in units:
            layer = layers[u.layer]
            R = u.row1 - u.row0
            nc = R * layer.m * 4
            C, Q = out[u.layer]
            C[u.row0:u.row1] = bufs[r][off:off + nc].view(torch.float32).view(R, layer.m)
            off += nc
            nq = R * layer.d_in
            Q[u.row0:u.row1] = bufs[r][off:off + nq].view(R, layer.d_in)
            off += nq
    return out


def run(layers, rank: int, world: int,
        compute: Callable[[object, int, int, int], Tuple[torch.Tensor, torch.Tensor]],
        device, group=None):
    """This rank's units through compute(layer, group, row0, row1) -> (C rows, Q rows), then the
    all-gather. Returns (per-layer (C, Q) on `device`, this rank's units)."""
    assignment = plan(layers, world)
    results: Dict[Tuple[int, int], Tuple[torch.Tensor, torch.Tensor]] = {}
    # layer order, so that units of one layer (and layers of one X draw) run back to back
    for u in sorted(assignment[rank], key=lambda u: (u.layer, u.group)):
        results[(u.layer, u.group)] = compute(layers[u.layer], u.group, u.row0, u.row1)
    return gather(layers, assignment, results, device, group), assignment[rank]


def token_range(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Rank `rank`'s contiguous slice [t0, t1) of n tokens (the first n % world ranks get one
    more)."""
    base, extra = divmod(n, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def reduce_fisher(F_partial: torch.Tensor, keep_groups: bool = False, group=None) -> torch.Tensor:
    """Token-sharded Fisher build, the exchange step: every rank built F [groups][d][d] over its
    own tokens (s_g[t] depends only on token t's gradient row, so the blocks are sums over tokens
    and the partial blocks add up to the whole). Sums them in place on every rank (all-reduce), or
    with keep_groups=True returns only this rank's share of the groups (reduce-scatter over the
    group dimension; groups must be a multiple of the world size)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return F_partial
    if not keep_groups:
        dist.all_reduce(F_partial, group=group)
        return F_partial
    groups = F_partial.shape[0]
    if groups % world != 0:
        raise ValueError(f"{groups} groups do not split over {world} ranks")
    out = torch.empty((groups // world,) + tuple(F_partial.shape[1:]), dtype=F_partial.dtype,
                      device=F_partial.device)
    if dist.get_backend(group) == "nccl":
        dist.reduce_scatter_tensor(out, F_partial.contiguous(), group=group)
    else:   # backends without reduce-scatter: the full sum, then this rank's slice
        dist.all_reduce(F_partial, group=group)
        r = dist.get_rank(group)
        out.copy_(F_partial[r * (groups // world):(r + 1) * (groups // world)])
    return out


def gpu_compute(lnq, wl, device):
    """compute() for run(): the unit on the GPU library. X is drawn once per distinct draw, G and
    W once per layer, each kept while consecutive units use it; the group's G columns and W rows
    are copied out contiguous. The group's block is built with groups = 1 over those columns,
    which is the group's F_g of the whole layer (s_g averages only the group's columns); with
    all-ones gradients (G is None) every group's block is X^T X."""
    xs, gw = {}, {}

    def compute(layer, g, row0, row1):
        xkey = (layer.x_seed, layer.x_kind, layer.n, layer.d_in)
        if xkey not in xs:
            xs.clear()
            xs[xkey] = wl.make_x(layer, device)
        if layer.name not in gw:
            gw.clear()
            gw[layer.name] = (wl.make_g(layer, device), wl.make_w(layer, device))
        X = xs[xkey]
        G, W = gw[layer.name]
        Gg = None if G is None else G[:, row0:row1].contiguous()
        Wg = W[row0:row1].contiguous()
        F = lnq.lnq_build_fisher(X, Gg, 1)
        del Gg
        C, Q = lnq.lnq_init_codebook(Wg, layer.m)
        lnq.lnq_quantize_rows(F, Wg, layer.m, layer.iters, C, Q)
        return C, Q

    return compute


def main(argv=None, compute=None, device=None, backend=None):
    """Quantises the decoder block: one process per GPU (torchrun sets RANK and WORLD_SIZE), each
    running its units, then the all-gather. Rank 0 prints one JSON line: rows quantised, the time
    of the slowest rank (CUDA events on GPUs, wall clock on CPU) and rows per second.
    compute / device / backend: overrides for running the host logic without a GPU."""
    import argparse
    import json
    import os
    import time

    ap = argparse.ArgumentParser(description=main.__doc__)
    ap.add_argument("--bits", type=int, default=4, choices=(1, 2, 3, 4))
    args = ap.parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    from . import workloads as wl
    if device is None:
        local = int(os.environ.get("LOCAL_RANK", "0"))
        device = torch.device("cuda", local)
        torch.cuda.set_device(device)
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend or ("nccl" if device.type == "cuda" else "gloo"))
    try:
        if compute is None:
            import post_weight_quantization_guided_b200 as lnq
            compute = gpu_compute(lnq, wl, device)
        layers = wl.decoder_block(1 << args.bits)
        if world > 1:
            dist.barrier()
        if device.type == "cuda":
            torch.cuda.synchronize(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
        t0 = time.perf_counter()
        out, mine = run(layers, rank, world, compute, device)
        if device.type == "cuda":
            e1.record()
            torch.cuda.synchronize(device)
            ms = e0.elapsed_time(e1)
        else:
            ms = (time.perf_counter() - t0) * 1e3
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        rows = sum(layer.d_out for layer in layers)
        line = {"workload": f"decoder block, {len(layers)} linears, n = {layers[0].n}, "
                            f"m = {1 << args.bits}",
                "ranks": world, "units": len(units_of(layers)), "rows": rows,
                "ms": float(t.item()), "rows_per_s": rows / (float(t.item()) / 1e3)}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return line, out
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
