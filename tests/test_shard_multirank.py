"""Several layers across ranks (post_weight_quantization_guided_b200.shard): the plan, and two
gloo ranks on CPU whose gathered (C, Q) equal one process's whole-layer result.

"GuidedQuant" (jinukkim.me blog), GuidedQuant section, third equation and the grouping sentence:
rows are independent given their group's Fisher block, so (layer, group) units can run anywhere.
The unit computation here is the oracle (CPU); on GPUs it is the library (shard.gpu_compute).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _layers(wl):
    return [wl.TINY,
            wl.scaled(wl.TINY, name="tiny_b", d_in=64, d_out=48, groups=3, m=4, seed=7,
                      x_seed=7),
            wl.scaled(wl.TINY, name="tiny_c", d_out=32, groups=2, m=16, iters=2, seed=8),
            wl.scaled(wl.TINY, name="tiny_d", d_in=32, d_out=8, groups=1, m=2, seed=9,
                      x_seed=9, g_kind="ones")]


def _oracle_compute(orc, wl):
    def compute(layer, g, row0, row1):
        X = wl.make_x(layer).double().numpy()
        G = wl.make_g(layer)
        Gg = None if G is None else G[:, row0:row1].double().numpy()
        W = wl.make_w(layer)[row0:row1].double().numpy()
        F = orc.fisher_full(X, Gg, 1)[0]
        C, Q, _, _ = orc.lnq_rows(F, W, layer.m, layer.iters)
        return torch.from_numpy(C.astype(np.float32)), torch.from_numpy(Q)
    return compute


def _expected(orc, wl, layers):
    out = []
    for layer in layers:
        X = wl.make_x(layer).double().numpy()
        G = wl.make_g(layer)
        W = wl.make_w(layer).double().numpy()
        F = orc.fisher_full(X, None if G is None else G.double().numpy(), layer.groups)
        R = layer.d_out // layer.groups
        Cs, Qs = [], []
        for g in range(layer.groups):
            C, Q, _, _ = orc.lnq_rows(F[g], W[g * R:(g + 1) * R], layer.m, layer.iters)
            Cs.append(C.astype(np.float32))
            Qs.append(Q)
        out.append((np.concatenate(Cs), np.concatenate(Qs)))
    return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as orc
        from post_weight_quantization_guided_b200 import shard
        from post_weight_quantization_guided_b200 import workloads as wl
        layers = _layers(wl)
        res, mine = shard.run(layers, rank, world, _oracle_compute(orc, wl), torch.device("cpu"))
        dist.barrier()
        out[rank] = ([(C.numpy(), Q.numpy()) for _, (C, Q) in sorted(res.items())],
                     [(u.layer, u.group) for u in mine])
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_gather_the_whole_layers(orc):
    from post_weight_quantization_guided_b200 import workloads as wl
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    layers = _layers(wl)
    # each rank ran a different, non-empty share, and together they cover every unit once
    mine0, mine1 = set(res[0][1]), set(res[1][1])
    assert mine0 and mine1 and not (mine0 & mine1)
    assert mine0 | mine1 == {(li, g) for li, l in enumerate(layers) for g in range(l.groups)}
    want = _expected(orc, wl, layers)
    for r in range(world):
        for li, (C, Q) in enumerate(res[r][0]):
            np.testing.assert_array_equal(Q, want[li][1])
            np.testing.assert_array_equal(C, want[li][0])


def test_plan_covers_every_unit_once_and_balances():
    sys.path.insert(0, ROOT)
    from post_weight_quantization_guided_b200 import shard
    from post_weight_quantization_guided_b200 import workloads as wl
    layers = wl.decoder_block(16)
    units = shard.units_of(layers)
    assert len(units) == 28
    for world in (1, 2, 3, 4, 8, 40):
        a = shard.plan(layers, world)
        assert a == shard.plan(layers, world)              # deterministic
        got = sorted((u.layer, u.group) for r in a for u in r)
        assert got == sorted((u.layer, u.group) for u in units)
        loads = [sum(u.cost for u in r) for r in a]
        total = sum(u.cost for u in units)
        # greedy largest-first bound: no rank exceeds the mean by more than one unit
        assert max(loads) <= total / world + max(u.cost for u in units) * (1 + 1e-12)
        if world > len(units):
            assert sum(1 for r in a if not r) == world - len(units)
    with pytest.raises(ValueError):
        shard.plan(layers, 0)


def test_one_rank_gather_needs_no_process_group():
    sys.path.insert(0, ROOT)
    from post_weight_quantization_guided_b200 import shard
    from post_weight_quantization_guided_b200 import workloads as wl
    layers = [wl.scaled(wl.TINY, d_in=16, d_out=6, groups=3, m=2)]

    def fake(layer, g, row0, row1):
        R = row1 - row0
        C = torch.arange(R * layer.m, dtype=torch.float32).view(R, layer.m) + 100 * g
        Q = (torch.arange(R * layer.d_in) % layer.m).to(torch.uint8).view(R, layer.d_in)
        return C, Q + g % 2

    res, mine = shard.run(layers, 0, 1, fake, torch.device("cpu"))
    C, Q = res[0]
    for g in range(3):
        Cg, Qg = fake(layers[0], g, 2 * g, 2 * g + 2)
        assert torch.equal(C[2 * g:2 * g + 2], Cg) and torch.equal(Q[2 * g:2 * g + 2], Qg)


def _main_rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from post_weight_quantization_guided_b200 import shard

    def fake(layer, g, row0, row1):
        R = row1 - row0
        return (torch.full((R, layer.m), float(g), dtype=torch.float32),
                torch.full((R, layer.d_in), g, dtype=torch.uint8))

    line, res = shard.main(["--bits", "3"], compute=fake, device=torch.device("cpu"))
    out[rank] = (line, [(float(C.sum()), int(Q.sum())) for _, (C, Q) in sorted(res.items())])


@pytest.mark.timeout(300)
def test_main_runs_the_decoder_block_on_two_gloo_ranks():
    """The command-line runner's host logic: the block's 28 units split over two ranks, the job
    time is the slower rank's, and both ranks hold every layer's gathered result."""
    from post_weight_quantization_guided_b200 import workloads as wl
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_main_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    layers = wl.decoder_block(8)
    want = [(float(sum(g * (l.d_out // l.groups) * l.m for g in range(l.groups))),
             sum(g * (l.d_out // l.groups) * l.d_in for g in range(l.groups))) for l in layers]
    for r in range(world):
        line, sums = res[r]
        assert line["units"] == 28 and line["ranks"] == 2
        assert line["rows"] == sum(l.d_out for l in layers)
        assert sums == want
    assert res[0][0]["ms"] == res[1][0]["ms"]


def _fisher_rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as orc
        from post_weight_quantization_guided_b200 import shard
        from post_weight_quantization_guided_b200 import workloads as wl
        layer = wl.TINY
        X = wl.make_x(layer).double()
        G = wl.make_g(layer).double()
        t0, t1 = shard.token_range(layer.n, rank, world)
        Fp = torch.from_numpy(orc.fisher_full(X[t0:t1].numpy(), G[t0:t1].numpy(), layer.groups))
        try:
            mine = shard.reduce_fisher(Fp.clone(), keep_groups=True).numpy()
        except ValueError:      # raised on every rank alike, before any collective
            mine = None
        every = shard.reduce_fisher(Fp.clone())
        out[rank] = (every.numpy(), mine, (t0, t1))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_token_sharded_fisher_sums_to_the_whole(orc, world):
    """gloo ranks each build the tiny layer's four blocks over their own tokens with the oracle
    (with 3 ranks the 256 tokens do not split evenly). The all-reduce gives every rank the
    whole-token blocks; the reduce-scatter path gives each rank its own groups, and refuses a
    group count that does not split over the ranks."""
    from post_weight_quantization_guided_b200 import workloads as wl
    from post_weight_quantization_guided_b200 import shard
    layer = wl.TINY
    assert [shard.token_range(10, r, 3) for r in range(3)] == [(0, 4), (4, 7), (7, 10)]
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_fisher_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    F = orc.fisher_full(wl.make_x(layer).double().numpy(), wl.make_g(layer).double().numpy(),
                        layer.groups)
    spans = sorted(res[r][2] for r in range(world))
    assert spans[0][0] == 0 and spans[-1][1] == layer.n
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    tol = dict(rtol=1e-12, atol=1e-12 * np.abs(F).max())
    per = layer.groups // world
    for r in range(world):
        np.testing.assert_allclose(res[r][0], F, **tol)
        if layer.groups % world == 0:
            np.testing.assert_allclose(res[r][1], F[r * per:(r + 1) * per], **tol)
        else:
            assert res[r][1] is None
