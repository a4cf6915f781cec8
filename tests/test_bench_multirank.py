"""The multi-rank host logic of bench.py on two gloo ranks (CPU): per-rank workloads, the
maximum of the timings over ranks, and the whole-job throughput."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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
        import bench
        from post_weight_quantization_guided_b200 import workloads as wl
        layer = bench.per_rank_layer(wl, rank)
        # rank r reports (r + 1, 10 - r) ms: the job's times are the maxima (2, 10)
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], world, torch.device("cpu"))
        dist.barrier()
        out[rank] = (layer.seed, layer.x_seed, layer.d_in, layer.d_out, got[0], got[1])
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        assert res[r][4] == 2.0 and res[r][5] == 10.0    # both ranks see the maxima
    assert res[0][2:4] == res[1][2:4]                     # same shapes
    assert res[0][0] != res[1][0] and res[0][1] != res[1][1]  # different draws


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(2, 4096, 20.0) == pytest.approx(2 * 4096 / 0.02)
    assert bench.job_throughput(1, 4096, 20.0) == pytest.approx(4096 / 0.02)
