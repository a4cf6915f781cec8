"""The bench's work accounting on the CPU: the per-launch unit counts behind every roofline
fraction, checked against counts taken by enumeration, and the roofline and traffic helpers.

The unit counts follow the hot path's steps: the guided Fisher blocks ("GuidedQuant" blog post,
GuidedQuant section, third equation: one symmetric d x d block per group, each unique entry a sum
over n tokens) and LNQ's codebook step (LNQ section: M = P^T F P, formed from the upper triangle
of the symmetric F).
"""
import itertools
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from post_weight_quantization_guided_b200 import workloads as wl  # noqa: E402


def _layer(d_in, d_out, n=64, groups=2, m=16):
    return wl.scaled(wl.Q_PROJ, d_in=d_in, d_out=d_out, n=n, groups=groups, m=m)


@pytest.mark.parametrize("d", [1, 3, 8, 37])
def test_fisher_flops_count_every_unique_entry(d):
    L = _layer(d, 8, n=5, groups=3)
    unique = sum(1 for i, k in itertools.product(range(d), repeat=2) if i <= k)
    # one multiply and one add per token for each unique entry of each group's block
    assert bench.algorithmic_work(L, 16, "fisher_syrk") == (3 * unique * 2 * 5, "flop")


@pytest.mark.parametrize("d", [2, 5, 64])
def test_codebook_lane_ops_are_half_the_square_per_row(d):
    L = _layer(d, 12)
    work, unit = bench.algorithmic_work(L, 16, "lnq_mgemm")
    assert unit == "lane_op"
    # one add per ordered pair (i, k) with the symmetry of F: d^2 / 2 per row
    pairs = sum(1 for _ in itertools.product(range(d), repeat=2))
    assert work == pytest.approx(12 * pairs / 2)


@pytest.mark.parametrize("d", [64, 256, 300, 4096, 11008])
def test_executed_product_flops_enumerate_the_block_triangle(d):
    L = _layer(d, 4, m=8)
    nk = -(-d // 64)            # K blocks of 64 coordinates
    npair = -(-d // 256)        # pair blocks of 256 coordinates
    kblocks = 0
    for ip in range(npair):
        # the tile of pair block ip runs over the K blocks from its own diagonal block on
        kblocks += sum(1 for kb in range(nk) if kb >= 4 * ip)
    want = 4 * 2.0 * (2 * 8) * 256 * 64 * kblocks   # rows x 2 flops x (2 pieces x m) x M x K
    assert bench.executed_tensor_flops(L, 8, "lnq_mgemm") == pytest.approx(want)
    # the residual product: three piece products of every 256-coordinate block with all of F
    want_r = 4 * 2.0 * 3 * (npair * 256) * (nk * 64)
    assert bench.executed_tensor_flops(L, 8, "lnq_residual_gemm") == pytest.approx(want_r)


def test_sweep_work_adds_the_measured_tail():
    L = _layer(100, 10, m=4)
    assert bench.algorithmic_work(L, 4, "lnq_sweep", sweep_tail=1234.0) == (
        1234.0 + 3 * 4 * 100 * 10, "lane_op")
    assert bench.algorithmic_work(L, 4, "lnq_sweep")[0] == 3 * 4 * 100 * 10


def test_launch_counts_per_call():
    L = _layer(64, 8)
    assert bench.launches_per_call("lnq_mgemm", L, 5) == 5
    assert bench.launches_per_call("lnq_sweep", L, 5) == 5
    assert bench.launches_per_call("lnq_residual_gemm", L, 5) == 7   # -F w, 5 sweeps, objective
    assert bench.launches_per_call("fisher_syrk", L, 5) == 1
    ones = wl.scaled(L, g_kind="ones")
    assert bench.launches_per_call("token_stats", ones, 5) == 0
    assert bench.launches_per_call("token_stats", L, 5) == 1


@pytest.mark.parametrize("source", ["measured", "fallback"])
def test_roofline_fractions_and_labels(source):
    peaks = {"hbm_gbs": 5000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
             "source": source}
    fp32 = {"sustained": 30.0, "burst": 32.0}
    r = bench.roofline(2.5e9, "byte", 1.0, peaks, fp32)        # 2.5 GB in 1 ms
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(2500.0)
    assert r["frac"] == pytest.approx(0.5) and f"of {source}" in r["peak_kind"]
    r = bench.roofline(7e11, "flop", 1.0, peaks, fp32)         # 700 TFLOP/s
    assert r["peak"] == 1400.0 and r["frac"] == pytest.approx(0.5)
    assert "sustained" in r["peak_kind"] and f"of {source}" in r["peak_kind"]
    burst_only = {k: v for k, v in peaks.items() if k != "bf16_tflops_sustained"}
    r = bench.roofline(8e11, "flop", 1.0, burst_only, fp32)
    assert r["peak"] == 1600.0 and "burst" in r["peak_kind"]
    r = bench.roofline(1.5e10, "lane_op", 1.0, peaks, fp32)    # 15 T lane-ops/s
    assert r["bound"] == "alu" and r["frac"] == pytest.approx(0.5)


def test_traffic_needs_the_measured_source(monkeypatch):
    L = wl.decoder_block(16)[0]
    rec = dict(bench.TRAFFIC["lnq_mgemm"])
    per_row = rec["bytes_per_row"]["4096/4096/16"]
    got = bench.measured_traffic("lnq_mgemm", [(L, 3)])
    path = os.path.join(bench.ROOT, "post_weight_quantization_guided_b200", "csrc", rec["source"])
    import hashlib
    same = hashlib.sha256(open(path, "rb").read()).hexdigest() == rec["sha256"]
    assert (got == pytest.approx(per_row * L.d_out)) if same else got is None
    changed = dict(rec, sha256="0" * 64)
    monkeypatch.setitem(bench.TRAFFIC, "lnq_mgemm", changed)
    assert bench.measured_traffic("lnq_mgemm", [(L, 3)]) is None
    assert bench.measured_traffic("lnq_sweep", [(L, 3)]) is None


def test_cpu_baseline_leg_runs_on_a_small_block(orc):
    """The bench's oracle leg on CPU tensors of a scaled block: it samples Fisher tiles and LNQ
    rows of the first and last layer and extrapolates to one step of every layer."""
    import numpy as np
    import torch
    blk = wl.decoder_block(16)
    layers = [wl.scaled(L, d_in=128 if L.d_in == 4096 else 160, d_out=32 if L.d_out == 4096 else 48,
                        n=128, iters=2) for L in blk]
    cache = {}

    def inputs(L):
        if L.name not in cache:
            cache[L.name] = wl.make_layer(L, torch.device("cpu"))
        return cache[L.name]

    F_small = {}
    for L in (layers[0], layers[-1]):
        X, G, _ = inputs(L)
        Gh = G[:, :L.rows_per_group].double().numpy()
        s = orc.group_scales(Gh, L.n, L.rows_per_group, 1)[0]
        Xh = X.double().numpy()
        F_small[L.name] = orc.fisher_block(Xh, Xh, s, 1.0)
    out = bench.cpu_baseline_block(layers, inputs, F_small, budget_s=0.2, threads=2)
    assert out["kind"] == "oracle" and out["cores"] == 2 and out["unit"] == bench.UNIT
    rows = 2 * sum(L.d_out for L in layers)
    secs = out["fisher_s_extrapolated"] + out["lnq_s_extrapolated"]
    assert secs > 0 and out["value"] == pytest.approx(rows / secs)
    assert np.isfinite(out["value"]) and "d_in=160" in out["sample"]
