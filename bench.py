"""Benchmark of the GuidedQuant + LNQ hot path on B200.

Headline workload: the seven linears of a Llama-2-7B-shaped decoder block (q, k, v, o 4096 x 4096;
gate, up 4096 -> 11008; down 11008 -> 4096), n = 131072 calibration tokens, 4 Fisher groups,
5 LNQ iterations, quantised at 4 bits (m = 16) and at 3 bits (m = 8). One step quantises the
whole block at both bit widths: per layer the guided Fisher build (s_g reduction, then the
tcgen05 SYRK with the diag(s_g) scaling fused into its operand load), then for each bit width the
codebook initialisation, 5 x (codebook step + assignment sweep) and the per-row objective. F does
not depend on the bit width, so each layer's F is built once and used by both.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--no-q-proj]

`value` is rows quantised per second over the whole step (both bit widths, Fisher build
included); the line also gives, per bit width, the end-to-end block time (the Fisher builds plus
that bit width's LNQ) and the LNQ-only rate d_out / (t_init + t_iterations) summed over layers.
With N > 1 (torchrun, one process per GPU) every rank quantises its own block (seeds offset per
rank): weak scaling, no collective on the data path. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = ("LNQ rows quantized/s per layer (guided Fisher build + init + LNQ iterations + "
          "objective)")
UNIT = "rows/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
FISHER_KERNELS = ("token_stats", "fisher_syrk")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


# ------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(device_index)
        self.ident = ident

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # the timed region starts once the sampler is producing samples
        t0 = time.time()
        while time.time() - t0 < 10.0:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 7:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[3 + k] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((float(r[2]) for r in rows
                                    if r[2].replace(".", "").isdigit()), default=None)}


# ------------------------------------------------------------------------------------------
# Algorithmic work per launch: the per-unit figure times the units one launch processes
# ------------------------------------------------------------------------------------------
def launches_per_call(kernel, layer, iters):
    """Launches of `kernel` made by one layer's Fisher build (Fisher kernels) or by one
    init + lnq_quantize_rows(iters, with J) call (LNQ kernels)."""
    guided = layer.g_kind != "ones"
    fixed = {"token_stats": 1 if guided else 0, "fisher_syrk": 1, "lnq_init": 1,
             "lnq_split_f16": 1, "lnq_objective": 1}
    per_iter = ("lnq_operand_image", "lnq_mgemm", "lnq_solve", "lnq_sweep")
    if kernel in fixed:
        return fixed[kernel]
    if kernel in per_iter:
        return iters
    if kernel in ("lnq_residual_scale", "lnq_residual_image", "lnq_residual_gemm"):
        return 2 + iters        # -F w once, u = F r before every sweep and for the objective
    return 0


def algorithmic_work(layer, m, kernel, sweep_tail=None):
    """(amount, unit) of one launch of `kernel` on `layer` at m codewords.

    sweep_tail: for lnq_sweep, the measured sum over moved coordinates of (d - i) per launch."""
    d, n, g, dout = layer.d_in, layer.n, layer.groups, layer.d_out
    if kernel == "fisher_syrk":
        # every unique entry of each symmetric block: 2 n flops for each of d(d+1)/2 entries
        return float(g) * n * d * (d + 1), "flop"
    if kernel == "token_stats":
        return 2.0 * n * (d + dout) + 4.0 * n * (g + 1), "byte"    # read X and G, write S and M
    if kernel == "lnq_init":
        return 4.0 * dout * d + dout * d + 4.0 * dout * m, "byte"  # read W, write Q and C
    ld = (d + 7) // 8 * 8
    if kernel in ("lnq_operand_image", "lnq_residual_image"):
        # write the right-operand image (256 columns x d coordinates x 2 bytes per row tile), read
        # Q (and W for the residual) once
        rt = 256 // m if kernel == "lnq_operand_image" else 128
        tiles = g * -(-(dout // g) // rt)
        reads = dout * d * (1.0 if kernel == "lnq_operand_image" else 5.0)
        return tiles * 256 * (-(-d // 64) * 64) * 2.0 + reads, "byte"
    if kernel == "lnq_split_f16":
        return 4.0 * g * d * d + 4.0 * g * d * ld, "byte"           # read F, write 2 fp16 pieces
    if kernel == "lnq_residual_scale":
        return 5.0 * dout * d, "byte"                               # read W and Q
    if kernel == "lnq_mgemm":
        # the codebook step's M = P^T F P: d^2 / 2 FADD per row with the symmetry of F
        return 0.5 * d * d * dout, "lane_op"
    if kernel == "lnq_residual_gemm":
        # u = F r for every row: a dense contraction of F with the residual columns, 2 d^2 flops
        # per row (executed as three fp16 piece products on tensor cores)
        return 2.0 * d * d * dout, "flop"
    if kernel == "lnq_solve":
        # read the binned partial sums (m x m per 128 coordinates), U and Q; write C
        halves = 2 * -(-d // 256)
        return dout * (halves * m * m * 4.0 + d * 5.0 + 4.0 * m), "byte"
    if kernel == "lnq_sweep":
        # the moves' updates of u (sum over moved coordinates of d - i FMA) plus the candidate
        # comparisons (3 m per coordinate)
        return float(sweep_tail or 0.0) + 3.0 * m * d * dout, "lane_op"
    if kernel == "lnq_objective":
        return dout * d * (4.0 + 4 + 1), "byte"                     # read U, W, Q
    return 0.0, "unknown"


# Executed tensor-core work of the products that run on tcgen05 (fp16 pieces, fp32 accumulate):
#   lnq_mgemm: F's two pieces against m one-hot columns per row, over the upper block triangle
#     (pair blocks of 256 coordinates; the K blocks of 64 from the diagonal block on);
#   lnq_residual_gemm: three piece products per row (H1 R1, H1 R2, H2 R1) over all of F.
def executed_tensor_flops(layer, m, kernel):
    d, dout = layer.d_in, layer.d_out
    nk, pairs = -(-d // 64), -(-d // 256)
    if kernel == "lnq_mgemm":
        kblocks = sum(nk - 4 * ip for ip in range(pairs))
        return 2.0 * 2 * m * 256 * 64 * kblocks * dout
    if kernel == "lnq_residual_gemm":
        return 2.0 * 3 * (pairs * 256) * (nk * 64) * dout
    return None


# DRAM bytes per launch of the dominant kernel from ncu captures (dram__bytes_read.sum +
# dram__bytes_write.sum of one launch, the block's own layer shapes with 16384 calibration
# tokens, which do not change this kernel's work), per output row for each (d_in, d_out, m),
# valid only while the kernel's source is the one that was measured.
TRAFFIC = {
    "lnq_mgemm": {
        "source": "lnq_vgemm.cu",
        "sha256": "eb71dc725b8bf11887f2350945960880c807ff5d1ff296aa89c87c9375f79969",
        "bytes_per_row": {
            "4096/4096/16": 1177223168 / 4096, "4096/4096/8": 609373696 / 4096,
            "4096/11008/16": 2883097856 / 11008, "4096/11008/8": 1477671936 / 11008,
            "11008/4096/16": 34628989696 / 4096, "11008/4096/8": 17168465408 / 4096,
        },
    },
}


def measured_traffic(kernel, launches):
    """Average DRAM bytes per launch over `launches` = [(layer, count)], or None."""
    rec = TRAFFIC.get(kernel)
    if rec is None:
        return None
    path = os.path.join(ROOT, "post_weight_quantization_guided_b200", "csrc", rec["source"])
    try:
        digest = hashlib.sha256(open(path, "rb").read()).hexdigest()
    except OSError:
        return None
    if digest != rec["sha256"]:
        return None
    total, count = 0.0, 0
    for layer, c in launches:
        per_row = rec["bytes_per_row"].get(f"{layer.d_in}/{layer.d_out}/{layer.m}")
        if per_row is None:
            return None
        total += c * per_row * layer.d_out
        count += c
    return total / count if count else None


def roofline(work, unit, ms, peaks, fp32_peak):
    """Roofline object for `work` algorithmic units done in `ms` of device time."""
    sec = ms / 1e3
    src = peaks.get("source", "measured")
    if unit == "flop":
        sustained = "bf16_tflops_sustained" in peaks
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        achieved = work / sec / 1e12
        kind = f"bf16 dense, {'sustained' if sustained else 'burst'} (of {src})"
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_kind": kind}
    if unit == "byte":
        peak = peaks["hbm_gbs"]
        achieved = work / sec / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": f"HBM copy (of {src})"}
    peak = fp32_peak["sustained"]
    achieved = work / sec / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tlane-op/s",
            "frac": achieved / peak,
            "peak_kind": "FP32 FFMA lane-ops, sustained (of measured, this run's probe)"}


# ------------------------------------------------------------------------------------------
# FP32 lane-operation peak, measured with the library's FFMA probe
# ------------------------------------------------------------------------------------------
def measure_fp32_peak(device):
    from post_weight_quantization_guided_b200 import binding as b
    sink = torch.zeros(1, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    iters = 1 << 14
    for _ in range(3):
        b.lnq_fp32_probe(iters, sink)
    torch.cuda.synchronize(device)
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ops = b.lnq_fp32_probe(iters, sink)
        e1.record(stream)
        torch.cuda.synchronize(device)
        best = max(best, ops / (e0.elapsed_time(e1) / 1e3))
    # sustained: back-to-back launches for about two seconds
    per_launch_s = ops / best
    reps = max(4, int(2.0 / per_launch_s))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    total = 0
    e0.record(stream)
    for _ in range(reps):
        total += b.lnq_fp32_probe(iters, sink)
    e1.record(stream)
    torch.cuda.synchronize(device)
    sustained = total / (e0.elapsed_time(e1) / 1e3)
    return {"burst": best / 1e12, "sustained": sustained / 1e12, "unit": "Tlane-op/s",
            "how": f"FFMA probe over all SMs: best of 5 launches (burst), {reps} launches "
                   "back to back (sustained)"}


# ------------------------------------------------------------------------------------------
# Multi-rank host logic (one block per rank, weak scaling, no data-path collective)
# ------------------------------------------------------------------------------------------
def per_rank_layer(wl, rank):
    """Rank r's q_proj-shaped layer: same shapes and distributions, seeds offset by 100 r."""
    base = wl.Q_PROJ
    return wl.scaled(base, seed=base.seed + 100 * rank, x_seed=base.x_seed + 100 * rank)


def per_rank_block(wl, rank, m):
    """Rank r's decoder block at m codewords: the seeds of every layer offset by 100 r."""
    return [wl.scaled(L, seed=L.seed + 100 * rank, x_seed=L.x_seed + 100 * rank)
            for L in wl.decoder_block(m)]


def max_over_ranks(values, world, device):
    """Element-wise maximum over the ranks of a list of timings (the job ends with its slowest
    rank)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t]


def job_throughput(world, rows_per_rank, ms_per_step):
    """Whole-job rows per second: every rank quantises rows_per_rank rows per step."""
    return world * rows_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------------------------------
# Oracle (CPU) baseline on a bounded sample
# ------------------------------------------------------------------------------------------
def _oracle_lnq_rate(orc, F0, W0, m, iters, budget_s, threads):
    """Rows per second of the oracle's LNQ (init + iters) on rows of W0 against F0."""
    rows, t = 0, 0.0
    while (t < budget_s or rows == 0) and rows < W0.shape[0]:
        k = min(threads, W0.shape[0] - rows)
        t0 = time.perf_counter()
        orc.lnq_rows(F0, W0[rows:rows + k], m, iters, init=True, nthreads=threads)
        t += time.perf_counter() - t0
        rows += k
    return rows / t, rows


def _oracle_tile_seconds(orc, X, s, budget_s, rng, max_tiles=64):
    """Seconds per 64 x 64 Fisher tile of the oracle over all of X's tokens."""
    d = X.shape[1]
    tiles, t = 0, 0.0
    while (t < budget_s or tiles == 0) and tiles < max_tiles:
        i0, k0 = (int(v) for v in rng.integers(0, d - 64, 2))
        A = X[:, i0:i0 + 64].double().cpu().numpy()
        B = X[:, k0:k0 + 64].double().cpu().numpy()
        t0 = time.perf_counter()
        orc.fisher_block(A, B, s, 1.0)
        t += time.perf_counter() - t0
        tiles += 1
    return t / tiles, tiles


def block_cpu_estimate(orc, layers16, tile_s, rates):
    """Extrapolated oracle seconds for one step of the block: every layer's Fisher blocks (64 x 64
    tiles) plus LNQ of every row at both bit widths. rates[(d_in, m)] = oracle rows/s."""
    fisher = sum(L.groups * (-(-L.d_in // 64)) ** 2 * tile_s for L in layers16)
    lnq = sum(L.d_out / rates[(L.d_in, m)] for L in layers16 for m in (16, 8))
    return fisher, lnq


def cpu_baseline_block(layers16, inputs, F_small, budget_s=20.0, threads=None):
    """Oracle throughput in rows/s on a bounded sample of the block, extrapolated to one step:
    64 x 64 Fisher tiles at n = 131072 (any tile costs the same) and LNQ rows (init + 5
    iterations) of a d_in = 4096 and a d_in = 11008 layer at both bit widths, on the GPU's F."""
    from oracle import oracle as orc
    threads = threads or os.cpu_count()
    rng = np.random.default_rng(0)
    q = layers16[0]
    X, G, _ = inputs(q)
    R = q.rows_per_group
    s = np.empty(q.n)
    for r0 in range(0, q.n, 8192):
        Gh = G[r0:r0 + 8192, 0:R].double().cpu().numpy()
        s[r0:r0 + Gh.shape[0]] = orc.group_scales(Gh, Gh.shape[0], R, 1)[0]
    tile_s, tiles = _oracle_tile_seconds(orc, X, s, budget_s * 0.25, rng)
    rates, sampled = {}, []
    for L in (layers16[0], layers16[-1]):
        F0 = F_small[L.name]
        W0 = inputs(L)[2][:L.rows_per_group].double().cpu().numpy()
        for m in (16, 8):
            rate, rows = _oracle_lnq_rate(orc, F0, W0, m, L.iters, budget_s * 0.18, threads)
            rates[(L.d_in, m)] = rate
            sampled.append(f"{rows} rows at d_in={L.d_in}, m={m}")
    fisher_s, lnq_s = block_cpu_estimate(orc, layers16, tile_s, rates)
    rows = 2 * sum(L.d_out for L in layers16)
    return {"value": rows / (fisher_s + lnq_s), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": (f"Fisher: {tiles} 64x64 tiles (n={q.n}) extrapolated to every layer's "
                       f"{q.groups} blocks; LNQ (init + {q.iters} iterations, group 0 rows, on "
                       f"the GPU's F): {', '.join(sampled)}, extrapolated to all rows of the "
                       f"block at both bit widths; FP64, {threads} OpenMP threads"),
            "fisher_s_extrapolated": fisher_s, "lnq_s_extrapolated": lnq_s}


# ------------------------------------------------------------------------------------------
# Main arm: the decoder block
# ------------------------------------------------------------------------------------------
class BlockInputs:
    """Device-resident inputs of a block: X per distinct draw, G and W per layer."""

    def __init__(self, wl, layers, device):
        self.X, self.G, self.W = {}, {}, {}
        for L in layers:
            if L.x_seed not in self.X:
                self.X[L.x_seed] = wl.make_x(L, device)
            self.G[L.name] = wl.make_g(L, device)
            self.W[L.name] = wl.make_w(L, device)

    def __call__(self, L):
        return self.X[L.x_seed], self.G[L.name], self.W[L.name]


def run_block(args, rank, world, device):
    import post_weight_quantization_guided_b200 as lnq
    from post_weight_quantization_guided_b200 import binding as b
    from post_weight_quantization_guided_b200 import workloads as wl

    lnq.binding.lib()
    torch.cuda.set_device(device)
    mset = (16, 8)
    blocks = {m: per_rank_block(wl, rank, m) for m in mset}
    layers = blocks[16]
    nl = len(layers)
    inputs = BlockInputs(wl, layers, device)
    # outputs per (layer, m); one F buffer (the largest) reused layer by layer
    out = {}
    for m in mset:
        for L in blocks[m]:
            out[(L.name[:-len(f"_m{m}")], m)] = (
                torch.empty((L.d_out, m), dtype=torch.float32, device=device),
                torch.empty((L.d_out, L.d_in), dtype=torch.uint8, device=device),
                torch.empty(L.d_out, dtype=torch.float64, device=device))
    base = [L.name[:-len("_m16")] for L in layers]
    dmax = max(L.d_in for L in layers)
    Fbuf = torch.empty(max(L.groups * L.d_in * L.d_in for L in layers), dtype=torch.float32,
                       device=device)
    st = torch.empty(max(L.d_out for L in layers), dtype=torch.int32, device=device)
    fsz = max(b.lnq_workspace_size(b.LNQ_OP_BUILD_FISHER, L.n, L.d_in, L.d_out, L.groups, 16)
              for L in layers)
    qsz = max(b.lnq_workspace_size(b.LNQ_OP_QUANTIZE_ROWS, 0, L.d_in, L.d_out, L.groups, m)
              for L in layers for m in mset)
    ws_f = torch.empty(fsz, dtype=torch.uint8, device=device)
    ws_q = torch.empty(qsz, dtype=torch.uint8, device=device)
    ws_i = torch.empty(256, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def F_of(L):
        return Fbuf[:L.groups * L.d_in * L.d_in].view(L.groups, L.d_in, L.d_in)

    def layer_fisher(k, src=None):
        L = layers[k]
        X, G, _ = src(L) if src else inputs(L)
        lnq.lnq_build_fisher(X, G, L.groups, F=F_of(L), ws=ws_f)

    def layer_lnq(k, m, src=None, dst=None):
        L = blocks[m][k]
        W = (src(layers[k]) if src else inputs(layers[k]))[2]
        C, Q, J = (dst or out)[(base[k], m)]
        lnq.lnq_init_codebook(W, m, C, Q, ws=ws_i)
        lnq.lnq_quantize_rows(F_of(L), W, m, L.iters, C, Q, J, st[:L.d_out], ws=ws_q)

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        for k in range(nl):
            layer_fisher(k)
            if evs is not None:
                evs[1 + 3 * k].record(stream)
            for mi, m in enumerate(mset):
                layer_lnq(k, m)
                if evs is not None:
                    evs[2 + 3 * k + mi].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert b.lnq_workspace_check(ws_f) == b.LNQ_OK and b.lnq_workspace_check(ws_q) == b.LNQ_OK
    fp32_peak = measure_fp32_peak(device)

    # ---------------------------------------------------------------- device-timed region
    # The block's inputs (6 GB of X, 11 GB of G) exceed L2 many times over, and every layer
    # streams through them: no L2 flush is needed between steps.
    sampler = ClockSampler(device.index) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    if sampler:
        sampler.start()
    b.lnq_profile_read()
    b.lnq_profile_enable(True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(1 + 3 * nl)]
           for _ in range(args.steps)]
    for k in range(args.steps):
        step(evs[k])
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    b.lnq_profile_enable(False)
    prof = b.lnq_profile_read()
    clocks = sampler.stop() if sampler else None
    fisher_ms = lnq_ms = 0.0
    lnq_m_ms = {m: 0.0 for m in mset}
    total_ms = 0.0
    for e in evs:
        total_ms += e[0].elapsed_time(e[-1])
        for k in range(nl):
            prev = e[0] if k == 0 else e[3 * k]
            fisher_ms += prev.elapsed_time(e[1 + 3 * k])
            for mi, m in enumerate(mset):
                t = e[1 + 3 * k + mi].elapsed_time(e[2 + 3 * k + mi])
                lnq_m_ms[m] += t
                lnq_ms += t
    assert b.lnq_workspace_check(ws_f) == b.LNQ_OK and b.lnq_workspace_check(ws_q) == b.LNQ_OK
    for key, (C, Q, J) in out.items():
        assert bool(torch.isfinite(J).all()), key

    # ---------------------------------------------------------------- sweep counters (untimed)
    # The run is deterministic, so one more pass reads the moves every timed step made.
    tails, moves = {}, {}
    for k in range(nl):
        layer_fisher(k)
        for m in mset:
            layer_lnq(k, m)
            mv, tl = b.lnq_sweep_counters(ws_q)
            moves[(k, m)], tails[(k, m)] = mv, tl
    torch.cuda.synchronize(device)
    # group 0's Fisher block of two layers for the oracle's LNQ sample
    F_small = {}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for L in (layers[0], layers[-1]):
            X, G, _ = inputs(L)
            Fs = lnq.lnq_build_fisher(X, G, L.groups, F=F_of(L), ws=ws_f)
            F_small[L.name] = Fs[0].double().cpu().numpy()

    # ---------------------------------------------------------------- end to end (host buffers)
    # Every step copies the block's inputs from pinned host memory (each distinct X once, G and W
    # per layer) and reads every result back (C, Q, J per layer and bit width), all inside the
    # timed region. Copies run on a second stream with two device buffer sets, so layer k+1's
    # inputs and layer k's results cross the bus while layer k's kernels run.
    def pinned(t):
        return torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t)

    pin_X = {sd: pinned(x) for sd, x in inputs.X.items()}
    pin_G = {nm: pinned(g) for nm, g in inputs.G.items()}
    pin_W = {nm: pinned(w) for nm, w in inputs.W.items()}
    res_host = {key: [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in v]
                for key, v in out.items()}
    dev_X = [torch.empty(max(x.numel() for x in inputs.X.values()), dtype=torch.bfloat16,
                         device=device) for _ in range(2)]
    dev_G = [torch.empty(max(g.numel() for g in inputs.G.values()), dtype=torch.bfloat16,
                         device=device) for _ in range(2)]
    dev_W = [torch.empty(max(w.numel() for w in inputs.W.values()), dtype=torch.float32,
                         device=device) for _ in range(2)]
    res_dev = [{key: [torch.empty_like(t) for t in v] for key, v in out.items()
                if key[0] == base[k]} for k in range(nl)]
    h2d = (sum(x.numel() * 2 for x in pin_X.values()) + sum(g.numel() * 2 for g in pin_G.values())
           + sum(w.numel() * 4 for w in pin_W.values()))
    d2h = sum(t.numel() * t.element_size() for v in out.values() for t in v)
    copy = torch.cuda.Stream(device)
    e2e_steps = max(1, args.steps)
    nseq = e2e_steps * nl
    in_ready = [torch.cuda.Event() for _ in range(nseq)]
    computed = [torch.cuda.Event() for _ in range(nseq)]
    read_back = [torch.cuda.Event() for _ in range(nseq)]
    # X draws in sequence order: a layer that shares the previous layer's X reuses its buffer;
    # a new draw goes to the buffer the draw before the previous one used
    draw_of, draw_first, draw_last = [], [], []
    for sq in range(nseq):
        new = sq == 0 or layers[(sq - 1) % nl].x_seed != layers[sq % nl].x_seed
        if new:
            draw_first.append(sq)
            draw_last.append(sq)
        draw_of.append(len(draw_first) - 1)
        draw_last[-1] = sq

    def views(sq):
        L = layers[sq % nl]
        u = sq % 2
        X = dev_X[draw_of[sq] % 2][:L.n * L.d_in].view(L.n, L.d_in)
        G = dev_G[u][:L.n * L.d_out].view(L.n, L.d_out)
        W = dev_W[u][:L.d_out * L.d_in].view(L.d_out, L.d_in)
        return X, G, W

    def copy_inputs(sq):
        L = layers[sq % nl]
        X, G, W = views(sq)
        with torch.cuda.stream(copy):
            if sq >= 2:
                copy.wait_event(computed[sq - 2])   # layer sq-2 is done with G/W buffer set
            dr = draw_of[sq]
            if draw_first[dr] == sq:
                if dr >= 2:
                    copy.wait_event(computed[draw_last[dr - 2]])   # done with this X buffer
                X.copy_(pin_X[L.x_seed], non_blocking=True)
            G.copy_(pin_G[L.name], non_blocking=True)
            W.copy_(pin_W[L.name], non_blocking=True)
            in_ready[sq].record(copy)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy.wait_event(e0)
    copy_inputs(0)
    for sq in range(nseq):
        k = sq % nl
        if sq + 1 < nseq:
            copy_inputs(sq + 1)
        stream.wait_event(in_ready[sq])
        if sq >= 2:
            stream.wait_event(read_back[sq - 2])   # earlier results have left their buffers
        src = (lambda _L, _sq=sq: views(_sq))
        layer_fisher(k, src)
        for m in mset:
            layer_lnq(k, m, src, res_dev[k])
        computed[sq].record(stream)
        with torch.cuda.stream(copy):
            copy.wait_event(computed[sq])
            for m in mset:
                for t_h, t_d in zip(res_host[(base[k], m)], res_dev[k][(base[k], m)]):
                    t_h.copy_(t_d, non_blocking=True)
            read_back[sq].record(copy)
    stream.wait_stream(copy)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e0.elapsed_time(e1)
    for key, (C, Q, J) in out.items():
        assert np.array_equal(res_host[key][1].numpy(), Q.cpu().numpy()), key
    del pin_X, pin_G, pin_W, dev_X, dev_G, dev_W, res_dev

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, device)
    if rank != 0:
        return None, None
    rows_per_step = sum(L.d_out for L in layers) * len(mset)
    ms_per_step = total_ms / args.steps
    peaks = load_peaks()

    # ---------------------------------------------------------------- per-kernel roofline
    kernels = {}
    all_ms = sum(v[1] for v in prof.values())
    for name, (launches, ms) in prof.items():
        work, unit, hw, lw = 0.0, None, 0.0, []
        for k, L in enumerate(layers):
            if name in FISHER_KERNELS:
                c = launches_per_call(name, L, 0)
                if c:
                    w, unit = algorithmic_work(L, 16, name)
                    work += c * w
                    lw.append((L, c))
                continue
            for m in mset:
                Lm = blocks[m][k]
                c = launches_per_call(name, Lm, Lm.iters)
                if not c:
                    continue
                tail = tails[(k, m)] / Lm.iters if name == "lnq_sweep" else None
                w, unit = algorithmic_work(Lm, m, name, tail)
                work += c * w
                lw.append((Lm, c))
                ex = executed_tensor_flops(Lm, m, name)
                if ex is not None:
                    hw += c * ex
        work *= args.steps
        hw *= args.steps
        if unit is None or unit == "unknown":
            continue
        entry = {"launches_per_step": launches / args.steps, "avg_ms": ms / launches,
                 "share": ms / all_ms, "roofline": roofline(work, unit, ms, peaks, fp32_peak)}
        if hw:
            tens = hw / (ms / 1e3) / 1e12
            pk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
            entry["tensor_executed"] = {"achieved": tens, "peak": pk, "unit": "TFLOP/s",
                                        "frac": tens / pk}
        entry["_launches"] = lw
        if abs(sum(c for _, c in lw) * args.steps - launches) > 0:
            entry["launch_count_mismatch"] = [sum(c for _, c in lw) * args.steps, launches]
        kernels[name] = entry
    dominant = max(kernels, key=lambda k: kernels[k]["share"])
    roof = dict(kernels[dominant]["roofline"])
    roof["kernel"] = dominant
    roof["traffic"] = measured_traffic(dominant, kernels[dominant]["_launches"])
    roof["peak_source"] = peaks["source"]
    for v in kernels.values():
        del v["_launches"]
    fisher_flops = sum(algorithmic_work(L, 16, "fisher_syrk")[0] for L in layers)
    sweep_moves = {f"m{m}": sum(moves[(k, m)] for k in range(nl)) for m in mset}
    line = {
        "metric": METRIC, "value": job_throughput(world, rows_per_step, ms_per_step),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic (seeded draws with the decoder block's shapes and distributions)",
        "config": {"workload": "llama2_7b_decoder_block_7_linears_n131072_m16_and_m8",
                   "layers": [f"{L.name[:-4]} {L.d_in}->{L.d_out}" for L in layers],
                   "n": layers[0].n, "groups": layers[0].groups, "m": list(mset),
                   "iters": layers[0].iters, "rows_per_step": world * rows_per_step,
                   "fisher_per_layer": "built once, used by both bit widths",
                   "parallelism": f"block-per-gpu x{world}",
                   "l2": "inputs larger than L2 (17 GB per step streamed), no flush"},
        "gpu_launches": int(round(sum(v[0] for v in prof.values()) / args.steps)) * args.steps,
        "e2e": {"value": job_throughput(world, rows_per_step, e2e_ms / e2e_steps), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "block_ms": {f"m{m}": (fisher_ms + lnq_m_ms[m]) / args.steps for m in mset},
        "fisher_ms_per_step": fisher_ms / args.steps,
        "lnq_rows_per_s": {f"m{m}": sum(L.d_out for L in layers) / (lnq_m_ms[m] / args.steps
                                                                      / 1e3) for m in mset},
        "fisher_tflops": fisher_flops / (fisher_ms / args.steps / 1e3) / 1e12,
        "sweep_moves_per_step": sweep_moves,
        "roofline": roof,
        "fp32_peak": fp32_peak,
        "kernels": kernels,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_block(layers, inputs, F_small,
                                                  budget_s=args.cpu_budget)
    return line, fp32_peak


# ------------------------------------------------------------------------------------------
# Secondary workload: one q_proj layer (the consumer and the diagonal variant run on its result)
# ------------------------------------------------------------------------------------------
def run_q_proj(args, rank, device, fp32_peak, steps=5, warmup=3):
    import post_weight_quantization_guided_b200 as lnq
    from post_weight_quantization_guided_b200 import binding as b
    from post_weight_quantization_guided_b200 import workloads as wl

    layer = per_rank_layer(wl, rank)
    X, G, W = wl.make_layer(layer, device)
    d, dout, m, it = layer.d_in, layer.d_out, layer.m, layer.iters
    F = torch.empty((layer.groups, d, d), dtype=torch.float32, device=device)
    C = torch.empty((dout, m), dtype=torch.float32, device=device)
    Q = torch.empty((dout, d), dtype=torch.uint8, device=device)
    J = torch.empty(dout, dtype=torch.float64, device=device)
    st = torch.empty(dout, dtype=torch.int32, device=device)
    ws_f = b.workspace(b.LNQ_OP_BUILD_FISHER, layer.n, d, dout, layer.groups, m, device)
    ws_q = b.workspace(b.LNQ_OP_QUANTIZE_ROWS, 0, d, dout, layer.groups, m, device)
    ws_i = b.workspace(b.LNQ_OP_INIT_CODEBOOK, 0, d, dout, 1, m, device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        lnq.lnq_build_fisher(X, G, layer.groups, F=F, ws=ws_f)
        lnq.lnq_init_codebook(W, m, C, Q, ws=ws_i)
        lnq.lnq_quantize_rows(F, W, m, it, C, Q, J, st, ws=ws_q)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    b.lnq_profile_read()
    b.lnq_profile_enable(True)
    ms = 0.0
    for k in range(steps):
        flush.fill_(k & 0xFF)           # evict L2 between timed steps (untimed)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms += e0.elapsed_time(e1)
    b.lnq_profile_enable(False)
    prof = b.lnq_profile_read()
    assert b.lnq_workspace_check(ws_q) == b.LNQ_OK
    step()
    mv, tail = b.lnq_sweep_counters(ws_q)
    peaks = load_peaks()
    kernels = {}
    for name, (launches, kms) in prof.items():
        w, unit = algorithmic_work(layer, m, name, tail / it if name == "lnq_sweep" else None)
        if unit == "unknown":
            continue
        kernels[name] = {"avg_ms": kms / launches, "launches_per_step": launches / steps,
                         "roofline": roofline(w * launches, unit, kms, peaks, fp32_peak)}
    res = {"workload": layer.name, "steps": steps, "ms_per_step": ms / steps,
           "rows_per_s": dout / (ms / steps / 1e3), "sweep_moves": mv, "sweep_tail": tail,
           "kernels": kernels, "l2": "flushed between timed steps (256 MB write)"}

    # the consumer of (C, Q): the lookup-table GEMV on the step's codes (batch 1); the packed codes
    # are cycled through enough copies that they come from HBM, not L2
    bits = m.bit_length() - 1
    Pk = lnq.lnq_pack_codes(Q, bits)
    copies = max(2, int(3 * 126e6 / (Pk.numel() * 4)) + 1)
    Ps = [Pk.clone() for _ in range(copies)]
    xg = torch.randn(1, d, device=device, generator=torch.Generator(device=device).manual_seed(5))
    yg = torch.empty(1, dout, device=device)
    for k in range(4):
        lnq.lnq_lut_gemv(xg, Ps[k % copies], C, d, y=yg)
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for k in range(copies):
            lnq.lnq_lut_gemv(xg, Ps[k], C, d, y=yg)
    graph.replay()
    torch.cuda.synchronize(device)
    replays = 10
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(replays):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize(device)
    lut_us = g0.elapsed_time(g1) * 1e3 / (replays * copies)
    del graph, Ps
    lut_bytes = Pk.numel() * 4 + C.numel() * 4 + d * 4 + dout * 4
    res_lut = {"workload": f"{layer.name}: {bits}-bit packed codes, batch 1",
               "us_per_call": lut_us, "algorithmic_bytes": lut_bytes,
               "achieved_gbs": lut_bytes / (lut_us * 1e-6) / 1e9, "peak_gbs": peaks["hbm_gbs"],
               "frac": lut_bytes / (lut_us * 1e-6) / 1e9 / peaks["hbm_gbs"]}

    # LNQ with diagonal Fisher blocks (the same iterations, F_g = diag of the step's F_g)
    Fd = torch.diagonal(F, dim1=1, dim2=2).contiguous()
    C0d, Q0d = lnq.lnq_init_codebook(W, m)
    Cx, Qx = C0d.clone(), Q0d.clone()
    Jx = torch.empty(dout, dtype=torch.float64, device=device)
    for _ in range(3):
        Cx.copy_(C0d)
        Qx.copy_(Q0d)
        lnq.lnq_quantize_rows_diag(Fd, W, m, it, Cx, Qx, Jx)
    reps, diag_ms = 10, 0.0
    for _ in range(reps):
        Cx.copy_(C0d)
        Qx.copy_(Q0d)
        flush.fill_(0x5A)               # evict L2 (untimed)
        g0.record(stream)
        lnq.lnq_quantize_rows_diag(Fd, W, m, it, Cx, Qx, Jx)
        g1.record(stream)
        torch.cuda.synchronize(device)
        diag_ms += g0.elapsed_time(g1) / reps
    diag_bytes = dout * d * (4 + 1 + 1) + 2 * dout * m * 4 + dout * 8 + layer.groups * d * 4
    res_diag = {"workload": f"{layer.name}: {it} iterations, m = {m}", "ms_per_call": diag_ms,
                "rows_per_s": dout / (diag_ms / 1e3), "algorithmic_bytes": diag_bytes,
                "achieved_gbs": diag_bytes / (diag_ms * 1e-3) / 1e9,
                "frac_hbm": diag_bytes / (diag_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}

    # A/B: the GANQ-style solver (Cholesky / back-substitution assignment, the same codebook
    # step) against LNQ on the same F, W and initial codebooks, the same number of iterations
    ws_g = b.workspace(b.LNQ_OP_GANQ_ROWS, 0, d, dout, layer.groups, m, device)
    Cg, Qg = C0d.clone(), Q0d.clone()
    Jg = torch.empty(dout, dtype=torch.float64, device=device)
    lnq.lnq_ganq_rows(F, W, m, it, Cg, Qg, Jg, ws=ws_g)       # warm-up
    torch.cuda.synchronize(device)
    reps, ganq_ms = 3, 0.0
    b.lnq_profile_read()
    b.lnq_profile_enable(True)
    for _ in range(reps):
        Cg.copy_(C0d)
        Qg.copy_(Q0d)
        flush.fill_(0x3C)
        g0.record(stream)
        lnq.lnq_ganq_rows(F, W, m, it, Cg, Qg, Jg, ws=ws_g)
        g1.record(stream)
        torch.cuda.synchronize(device)
        ganq_ms += g0.elapsed_time(g1) / reps
    b.lnq_profile_enable(False)
    gprof = b.lnq_profile_read()
    Cl, Ql = C0d.clone(), Q0d.clone()
    Jl = torch.empty(dout, dtype=torch.float64, device=device)
    lnq.lnq_quantize_rows(F, W, m, it, Cl, Ql, Jl, ws=ws_q)
    torch.cuda.synchronize(device)
    del ws_g
    res_ganq = {"workload": f"{layer.name}: {it} iterations, m = {m}, from the same initial "
                            "codebooks as LNQ",
                "ms_per_call": ganq_ms, "rows_per_s": dout / (ganq_ms / 1e3),
                "kernels_ms_per_call": {k: v[1] / reps for k, v in gprof.items()},
                "sum_J": float(Jg.sum()), "lnq_sum_J": float(Jl.sum()),
                "J_ratio_vs_lnq": float(Jg.sum()) / float(Jl.sum()),
                "rows_lower_than_lnq": int((Jg < Jl).sum())}
    return res, res_lut, res_diag, res_ganq


# ------------------------------------------------------------------------------------------
# Reference arm: the oracle on the host cores
# ------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The oracle (plain FP64 CPU code) on the host cores, same metric and workload, each step a
    bounded sample extrapolated to the whole block."""
    if rank != 0:
        return None
    from post_weight_quantization_guided_b200 import workloads as wl
    from oracle import oracle as orc
    orc.build()
    layers = wl.decoder_block(16)
    q, down = layers[0], layers[-1]
    threads = os.cpu_count()
    # Untimed preparation: the q layer's inputs, and for the LNQ sample group 0's Fisher block of
    # the q and down layers over their first 8192 tokens (a plain float64 product; the sample's
    # cost per row does not depend on n).
    Xq = wl.make_x(q)
    Gq = wl.make_g(q)
    Rq = q.rows_per_group
    s = orc.group_scales(Gq[:, :Rq].double().numpy(), q.n, Rq, 1)[0]
    prepared = {}
    for L in (q, down):
        Ls = wl.scaled(L, n=8192)
        X = wl.make_x(Ls).double().numpy()
        Gs = wl.make_g(Ls)
        ss = orc.group_scales(Gs[:, :L.rows_per_group].double().numpy(), 8192,
                              L.rows_per_group, 1)[0]
        prepared[L.d_in] = ((X * ss[:, None]).T @ X,
                            wl.make_w(L)[:threads].double().numpy())
    vals = []
    rng = np.random.default_rng(0)
    for k in range(args.warmup + args.steps):
        tile_s, _ = _oracle_tile_seconds(orc, Xq, s, 0.0, rng, max_tiles=1)
        rates = {}
        for dd, (F0, W0) in prepared.items():
            for m in (16, 8):
                rows = 1 if dd > 4096 else 2
                t0 = time.perf_counter()
                orc.lnq_rows(F0, W0[:rows], m, q.iters, init=True, nthreads=threads)
                rates[(dd, m)] = rows / (time.perf_counter() - t0)
        fisher_s, lnq_s = block_cpu_estimate(orc, layers, tile_s, rates)
        if k >= args.warmup:
            vals.append(2 * sum(L.d_out for L in layers) / (fisher_s + lnq_s))
    value = statistics.median(vals)
    sample = ("per step: one 64x64 Fisher tile (n=131072), LNQ (init + 5 iterations) of 2 rows at "
              "d_in=4096 and 1 row at d_in=11008 for m=16 and m=8 (one OpenMP thread per row), "
              "extrapolated to the whole block at both bit widths")
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * 2 * sum(L.d_out for L in layers) / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "llama2_7b_decoder_block_7_linears_n131072_m16_and_m8",
                       "layers": [f"{L.name[:-4]} {L.d_in}->{L.d_out}" for L in layers],
                       "n": q.n, "groups": q.groups, "m": [16, 8], "iters": q.iters},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-q-proj", action="store_true",
                    help="skip the secondary single-layer workload")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    from datetime import timedelta
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    try:
        line, fp32_peak = run_block(args, rank, world, device)
        if not args.no_q_proj and rank == 0:
            torch.cuda.empty_cache()
            qp = run_q_proj(args, rank, device, fp32_peak)
            if line is not None:
                line["q_proj"], line["lut_gemv"], line["lnq_diag"], line["ganq_ab"] = qp
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
