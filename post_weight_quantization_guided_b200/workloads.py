"""Seeded synthetic workloads for the GuidedQuant + LNQ hot path.

This module only draws inputs. It holds none of the method's arithmetic, so both the CUDA path
and the CPU oracle can consume its tensors.

The shapes follow the Llama layers the pages evaluate on ("GuidedQuant" blog post, summarised
results on Llama-2-7B; LNQ section, 2-bit Llama-2-7B example). No model weights, calibration text
or gradients are available, so every tensor is drawn from the distributions below:

  X  layer input [n, d_in], bf16, row-major (token-major)
  G  end-loss gradient dL/dZ [n, d_out], bf16, or None for "all gradients equal 1"
  W  weights [d_out, d_in], fp32, row j = output channel w_j

Distribution parameters are (mean, standard deviation) for normals and (location, scale) for
Laplace. Student-t draws are scaled to the stated standard deviation.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Layer:
    """One linear layer to quantise: shapes, draw recipe and LNQ settings."""
    name: str
    d_in: int
    d_out: int
    n: int
    groups: int
    m: int
    iters: int
    seed: int
    x_kind: str            # "normal_outliers" | "silu_product"
    x_outlier_cols: int    # number of input channels scaled up
    x_outlier_scale: float
    x_seed: int            # layers with equal x_seed share one X draw
    g_kind: str            # "normal" | "laplace" | "ones"
    g_scale: float
    w_kind: str            # "normal" | "student_t"
    w_std: float
    w_dof: int = 0
    w_bf16: bool = False   # draw W in bf16 then widen to fp32
    x_f32_then_bf16: bool = False  # tiny case: drawn in fp32, rounded to bf16 at the boundary

    @property
    def rows_per_group(self) -> int:
        return self.d_out // self.groups

    @property
    def fisher_flops(self) -> float:
        """Dense-equivalent flops of the guided Fisher GEMM: 2 * groups * n * d_in^2."""
        return 2.0 * self.groups * self.n * self.d_in * self.d_in


def _layer(name, d_in, d_out, n, groups, m, iters, seed, **kw) -> Layer:
    return Layer(name=name, d_in=d_in, d_out=d_out, n=n, groups=groups, m=m, iters=iters,
                 seed=seed, **kw)


# Configuration 1: tiny single layer the oracle runs in full.
TINY = _layer("tiny_128x64_n256", 128, 64, 256, 4, 8, 3, seed=1,
              x_kind="normal_outliers", x_outlier_cols=4, x_outlier_scale=20.0, x_seed=1,
              g_kind="normal", g_scale=1e-2, w_kind="normal", w_std=0.02,
              x_f32_then_bf16=True)

# Configuration 2: Llama-2-7B q_proj shape, 4-bit, 4 Fisher groups (the benchmark workload).
Q_PROJ = _layer("llama2_7b_q_proj_4096x4096_n16384", 4096, 4096, 16384, 4, 16, 3, seed=2,
                x_kind="normal_outliers", x_outlier_cols=20, x_outlier_scale=30.0, x_seed=2,
                g_kind="normal", g_scale=1e-3, w_kind="student_t", w_std=0.02, w_dof=5,
                w_bf16=True)

# Configuration 3: MLP down_proj shape without guidance (F = X^T X, one group), 3-bit.
DOWN_PROJ = _layer("llama2_7b_down_proj_11008x4096_n32768", 11008, 4096, 32768, 1, 8, 4,
                   seed=3, x_kind="silu_product", x_outlier_cols=0, x_outlier_scale=1.0,
                   x_seed=3, g_kind="ones", g_scale=1.0, w_kind="normal", w_std=0.015)

# Configuration 4: Llama-3-8B up_proj shape, 2-bit, 8 Fisher groups.
UP_PROJ = _layer("llama3_8b_up_proj_4096x14336_n65536", 4096, 14336, 65536, 8, 4, 5, seed=4,
                 x_kind="normal_outliers", x_outlier_cols=41, x_outlier_scale=40.0, x_seed=4,
                 g_kind="laplace", g_scale=1e-3, w_kind="student_t", w_std=0.02, w_dof=4)


def decoder_block(m: int) -> List[Layer]:
    """Configuration 5: the seven linears of a Llama-2-7B decoder block, n = 128 x 1024 tokens,
    4 Fisher groups, 5 iterations. q/k/v share one X draw, gate/up share one, o and down have
    their own; each layer's G and W follow the single-layer configuration of the same kind."""
    n, it, gr = 131072, 5, 4
    attn = dict(x_kind="normal_outliers", x_outlier_cols=20, x_outlier_scale=30.0,
                g_kind="normal", g_scale=1e-3, w_kind="student_t", w_std=0.02, w_dof=5,
                w_bf16=True)
    mlp_in = dict(x_kind="normal_outliers", x_outlier_cols=41, x_outlier_scale=40.0,
                  g_kind="laplace", g_scale=1e-3, w_kind="student_t", w_std=0.02, w_dof=4)
    down = dict(x_kind="silu_product", x_outlier_cols=0, x_outlier_scale=1.0,
                g_kind="normal", g_scale=1e-3, w_kind="normal", w_std=0.015)
    return [
        _layer(f"block_q_m{m}", 4096, 4096, n, gr, m, it, seed=50, x_seed=50, **attn),
        _layer(f"block_k_m{m}", 4096, 4096, n, gr, m, it, seed=51, x_seed=50, **attn),
        _layer(f"block_v_m{m}", 4096, 4096, n, gr, m, it, seed=52, x_seed=50, **attn),
        _layer(f"block_o_m{m}", 4096, 4096, n, gr, m, it, seed=53, x_seed=53, **attn),
        _layer(f"block_gate_m{m}", 4096, 11008, n, gr, m, it, seed=54, x_seed=54, **mlp_in),
        _layer(f"block_up_m{m}", 4096, 11008, n, gr, m, it, seed=55, x_seed=54, **mlp_in),
        _layer(f"block_down_m{m}", 11008, 4096, n, gr, m, it, seed=56, x_seed=56, **down),
    ]


CONFIGS = {1: TINY, 2: Q_PROJ, 3: DOWN_PROJ, 4: UP_PROJ}


def scaled(layer: Layer, **changes) -> Layer:
    """A copy of `layer` with some fields replaced (smaller parity cases of the same recipe)."""
    return dataclasses.replace(layer, **changes)


# ---------------------------------------------------------------------------------------------
# Draws
# ---------------------------------------------------------------------------------------------

def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _student_t(shape, dof: int, gen, device) -> torch.Tensor:
    """Student-t with integer dof as z / sqrt(chi2_dof / dof), chi2 as a sum of squared normals."""
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(dof):
        e = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        chi2 += e * e
    return z / torch.sqrt(chi2 / dof)


def _laplace(shape, scale: float, gen, device) -> torch.Tensor:
    """Laplace(0, scale) as scale * (E1 - E2) with E = -log(1 - U), U in [0, 1)."""
    e1 = -torch.log1p(-torch.rand(shape, generator=gen, device=device, dtype=torch.float32))
    e2 = -torch.log1p(-torch.rand(shape, generator=gen, device=device, dtype=torch.float32))
    return scale * (e1 - e2)


def make_x(layer: Layer, device="cpu", chunk_rows: int = 8192) -> torch.Tensor:
    """Layer input X [n, d_in] in bf16."""
    gen = _gen(1000 + layer.x_seed, device)
    X = torch.empty((layer.n, layer.d_in), dtype=torch.bfloat16, device=device)
    if layer.x_kind == "normal_outliers":
        scale = torch.ones(layer.d_in, dtype=torch.float32, device=device)
        if layer.x_outlier_cols > 0:
            cols = torch.randperm(layer.d_in, generator=gen, device=device)[:layer.x_outlier_cols]
            scale[cols] = layer.x_outlier_scale
        for r0 in range(0, layer.n, chunk_rows):
            r1 = min(layer.n, r0 + chunk_rows)
            z = torch.randn((r1 - r0, layer.d_in), generator=gen, device=device,
                            dtype=torch.float32)
            X[r0:r1] = (z * scale).to(torch.bfloat16)
    elif layer.x_kind == "silu_product":
        for r0 in range(0, layer.n, chunk_rows):
            r1 = min(layer.n, r0 + chunk_rows)
            a = torch.randn((r1 - r0, layer.d_in), generator=gen, device=device,
                            dtype=torch.float32)
            b = torch.randn((r1 - r0, layer.d_in), generator=gen, device=device,
                            dtype=torch.float32)
            X[r0:r1] = (torch.nn.functional.silu(a) * b).to(torch.bfloat16)
    else:
        raise ValueError(layer.x_kind)
    return X


def make_g(layer: Layer, device="cpu", chunk_rows: int = 8192) -> Optional[torch.Tensor]:
    """End-loss gradients G [n, d_out] in bf16, or None when every gradient is 1."""
    if layer.g_kind == "ones":
        return None
    gen = _gen(2000 + layer.seed, device)
    G = torch.empty((layer.n, layer.d_out), dtype=torch.bfloat16, device=device)
    for r0 in range(0, layer.n, chunk_rows):
        r1 = min(layer.n, r0 + chunk_rows)
        shape = (r1 - r0, layer.d_out)
        if layer.g_kind == "normal":
            v = layer.g_scale * torch.randn(shape, generator=gen, device=device,
                                            dtype=torch.float32)
        elif layer.g_kind == "laplace":
            v = _laplace(shape, layer.g_scale, gen, device)
        else:
            raise ValueError(layer.g_kind)
        G[r0:r1] = v.to(torch.bfloat16)
    return G


def make_w(layer: Layer, device="cpu") -> torch.Tensor:
    """Weights W [d_out, d_in] in fp32."""
    gen = _gen(3000 + layer.seed, device)
    shape = (layer.d_out, layer.d_in)
    if layer.w_kind == "normal":
        W = layer.w_std * torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    elif layer.w_kind == "student_t":
        var = layer.w_dof / (layer.w_dof - 2.0)
        W = _student_t(shape, layer.w_dof, gen, device) * (layer.w_std / math.sqrt(var))
    else:
        raise ValueError(layer.w_kind)
    if layer.w_bf16:
        W = W.to(torch.bfloat16).to(torch.float32)
    return W.contiguous()


def make_layer(layer: Layer, device="cpu"):
    """(X, G, W) for one layer."""
    return make_x(layer, device), make_g(layer, device), make_w(layer, device)
