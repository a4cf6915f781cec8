"""Pins for the oracle's guided Fisher build, each against something other than the oracle.

Passages: "GuidedQuant" blog post, GuidedQuant section -- the first equation (plain layer-wise
output error, whose Hessian is X^T X) and the third equation (gradient-weighted output error
= n * sum_j (w_j - w^_j)^T F_j (w_j - w^_j)), plus the sentence on grouping Fisher blocks and
averaging within a group.
"""
import numpy as np
import pytest
import torch

from conftest import golden
from post_weight_quantization_guided_b200 import workloads as wl


def _tiny_inputs():
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, "cpu")
    return layer, X.double().numpy(), G.double().numpy(), W.double().numpy()


def test_hand_worked_fisher_golden(orc):
    g = golden("fisher_hand_n3_d2.json")
    X, G = np.array(g["X"], float), np.array(g["G"], float)
    for key, groups in (("groups_1", 1), ("groups_2", 2)):
        S = orc.group_scales(G, 3, 2, groups)
        np.testing.assert_array_equal(S, np.array(g[key]["s"]))
        np.testing.assert_array_equal(orc.fisher_full(X, G, groups), np.array(g[key]["F"]))


def test_unit_gradients_give_gram_matrix(orc):
    """All gradients 1 => F = X^T X (first vs third objective on the GuidedQuant page)."""
    layer, X, _, _ = _tiny_inputs()
    F = orc.fisher_full(X, None, 1)[0]
    ref = X.T @ X
    np.testing.assert_allclose(F, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # explicit all-ones G must agree with G = None
    ones = np.ones((layer.n, layer.d_out))
    F1 = orc.fisher_full(X, ones, 1)[0]
    np.testing.assert_allclose(F1, F, rtol=1e-13)


def test_weighted_output_error_identity(orc):
    """||G (.) (X W^T - X What^T)||_F^2 == n * sum_j D_j^T F_j D_j with F_j = (1/n) X^T diag(G_j^2) X.

    The left side is evaluated directly with numpy matrix products (no oracle code)."""
    layer, X, G, W = _tiny_inputs()
    n, d_out = layer.n, layer.d_out
    rng = np.random.default_rng(7)
    What = W + 0.01 * rng.standard_normal(W.shape)
    lhs = np.sum((G * (X @ W.T - X @ What.T)) ** 2)
    Fj = orc.fisher_full(X, G, d_out, alpha=1.0 / n)          # one block per output row
    D = W - What
    rhs = n * sum(D[j] @ Fj[j] @ D[j] for j in range(d_out))
    assert abs(lhs - rhs) <= 1e-10 * lhs


def test_grouped_block_is_mean_of_row_blocks(orc):
    layer, X, G, _ = _tiny_inputs()
    Fj = orc.fisher_full(X, G, layer.d_out)
    Fg = orc.fisher_full(X, G, layer.groups)
    R = layer.rows_per_group
    for g in range(layer.groups):
        ref = Fj[g * R:(g + 1) * R].mean(axis=0)
        np.testing.assert_allclose(Fg[g], ref, rtol=1e-11, atol=1e-13 * np.abs(ref).max())


def test_group_scales_definition(orc):
    layer, _, G, _ = _tiny_inputs()
    S = orc.group_scales(G, layer.n, layer.d_out, layer.groups)
    R = layer.rows_per_group
    ref = np.stack([(G[:, g * R:(g + 1) * R] ** 2).mean(axis=1) for g in range(layer.groups)])
    np.testing.assert_allclose(S, ref, rtol=1e-14)
    np.testing.assert_array_equal(orc.group_scales(None, layer.n, 1, 1), np.ones((1, layer.n)))


def test_fisher_symmetric_psd_and_diag(orc):
    layer, X, G, _ = _tiny_inputs()
    Fg = orc.fisher_full(X, G, layer.groups)
    rng = np.random.default_rng(3)
    for g in range(layer.groups):
        np.testing.assert_array_equal(Fg[g], Fg[g].T)
        for _ in range(20):
            v = rng.standard_normal(layer.d_in)
            assert v @ Fg[g] @ v >= 0.0
        S = orc.group_scales(G, layer.n, layer.d_out, layer.groups)
        np.testing.assert_allclose(orc.fisher_diag(X, S[g]), np.diag(Fg[g]), rtol=1e-13)


def test_block_of_column_subsets_matches_full(orc):
    layer, X, G, _ = _tiny_inputs()
    S = orc.group_scales(G, layer.n, layer.d_out, layer.groups)
    F = orc.fisher_full(X, G, layer.groups, alpha=0.5)
    I, K = np.arange(10, 30), np.arange(64, 100)
    blk = orc.fisher_block(X[:, I], X[:, K], S[2], alpha=0.5)
    np.testing.assert_allclose(blk, F[2][np.ix_(I, K)], rtol=1e-13)


def test_identity_pin_catches_planted_mistakes(orc):
    """Planted mistakes in the Fisher construction (on the CPU, via wrong inputs to the oracle):
    gradients not squared, or the wrong group, must break the identity pin."""
    layer, X, G, W = _tiny_inputs()
    n = layer.n
    rng = np.random.default_rng(11)
    What = W + 0.01 * rng.standard_normal(W.shape)
    lhs = np.sum((G * (X @ W.T - X @ What.T)) ** 2)
    D = W - What
    # |G| instead of G^2
    Fbad = orc.fisher_full(X, np.sqrt(np.abs(G)), layer.d_out, alpha=1.0 / n)
    bad = n * sum(D[j] @ Fbad[j] @ D[j] for j in range(layer.d_out))
    assert abs(lhs - bad) > 1e-3 * lhs
    # rows paired with the wrong block
    Fj = orc.fisher_full(X, G, layer.d_out, alpha=1.0 / n)
    bad2 = n * sum(D[j] @ Fj[(j + 1) % layer.d_out] @ D[j] for j in range(layer.d_out))
    assert abs(lhs - bad2) > 1e-3 * lhs


def test_tiny_workload_recipe():
    """The tiny configuration's draws have the stated shapes, dtypes and outlier columns."""
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, "cpu")
    assert X.dtype == torch.bfloat16 and X.shape == (256, 128)
    assert G.dtype == torch.bfloat16 and G.shape == (256, 64)
    assert W.dtype == torch.float32 and W.shape == (64, 128)
    col_std = X.float().std(dim=0)
    assert int((col_std > 5).sum()) == layer.x_outlier_cols
    assert 0.005 < float(G.float().std()) < 0.02
    assert 0.015 < float(W.std()) < 0.025
    X2, G2, W2 = wl.make_layer(layer, "cpu")
    assert torch.equal(X, X2) and torch.equal(G, G2) and torch.equal(W, W2)
