"""GPU-versus-oracle parity with one Fisher block per output row (groups = d_out).

"GuidedQuant" blog post, GuidedQuant section, third equation: each output row j has its own block
F_j = (1/n) X^T diag(G_:,j^2) X before any grouping; grouping and averaging is what makes it
scale. With groups = d_out no averaging happens, so s_g is one squared gradient column, whose
spread across tokens is much wider than a group mean's. The library has no special case for it;
these tests check the Fisher blocks in full and LNQ rows in follow mode on the tiny layer.
Tolerances are in parity_helpers.
"""
import pytest
import torch

from parity_helpers import check_fisher_full, lnq_follow_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lnq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_guided_b200 import build
    build.build_library()
    import post_weight_quantization_guided_b200 as pkg
    return pkg


@pytest.mark.parametrize("m", [4, 8])
def test_one_block_per_row_tiny_layer(orc, lnq, m):
    from post_weight_quantization_guided_b200 import workloads as wl
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, torch.device("cuda:0"))
    F = lnq.lnq_build_fisher(X, G, layer.d_out)
    assert F.shape == (layer.d_out, layer.d_in, layer.d_in)
    check_fisher_full(orc, F, X, G, layer.d_out)
    summary, _, _ = lnq_follow_parity(orc, lnq, F, W, m, layer.iters)
    assert summary["moves"] > 0
