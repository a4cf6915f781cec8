"""GPU-versus-oracle parity on the decoder-block workload: the seven linears of a Llama-2-7B-shaped
block over 131072 synthetic tokens, 4 Fisher groups, 5 iterations, at 4 and at 3 bits.

"GuidedQuant" blog post, GuidedQuant section (guided Fisher blocks, grouping sentence) and LNQ
section (problem and iteration). q/k/v/o share one shape and recipe, as do gate/up; the three
distinct shapes (q: 4096 -> 4096; gate: 4096 -> 11008; down: 11008 -> 4096) run at both bit
widths of the benchmark. Sampled Fisher tiles plus the full diagonal of the first and last group;
follow-mode LNQ rows of every group through every iteration. Tolerances are in parity_helpers.

This file sorts after every other parity file and just before the no-allocation tests: it is the
longest (about a minute of oracle work per layer and bit width).
"""
import pytest
import torch

from parity_helpers import check_fisher_sampled, lnq_follow_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lnq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_guided_b200 import build
    build.build_library()
    import post_weight_quantization_guided_b200 as pkg
    return pkg


@pytest.fixture(scope="module")
def wl():
    from post_weight_quantization_guided_b200 import workloads
    return workloads


@pytest.mark.parametrize("index,bits", [(0, (4, 3)), (4, (4, 3)), (6, (4, 3))])
def test_decoder_block_layer(orc, lnq, wl, index, bits):
    layer = wl.decoder_block(16)[index]
    dev = torch.device("cuda:0")
    X, G, W = wl.make_layer(layer, dev)
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    check_fisher_sampled(orc, F, X, G, layer.groups, tiles_per_group=3,
                         check_groups=[0, layer.groups - 1])
    del X, G
    torch.cuda.empty_cache()
    rows = 1 if layer.d_in > 4096 else 2
    for b in bits:
        summary, _, _ = lnq_follow_parity(orc, lnq, F, W, 1 << b, layer.iters,
                                          rows_per_group=rows)
        assert summary["moves"] > 0
