"""The decoder block across ranks (shard.py) with the GPU library as the unit computation, at one
rank: every (linear, Fisher group) unit runs through `gpu_compute` and the gathered (C, Q) must
equal, bit for bit, a direct whole-layer call of the library (a unit's group block, built with
groups = 1 over the group's gradient columns, is the same F_g as the whole layer's block g, and
rows do not interact); sampled rows are then checked against the oracle in follow mode.

"GuidedQuant" (jinukkim.me blog), GuidedQuant section: the objective is a sum over layers and
output rows, and rows share a Fisher block only inside their group, so units are independent.
"""
import pytest
import torch

from parity_helpers import lnq_follow_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lnq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_guided_b200 import build
    build.build_library()
    import post_weight_quantization_guided_b200 as pkg
    return pkg


def _small_block(wl):
    """Three layers of the decoder-block recipe at small sizes: an attention-like and an MLP-input
    layer sharing nothing, and a down-like layer with a ragged width; 2 or 4 groups, 3 iterations."""
    blk = wl.decoder_block(8)
    return [wl.scaled(blk[0], d_in=256, d_out=96, n=1536, groups=2, iters=3),
            wl.scaled(blk[4], d_in=256, d_out=160, n=1536, groups=4, iters=3),
            wl.scaled(blk[6], d_in=392, d_out=64, n=2048, groups=2, iters=3)]


def test_shard_units_match_whole_layer_calls(orc, lnq):
    from post_weight_quantization_guided_b200 import shard
    from post_weight_quantization_guided_b200 import workloads as wl
    dev = torch.device("cuda:0")
    layers = _small_block(wl)
    out, mine = shard.run(layers, 0, 1, shard.gpu_compute(lnq, wl, dev), dev)
    assert len(mine) == len(shard.units_of(layers))
    torch.cuda.synchronize()
    for li, layer in enumerate(layers):
        X, G, W = wl.make_layer(layer, dev)
        F = lnq.lnq_build_fisher(X, G, layer.groups)
        C, Q = lnq.lnq_init_codebook(W, layer.m)
        lnq.lnq_quantize_rows(F, W, layer.m, layer.iters, C, Q)
        torch.cuda.synchronize()
        Cs, Qs = out[li]
        assert torch.equal(Qs, Q), layer.name
        assert torch.equal(Cs, C), layer.name
        # the whole layer's result against the oracle, sampled rows of every group, per iteration
        summary, _, _ = lnq_follow_parity(orc, lnq, F, W, layer.m, layer.iters, rows_per_group=3)
        assert summary["moves"] > 0

