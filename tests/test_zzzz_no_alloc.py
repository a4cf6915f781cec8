"""The no-allocation Fisher entry point (lnq_build_fisher_noalloc).

Callers that cannot allocate device memory when they need F use this entry point: a plugin
without an allocator handle, code inside another framework's fixed memory pool, or a
latency-critical path that cannot afford cudaMalloc's implicit synchronisation. Its scratch is a
static device array inside the library. The checks: it agrees with the workspace entry point
within the F tolerance on two calls in a row (so leftovers of one call do not leak into the
next), it allocates no device memory, and it refuses problems larger than the array before
touching the device.

This file sorts after every other test file, so that a run stopping at the first failure has
already run all of them.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity_helpers import F_TOL


@pytest.fixture(scope="module")
def b():
    from post_weight_quantization_guided_b200 import build, binding
    build.build_library()
    return binding


def _max_rel(F1, F2):
    F1, F2 = F1.double().cpu().numpy(), F2.double().cpu().numpy()
    worst = 0.0
    for g in range(F1.shape[0]):
        d = np.sqrt(np.outer(np.diag(F2[g]), np.diag(F2[g])))
        d[d == 0] = 1e-300
        worst = max(worst, float((np.abs(F1[g] - F2[g]) / d).max()))
    return worst


def test_rejects_problems_beyond_the_static_scratch(b):
    fake = 0x100000
    n, d_in, d_out, groups = 1 << 22, 4096, 4096, 8     # s_g alone needs 128 MiB of scratch
    assert b.lnq_workspace_size(b.LNQ_OP_BUILD_FISHER, n, d_in, d_out, groups) > 64 << 20
    st = b.lib().lnq_build_fisher_noalloc(fake, fake, n, d_in, d_out, groups, ctypes.c_float(1.0),
                                          fake, None)
    assert st == b.LNQ_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls(b):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_guided_b200 import workloads as wl
    dev = torch.device("cuda:0")
    layers = [wl.TINY,
              wl.scaled(wl.TINY, n=1000, d_in=392, d_out=12, groups=4, seed=7, x_seed=7)]
    outs = []
    for layer in layers:
        X, G, _ = wl.make_layer(layer, dev)
        F_ref = b.lnq_build_fisher(X, G, layer.groups)
        F_na = torch.full_like(F_ref, float("nan"))
        outs.append((X, G, layer, F_ref, F_na))
    torch.cuda.synchronize()
    free_before = []
    for X, G, layer, F_ref, F_na in outs:                # two calls in a row
        free_before.append(torch.cuda.mem_get_info(dev)[0])
        b.lnq_build_fisher_noalloc(X, G, layer.groups, F=F_na)
        torch.cuda.synchronize()
        assert _max_rel(F_na, F_ref) <= F_TOL
    # the second call found the array set up and allocated nothing
    assert torch.cuda.mem_get_info(dev)[0] == free_before[1]
    # unguided (G absent) through the same entry point
    X, _, layer, _, _ = outs[1]
    F_ref = b.lnq_build_fisher(X, None, 1)
    F_na = b.lnq_build_fisher_noalloc(X, None, 1)
    torch.cuda.synchronize()
    assert _max_rel(F_na, F_ref) <= F_TOL


@pytest.mark.gpu
def test_noalloc_timeout_is_reported_through_the_static_scratch(b):
    """A bounded wait that gives up inside the no-allocation call sets the flag in the static
    array's header; lnq_workspace_check(NULL) reads it as LNQ_ERR_TIMEOUT, and the next call with
    the default limit is correct again."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_weight_quantization_guided_b200 import workloads as wl
    dev = torch.device("cuda:0")
    layer = wl.scaled(wl.TINY, n=512, d_in=256, d_out=8, groups=2)
    X, G, _ = wl.make_layer(layer, dev)
    F_ref = b.lnq_build_fisher(X, G, layer.groups)
    F_na = torch.empty_like(F_ref)
    assert b.lnq_noalloc_check() == b.LNQ_OK
    try:
        b.lnq_set_wait_limit(0)
        b.lnq_build_fisher_noalloc(X, G, layer.groups, F=F_na)
        assert b.lnq_noalloc_check() == b.LNQ_ERR_TIMEOUT
    finally:
        b.lnq_set_wait_limit(-1)
    assert b.lnq_noalloc_check() == b.LNQ_OK                # the check cleared the flag
    b.lnq_build_fisher_noalloc(X, G, layer.groups, F=F_na)
    assert b.lnq_noalloc_check() == b.LNQ_OK
    assert _max_rel(F_na, F_ref) <= F_TOL

