"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point the
header declares, sizes workspaces, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "lnq.h")
FAKE = 0x100000  # 256-byte aligned, never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def L():
    from post_weight_quantization_guided_b200 import build, binding
    build.build_library()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LNQ_API\s+[\w\s\*]*?\b(lnq_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert names == sorted(["lnq_build_fisher", "lnq_init_codebook", "lnq_objective",
                            "lnq_quantize_rows", "lnq_set_wait_limit", "lnq_status_string",
                            "lnq_workspace_check", "lnq_workspace_size", "lnq_profile_enable",
                            "lnq_profile_read", "lnq_build_fisher_noalloc", "lnq_packed_words",
                            "lnq_pack_codes", "lnq_lut_gemv", "lnq_quantize_rows_diag",
                            "lnq_sweep_counters", "lnq_fp32_probe", "lnq_ganq_rows"])


def test_packed_words_and_argument_checks(L):
    """Host-side rules of the packed format and the consumer entry points (no GPU needed)."""
    assert [L.lnq_packed_words(4096, b) for b in (1, 2, 3, 4)] == [128, 256, 410, 512]
    assert L.lnq_packed_words(0, 4) == 0 and L.lnq_packed_words(10, 5) == 0
    bad = 1  # LNQ_ERR_INVALID_ARG, returned before any device work
    assert L.lnq_pack_codes(None, 4, 4, 4, None, None) == bad
    assert L.lnq_lut_gemv(None, 1, None, None, 4, 4, 4, None, None) == bad


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    from post_weight_quantization_guided_b200 import binding
    assert sorted(binding.EXPORTED) == declared_functions()


def test_status_strings(L):
    from post_weight_quantization_guided_b200 import binding as b
    for s in range(6):
        assert b.lnq_status_string(s)
    assert b.lnq_status_string(99) == "unknown status"


def test_workspace_sizes(L):
    from post_weight_quantization_guided_b200 import binding as b
    n, d, dout, g = 16384, 4096, 4096, 4
    sz = b.lnq_workspace_size(b.LNQ_OP_BUILD_FISHER, n, d, dout, g, 16)
    # header, s_g per group and token, the token maxima and the group scales: O(groups n), no
    # scaled copy of X (the scaling is fused into the product's operand load)
    assert 256 + g * n * 4 + n * 4 <= sz <= 256 + g * n * 4 + n * 4 + 1024 and sz % 256 == 0
    assert b.lnq_workspace_size(b.LNQ_OP_QUANTIZE_ROWS, 0, d, dout, g, 16) >= 256 + dout * 4
    assert b.lnq_workspace_size(b.LNQ_OP_INIT_CODEBOOK, 0, d, dout, 1, 16) == 256
    assert b.lnq_workspace_size(b.LNQ_OP_BUILD_FISHER, 0, d, dout, g, 16) == 0
    # the GANQ-style solver: the QUANTIZE_ROWS workspace plus an fp64 and an fp32 factor per group,
    # the reciprocal pivots, a residual per weight and the factor statuses
    q = b.lnq_workspace_size(b.LNQ_OP_QUANTIZE_ROWS, 0, d, dout, g, 16)
    extra = g * d * d * 12 + g * d * 4 + dout * d * 4 + g * 4
    sz = b.lnq_workspace_size(b.LNQ_OP_GANQ_ROWS, 0, d, dout, g, 16)
    assert q + extra <= sz <= q + extra + 5 * 256


def _fisher(L, **kw):
    a = dict(X=FAKE, G=FAKE, n=256, d_in=128, d_out=64, groups=4, alpha=1.0, F=FAKE, ws=FAKE,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return L.lnq_build_fisher(a["X"], a["G"], a["n"], a["d_in"], a["d_out"], a["groups"],
                              ctypes.c_float(a["alpha"]), a["F"], a["ws"], a["ws_bytes"],
                              a["stream"])


@pytest.mark.parametrize("kw", [
    dict(n=0), dict(d_in=0), dict(d_in=100), dict(d_out=0), dict(groups=0), dict(groups=3),
    dict(X=None), dict(F=None), dict(X=FAKE + 8), dict(G=FAKE + 4), dict(F=FAKE + 2),
    dict(G=None),                      # G == NULL needs groups == 1
])
def test_build_fisher_rejects_bad_arguments(L, kw):
    assert _fisher(L, **kw) == 1  # LNQ_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(ws=None), dict(ws=FAKE + 16), dict(ws_bytes=100)])
def test_build_fisher_rejects_bad_workspace(L, kw):
    assert _fisher(L, **kw) == 3  # LNQ_ERR_WORKSPACE


def _quant(L, **kw):
    a = dict(F=FAKE, groups=4, W=FAKE, d_out=64, d_in=128, m=8, iters=3, C=FAKE, Q=FAKE,
             J=None, st=None, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.lnq_quantize_rows(a["F"], a["groups"], a["W"], a["d_out"], a["d_in"], a["m"],
                               a["iters"], a["C"], a["Q"], a["J"], a["st"], a["ws"],
                               a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw", [
    dict(m=3), dict(m=32), dict(m=1), dict(iters=-1), dict(groups=5), dict(d_out=0),
    dict(d_in=0), dict(d_in=16385), dict(F=None), dict(C=None), dict(Q=None), dict(W=None),
])
def test_quantize_rows_rejects_bad_arguments(L, kw):
    assert _quant(L, **kw) == 1


@pytest.mark.parametrize("kw", [
    dict(m=3), dict(m=32), dict(iters=-1), dict(groups=5), dict(d_out=0), dict(d_in=0),
    dict(d_in=16385), dict(F=None), dict(C=None), dict(Q=None), dict(W=None),
])
def test_quantize_rows_diag_rejects_bad_arguments(L, kw):
    a = dict(F=FAKE, groups=4, W=FAKE, d_out=64, d_in=128, m=8, iters=3, C=FAKE, Q=FAKE)
    a.update(kw)
    assert L.lnq_quantize_rows_diag(a["F"], a["groups"], a["W"], a["d_out"], a["d_in"], a["m"],
                                    a["iters"], a["C"], a["Q"], None, None, None) == 1


@pytest.mark.parametrize("kw", [
    dict(m=3), dict(iters=-1), dict(groups=5), dict(d_out=0), dict(d_in=0), dict(d_in=16385),
    dict(F=None), dict(C=None), dict(Q=None), dict(W=None),
])
def test_ganq_rows_rejects_bad_arguments(L, kw):
    a = dict(F=FAKE, groups=4, W=FAKE, d_out=64, d_in=128, m=8, iters=3, C=FAKE, Q=FAKE)
    a.update(kw)
    assert L.lnq_ganq_rows(a["F"], a["groups"], a["W"], a["d_out"], a["d_in"], a["m"], a["iters"],
                           a["C"], a["Q"], None, None, FAKE, 1 << 40, None) == 1


def test_ganq_rows_rejects_small_workspace(L):
    from post_weight_quantization_guided_b200 import binding as b
    need = b.lnq_workspace_size(b.LNQ_OP_GANQ_ROWS, 0, 128, 64, 4, 8)
    assert L.lnq_ganq_rows(FAKE, 4, FAKE, 64, 128, 8, 3, FAKE, FAKE, None, None, FAKE, need - 256,
                           None) == 3


def test_quantize_rows_rejects_small_workspace(L):
    assert _quant(L, ws_bytes=256) == 3
    assert _quant(L, ws=None) == 3


@pytest.mark.parametrize("m,d_in", [(5, 128), (16, 0), (16, 20000)])
def test_init_and_objective_reject_bad_arguments(L, m, d_in):
    assert L.lnq_init_codebook(FAKE, 64, d_in, m, FAKE, FAKE, FAKE, 256, None) == 1
    assert L.lnq_objective(FAKE, 1, FAKE, FAKE, FAKE, 64, d_in, m, FAKE, FAKE, 256, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from post_weight_quantization_guided_b200 import binding as b
    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        b.lib()


def test_binding_refuses_host_tensors():
    """No CPU path: every compute entry of the binding rejects host tensors before any call."""
    import torch
    import post_weight_quantization_guided_b200 as pkg
    d, dout, m, g = 16, 8, 4, 2
    X = torch.zeros(32, d, dtype=torch.bfloat16)
    G = torch.zeros(32, dout, dtype=torch.bfloat16)
    F = torch.zeros(g, d, d)
    Fd = torch.zeros(g, d)
    W = torch.zeros(dout, d)
    C = torch.zeros(dout, m)
    Q = torch.zeros(dout, d, dtype=torch.uint8)
    P = torch.zeros(dout, 2, dtype=torch.int32)
    calls = [lambda: pkg.lnq_build_fisher(X, G, g),
             lambda: pkg.lnq_init_codebook(W, m),
             lambda: pkg.lnq_quantize_rows(F, W, m, 1, C, Q),
             lambda: pkg.lnq_quantize_rows_diag(Fd, W, m, 1, C, Q),
             lambda: pkg.lnq_objective(F, W, C, Q),
             lambda: pkg.lnq_pack_codes(Q, 2),
             lambda: pkg.lnq_lut_gemv(torch.zeros(1, d), P, C, d)]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()
