"""GPU-versus-oracle parity through the C ABI (needs a B200 and the built library).

Fisher blocks: "GuidedQuant" blog post, GuidedQuant section (third equation, grouping sentence).
LNQ: same post, LNQ section (problem and iteration). Tolerances are in parity_helpers.
"""
import numpy as np
import pytest
import torch

from parity_helpers import (check_fisher_full, check_fisher_sampled, lnq_follow_parity, J_TOL)

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


def _dev():
    return torch.device("cuda:0")


# --------------------------------------------------------------------------------- Fisher

def test_fisher_tiny_layer_full(orc, lnq, wl):
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    check_fisher_full(orc, F, X, G, layer.groups)


@pytest.mark.parametrize("n,d_in,d_out,groups,guided", [
    (200, 136, 6, 3, True),    # ragged n and d_in (one partial row block and column block)
    (77, 8, 4, 1, True),       # smallest d_in
    (64, 264, 5, 1, False),    # unguided, ragged
    (1, 64, 2, 2, True),       # a single token
    (130, 512, 8, 8, True),    # 4 x 2 tile grid, diagonal and off-diagonal tiles
    (1000, 392, 12, 4, True),
])
def test_fisher_ragged_shapes(orc, lnq, wl, n, d_in, d_out, groups, guided):
    layer = wl.scaled(wl.TINY, n=n, d_in=d_in, d_out=d_out, groups=groups,
                      x_outlier_cols=min(4, d_in), g_kind="normal" if guided else "ones")
    X, G, _ = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, groups)
    check_fisher_full(orc, F, X, G, groups)


def test_fisher_unit_gradients_and_alpha(orc, lnq, wl):
    layer = wl.scaled(wl.TINY, n=333, d_in=200, d_out=16, groups=1)
    X, _, _ = wl.make_layer(layer, _dev())
    F0 = lnq.lnq_build_fisher(X, None, 1)
    ones = torch.ones((layer.n, layer.d_out), dtype=torch.bfloat16, device=_dev())
    F1 = lnq.lnq_build_fisher(X, ones, 1)       # the guided (fp16 operand) path with s == 1
    torch.cuda.synchronize()
    Xh = X.double().cpu().numpy()
    ref = Xh.T @ Xh                        # library matmul, independent of the oracle
    dg = np.sqrt(np.outer(np.diag(ref), np.diag(ref)))
    assert np.max(np.abs(F0[0].double().cpu().numpy() - ref) / dg) < 1e-5   # exact bf16 inputs
    assert np.max(np.abs(F1[0].double().cpu().numpy() - ref) / dg) < 1e-5   # power-of-2 scaling
    Fa = lnq.lnq_build_fisher(X, None, 1, alpha=1.0 / layer.n)
    check_fisher_full(orc, Fa, X, None, 1, alpha=1.0 / layer.n)


def test_fisher_symmetric(lnq, wl):
    layer = wl.scaled(wl.TINY, n=500, d_in=392, d_out=12, groups=3)
    X, G, _ = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, 3)
    assert torch.equal(F, F.transpose(1, 2))


def test_fisher_q_proj_full_size_sampled(orc, lnq, wl):
    layer = wl.Q_PROJ
    X, G, _ = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    check_fisher_sampled(orc, F, X, G, layer.groups, tiles_per_group=6)


def test_fisher_down_proj_full_size_sampled(orc, lnq, wl):
    """Unguided layer at d_in = 11008 (all gradients 1, one group): F = X^T X."""
    layer = wl.DOWN_PROJ
    X, G, _ = wl.make_layer(layer, _dev())
    assert G is None and layer.groups == 1
    F = lnq.lnq_build_fisher(X, None, 1)
    check_fisher_sampled(orc, F, X, None, 1, tiles_per_group=6)


def test_fisher_up_proj_full_size_sampled(orc, lnq, wl):
    """Eight guided groups over 65536 tokens; the first, a middle and the last group are sampled."""
    layer = wl.UP_PROJ
    X, G, _ = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    check_fisher_sampled(orc, F, X, G, layer.groups, tiles_per_group=3,
                         check_groups=[0, layer.groups // 2, layer.groups - 1])


# --------------------------------------------------------------------------------- LNQ

def test_lnq_tiny_layer_all_rows(orc, lnq, wl):
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    summary, _, _ = lnq_follow_parity(orc, lnq, F, W, layer.m, layer.iters)
    assert summary["moves"] > 0


def test_lnq_resume_is_bit_identical(lnq, wl):
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    C, Q = lnq.lnq_init_codebook(W, layer.m)
    Ca, Qa = C.clone(), Q.clone()
    lnq.lnq_quantize_rows(F, W, layer.m, 3, C, Q)
    lnq.lnq_quantize_rows(F, W, layer.m, 1, Ca, Qa)
    lnq.lnq_quantize_rows(F, W, layer.m, 2, Ca, Qa)
    torch.cuda.synchronize()
    assert torch.equal(C, Ca) and torch.equal(Q, Qa)


def test_lnq_q_proj_full_size_sampled_rows(orc, lnq, wl):
    layer = wl.Q_PROJ
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    del X, G
    summary, _, _ = lnq_follow_parity(orc, lnq, F, W, layer.m, layer.iters, rows_per_group=16)
    assert summary["moves"] > 0


def test_lnq_q_proj_one_call_equals_one_iteration_calls(lnq, wl):
    """The bench's form of the call (all iterations and the objective in one lnq_quantize_rows)
    ends bit for bit in the state of one-iteration calls, whose every step the follow-mode test
    above checks against the oracle: 32 sweep windows, so the per-window move flags of one call
    carry nothing into the next iteration."""
    layer = wl.Q_PROJ
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    del X, G
    C, Q = lnq.lnq_init_codebook(W, layer.m)
    Ca, Qa = C.clone(), Q.clone()
    J = torch.empty(W.shape[0], dtype=torch.float64, device=W.device)
    Ja = torch.empty_like(J)
    lnq.lnq_quantize_rows(F, W, layer.m, layer.iters, C, Q, J)
    for _ in range(layer.iters):
        lnq.lnq_quantize_rows(F, W, layer.m, 1, Ca, Qa, Ja)
    torch.cuda.synchronize()
    assert torch.equal(C, Ca) and torch.equal(Q, Qa) and torch.equal(J, Ja)


def test_lnq_down_proj_full_size_sampled_rows(orc, lnq, wl):
    """d_in = 11008 (86 sweep windows, a ragged last one), m = 8, four iterations, one group."""
    layer = wl.DOWN_PROJ
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    del X, G
    summary, _, _ = lnq_follow_parity(orc, lnq, F, W, layer.m, layer.iters, rows_per_group=6)
    assert summary["moves"] > 0


def test_lnq_up_proj_full_size_sampled_rows(orc, lnq, wl):
    """d_out = 14336 in eight groups of 1792 rows, m = 4, five iterations."""
    layer = wl.UP_PROJ
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    del X, G
    summary, _, _ = lnq_follow_parity(orc, lnq, F, W, layer.m, layer.iters, rows_per_group=3)
    assert summary["moves"] > 0


@pytest.mark.parametrize("d_in", [100, 256, 300, 1000, 1500, 4096, 6000, 11008])
def test_init_every_sort_width(orc, lnq, d_in):
    """Init is bit-exact against the oracle for every sort layout: the shared-memory sort
    (d_in < 256) and the register sort with 1 to 64 keys per thread (p2 / 256)."""
    g = torch.Generator(device="cpu").manual_seed(d_in)
    W = (torch.randn(12, d_in, generator=g) * 0.02)
    W[:, : d_in // 5] = torch.round(W[:, : d_in // 5] * 200) / 200   # ties among the weights
    for m in (4, 16):
        C, Q = lnq.lnq_init_codebook(W.to(_dev()), m)
        torch.cuda.synchronize()
        Ch, Qh = C.double().cpu().numpy(), Q.cpu().numpy()
        Wh = W.double().numpy()
        for j in range(W.shape[0]):
            c0, q0 = orc.init_row(Wh[j], m)
            np.testing.assert_array_equal(Ch[j], c0.astype(np.float32).astype(np.float64))
            np.testing.assert_array_equal(Qh[j], q0)


@pytest.mark.parametrize("m", [2, 4, 8, 16])
def test_lnq_every_codebook_size(orc, lnq, wl, m):
    layer = wl.scaled(wl.TINY, d_in=96, d_out=8, n=300, groups=2, m=m)
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    lnq_follow_parity(orc, lnq, F, W, m, 3)


@pytest.mark.parametrize("m,d_in,d_out,groups", [
    (2, 300, 72, 2),     # three windows, ragged last one; 36 rows per group (a ragged row block)
    (4, 517, 40, 1),     # odd d_in: unaligned rows, scalar paths, ragged K block
    (8, 640, 48, 3),     # five full windows
    (16, 1000, 34, 2),   # eight windows, 17 rows per group
])
def test_lnq_multi_window_shapes(orc, lnq, wl, m, d_in, d_out, groups):
    # Several 128-coordinate windows, so the left-looking product over earlier moves (tensor
    # cores, fp16 pieces, history copies) and the window hand-over all take part; every row is
    # checked against the oracle in follow mode for two iterations.
    layer = wl.scaled(wl.TINY, d_in=d_in, d_out=d_out, n=640, groups=groups, m=m)
    X, G, W = wl.make_layer(layer, _dev())
    # the Fisher build takes d_in % 8 == 0: build on X padded with zero columns and keep the
    # leading d_in x d_in block, which is X^T diag(s) X of the real columns
    pad = (-d_in) % 8
    Xp = torch.cat([X, torch.zeros(X.shape[0], pad, dtype=X.dtype, device=X.device)], dim=1)
    F = lnq.lnq_build_fisher(Xp, G, layer.groups)[:, :d_in, :d_in].contiguous()
    summary, _, _ = lnq_follow_parity(orc, lnq, F, W, m, 2)
    assert summary["moves"] > 0


def test_lnq_empty_codewords_and_tiny_rows(orc, lnq, wl):
    # Rows with only 3 distinct values and m = 8 leave codewords empty; d_in = 5 is not a
    # multiple of anything.
    torch.manual_seed(0)
    d, d_out, m = 5, 4, 8
    A = torch.randn(20, d, dtype=torch.float64)
    F = (A.T @ A).float().unsqueeze(0).contiguous().to(_dev())
    W = torch.tensor([[0.1, 0.1, 0.2, 0.2, 0.3]] * d_out, dtype=torch.float32)
    W[1] = torch.tensor([1.0, -1.0, 0.5, 0.25, 0.0])
    W = W.to(_dev())
    lnq_follow_parity(orc, lnq, F, W, m, 3)


def test_lnq_singular_rows(orc, lnq):
    # Coordinates 0..3 see an all-zero block of F, so any codeword used only there has a zero
    # pivot: the row keeps its codebook and reports LNQ_ROW_SINGULAR, exactly as the oracle.
    d, m = 16, 4
    torch.manual_seed(1)
    A = torch.randn(40, d, dtype=torch.float64)
    F = A.T @ A
    F[:4, :] = 0
    F[:, :4] = 0
    F = F.float().unsqueeze(0).contiguous().to(_dev())
    W = torch.cat([torch.full((1, 4), 5.0), torch.randn(1, d - 4) * 0.01], dim=1).to(_dev())
    W = W.float().contiguous()
    st = torch.empty(1, dtype=torch.int32, device=_dev())
    C, Q = lnq.lnq_init_codebook(W, m)
    C0 = C.clone()
    lnq.lnq_quantize_rows(F, W, m, 1, C, Q, None, st)
    torch.cuda.synchronize()
    Fh = F[0].double().cpu().numpy()
    c_or, status = orc.codebook_row(Fh, W[0].double().cpu().numpy(), Q.cpu().numpy()[0],
                                    C0[0].double().cpu().numpy())
    assert status == 1 and int(st[0]) == 1
    assert torch.equal(C, C0)


# ----------------------------------------------------------------- LNQ, diagonal Fisher blocks

def _fisher_diagonal(lnq, wl, layer):
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    Fd = torch.diagonal(F, dim1=1, dim2=2).contiguous()
    return Fd, W


@pytest.mark.parametrize("m", [2, 4, 8, 16])
def test_lnq_diag_tiny_layer_every_codebook_size(orc, lnq, wl, m):
    Fd, W = _fisher_diagonal(lnq, wl, wl.TINY)
    summary, _, _ = lnq_follow_parity(orc, lnq, Fd, W, m, 3, diag=True)
    assert summary["moves"] > 0


@pytest.mark.parametrize("d_in,d_out,groups", [(1, 3, 1), (5, 4, 2), (300, 66, 3), (1027, 40, 2)])
def test_lnq_diag_ragged_shapes(orc, lnq, d_in, d_out, groups):
    # d_in not a multiple of 8 (the Fisher build's rule), so log-normal weights stand in for the
    # Fisher diagonal
    gen = torch.Generator().manual_seed(d_in)
    Fd = torch.exp(torch.randn(groups, d_in, generator=gen)).to(_dev())
    W = (torch.randn(d_out, d_in, generator=gen) * 0.02).to(_dev())
    lnq_follow_parity(orc, lnq, Fd, W, 8, 3, diag=True)


def test_lnq_diag_q_proj_full_size_sampled_rows(orc, lnq, wl):
    Fd, W = _fisher_diagonal(lnq, wl, wl.Q_PROJ)
    summary, C, Q = lnq_follow_parity(orc, lnq, Fd, W, 16, 3, rows_per_group=16, diag=True)
    assert summary["moves"] > 0
    # run to run: bit-identical, and two calls of one iteration equal one call of two
    C2, Q2 = lnq.lnq_init_codebook(W, 16)
    C3, Q3 = C2.clone(), Q2.clone()
    lnq.lnq_quantize_rows_diag(Fd, W, 16, 3, C2, Q2)
    lnq.lnq_quantize_rows_diag(Fd, W, 16, 1, C3, Q3)
    lnq.lnq_quantize_rows_diag(Fd, W, 16, 2, C3, Q3)
    torch.cuda.synchronize()
    assert torch.equal(C2, C) and torch.equal(Q2, Q)
    assert torch.equal(C3, C) and torch.equal(Q3, Q)


def test_lnq_diag_small_weight_class(orc, lnq):
    # A class whose weights f_i are 1e-9 of the row's largest: its fixed-point f sum is too coarse
    # (mean f under 2^-17 of the largest), so the kernel sums that class directly in fp64; the
    # codebook must still match the oracle's weighted mean to the usual tolerance.
    gen = torch.Generator().manual_seed(11)
    d, rows = 64, 4
    f = torch.ones(1, d)
    f[0, 48:] = 1e-9
    W = torch.randn(rows, d, generator=gen) * 0.01
    W[:, 48:] += 5.0
    lnq_follow_parity(orc, lnq, f.to(_dev()), W.contiguous().to(_dev()), 4, 3, diag=True)


def test_lnq_diag_mixed_sign_weights(orc, lnq):
    # f_i < 0 on a tenth of the coordinates (small in size, so the rows keep J > 0): those
    # coordinates take the codeword with the most negative fp64 change, the rest their nearest.
    gen = torch.Generator().manual_seed(12)
    d, rows, groups = 256, 8, 2
    f = torch.exp(torch.randn(groups, d, generator=gen))
    neg = torch.rand(groups, d, generator=gen) < 0.1
    f[neg] = -0.0005 * f[neg]
    W = torch.randn(rows, d, generator=gen) * 0.02
    summary, _, _ = lnq_follow_parity(orc, lnq, f.to(_dev()), W.to(_dev()), 8, 3, diag=True)
    assert summary["moves"] > 0


def test_lnq_diag_singular_rows(orc, lnq):
    # Row 0 (group 0): f = 0 on coordinates 0..3, which hold the row's only large values, so a
    # codeword used only there has no weight: the row keeps its codebook and reports
    # LNQ_ROW_SINGULAR. Row 1 (group 1) has positive weights everywhere and is not singular.
    d, m = 16, 4
    torch.manual_seed(1)
    f = torch.rand(2, d, dtype=torch.float32) + 0.5
    f[0, :4] = 0
    Fd = f.to(_dev())
    W = torch.cat([torch.full((2, 4), 5.0), torch.randn(2, d - 4) * 0.01], dim=1)
    W[1, :4] = torch.randn(4) * 0.01
    W = W.float().contiguous().to(_dev())
    st = torch.empty(2, dtype=torch.int32, device=_dev())
    J = torch.empty(2, dtype=torch.float64, device=_dev())
    C, Q = lnq.lnq_init_codebook(W, m)
    C0, Q0 = C.clone(), Q.clone()
    lnq.lnq_quantize_rows_diag(Fd, W, m, 1, C, Q, J, st)
    torch.cuda.synchronize()
    Fh = [np.diag(f[j].double().numpy()) for j in range(2)]
    for j, want in ((0, 1), (1, 0)):
        c_or, status = orc.codebook_row(Fh[j], W[j].double().cpu().numpy(), Q0.cpu().numpy()[j],
                                        C0[j].double().cpu().numpy())
        assert status == want and int(st[j]) == want
    assert torch.equal(C[0], C0[0])
    # the sweep still ran with the kept codebook: every coordinate with f > 0 is at its nearest
    # codeword, and the reported objective is the oracle's of the final state
    Ch, Qh, Wh = C.double().cpu().numpy(), Q.cpu().numpy(), W.double().cpu().numpy()
    for j in range(2):
        Jo = orc.objective_row(Fh[j], Wh[j], Ch[j], Qh[j])
        assert abs(float(J[j]) - Jo) <= J_TOL * Jo + 1e-30
        for i in range(4, d):
            assert abs(Ch[j][Qh[j][i]] - Wh[j][i]) <= np.abs(Ch[j] - Wh[j][i]).min()


def test_objective_entry_point(orc, lnq, wl):
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    C, Q = lnq.lnq_init_codebook(W, layer.m)
    lnq.lnq_quantize_rows(F, W, layer.m, 2, C, Q)
    J = lnq.lnq_objective(F, W, C, Q)
    torch.cuda.synchronize()
    Fh, Wh, Ch, Qh = (F.double().cpu().numpy(), W.double().cpu().numpy(),
                      C.double().cpu().numpy(), Q.cpu().numpy())
    R = layer.rows_per_group
    for j in range(layer.d_out):
        Jo = orc.objective_row(Fh[j // R], Wh[j], Ch[j], Qh[j])
        assert abs(J[j].item() - Jo) <= J_TOL * Jo


# --------------------------------------------------------------------------------- failures

def test_wait_limit_zero_reports_timeout_and_recovers(lnq, wl):
    """Every in-kernel wait gives up at once: the call reports a timeout through the workspace
    flag, the context stays usable, and the next call with the default limit is correct."""
    from post_weight_quantization_guided_b200 import binding as b
    layer = wl.scaled(wl.TINY, n=512, d_in=256, d_out=8, groups=2)
    X, G, _ = wl.make_layer(layer, _dev())
    ws = b.workspace(b.LNQ_OP_BUILD_FISHER, layer.n, layer.d_in, layer.d_out, layer.groups)
    try:
        b.lnq_set_wait_limit(0)
        lnq.lnq_build_fisher(X, G, layer.groups, ws=ws)
        assert b.lnq_workspace_check(ws) == b.LNQ_ERR_TIMEOUT
    finally:
        b.lnq_set_wait_limit(-1)
    F = lnq.lnq_build_fisher(X, G, layer.groups, ws=ws)
    assert b.lnq_workspace_check(ws) == b.LNQ_OK
    F2 = lnq.lnq_build_fisher(X, G, layer.groups)
    torch.cuda.synchronize()
    assert torch.equal(F, F2)


# --------------------------------------------------------------------------------- consumer

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d_out,d_in,nb", [(37, 1, 1), (64, 100, 3), (130, 1027, 8),
                                           (4096, 4096, 1)])
def test_lut_pack_and_gemv(orc, lnq, bits, d_out, d_in, nb):
    """Packed words bit-exact against the oracle's packing; y = x W^T within 1e-5 of
    sum_i |x_i c_q| (fp32 sums of at most ~130 terms per lane, then a 5-level tree); bit-identical
    on a second run."""
    m = 1 << bits
    g = torch.Generator().manual_seed(bits * 7919 + d_in)
    Q = torch.randint(0, m, (d_out, d_in), generator=g, dtype=torch.uint8)
    C = torch.randn(d_out, m, generator=g)
    x = torch.randn(nb, d_in, generator=g)
    P = lnq.lnq_pack_codes(Q.to(_dev()), bits)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(P.cpu().numpy().view(np.uint32), orc.pack_codes(Q.numpy(), bits))
    y = lnq.lnq_lut_gemv(x.to(_dev()), P, C.to(_dev()), d_in)
    y2 = lnq.lnq_lut_gemv(x.to(_dev()), P, C.to(_dev()), d_in)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    Qn, Cn, xn = Q.numpy(), C.double().numpy(), x.double().numpy()
    yo = orc.lut_gemv(xn, Cn, Qn)
    W_hat = np.take_along_axis(Cn, Qn.astype(np.int64), axis=1)
    scale = np.abs(xn) @ np.abs(W_hat).T
    err = np.abs(y.double().cpu().numpy() - yo)
    assert np.all(err <= 1e-5 * scale + 1e-30), float((err / (scale + 1e-30)).max())


@pytest.mark.parametrize("case", ["many_row_blocks_and_slices", "unaligned_words"])
def test_lut_gemv_large_and_unaligned(orc, lnq, case):
    """Several row blocks per CTA and several K slices per lane (3000 x 16384), and packed words
    that start off a 16-byte boundary."""
    bits, nb = 4, 2
    d_out, d_in = (3000, 16384) if case == "many_row_blocks_and_slices" else (300, 1000)
    m = 1 << bits
    g = torch.Generator().manual_seed(91 + d_in)
    Q = torch.randint(0, m, (d_out, d_in), generator=g, dtype=torch.uint8)
    C = torch.randn(d_out, m, generator=g)
    x = torch.randn(nb, d_in, generator=g)
    P = lnq.lnq_pack_codes(Q.to(_dev()), bits)
    if case == "unaligned_words":
        buf = torch.empty(P.numel() + 1, dtype=P.dtype, device=P.device)
        buf[1:].copy_(P.reshape(-1))
        P = buf[1:].view(P.shape)
        assert P.data_ptr() % 16 != 0
    y = lnq.lnq_lut_gemv(x.to(_dev()), P, C.to(_dev()), d_in)
    torch.cuda.synchronize()
    Qn, Cn, xn = Q.numpy(), C.double().numpy(), x.double().numpy()
    yo = orc.lut_gemv(xn, Cn, Qn)
    W_hat = np.take_along_axis(Cn, Qn.astype(np.int64), axis=1)
    scale = np.abs(xn) @ np.abs(W_hat).T
    err = np.abs(y.double().cpu().numpy() - yo)
    assert np.all(err <= 1e-5 * scale + 1e-30), float((err / (scale + 1e-30)).max())


def test_lut_gemv_on_a_quantised_layer(orc, lnq, wl):
    """The consumer on the tiny layer's own LNQ result (C, Q after three iterations)."""
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    C, Q = lnq.lnq_init_codebook(W, layer.m)
    lnq.lnq_quantize_rows(F, W, layer.m, layer.iters, C, Q)
    bits = layer.m.bit_length() - 1
    P = lnq.lnq_pack_codes(Q, bits)
    y = lnq.lnq_lut_gemv(X[:5].float().contiguous(), P, C, layer.d_in)
    torch.cuda.synchronize()
    xn = X[:5].double().cpu().numpy()
    yo = orc.lut_gemv(xn, C.double().cpu().numpy(), Q.cpu().numpy())
    W_hat = np.take_along_axis(C.double().cpu().numpy(), Q.cpu().numpy().astype(np.int64), axis=1)
    scale = np.abs(xn) @ np.abs(W_hat).T
    assert np.all(np.abs(y.double().cpu().numpy() - yo) <= 1e-5 * scale + 1e-30)
