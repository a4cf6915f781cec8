"""GPU-versus-oracle parity of the GANQ-style comparison solver (lnq_ganq_rows).

scime.ai summary of GANQ, Approach paragraph (Cholesky / back-substitution assignment, closed-form
least-squares codebook); the reading is the one in the oracle header (R7). Each GPU iteration is
checked against one oracle iteration started from the GPU's own state, following the GPU's
choice only where it is a near-tie (the GPU's sums are fp32 from an fp32 factor).
"""
import numpy as np
import pytest
import torch

from parity_helpers import C_TOL, J_TOL, SCALE_FLOOR, TIE_TOL

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


def ganq_follow_parity(orc, lnq, F, W, m, iters, rows_per_group=None, seed=0, chol=None):
    """init, then `iters` single-iteration GPU calls; after each, sampled rows of every group
    against one oracle iteration from the GPU's start state. Returns a summary."""
    groups, d = F.shape[0], F.shape[1]
    d_out = W.shape[0]
    R = d_out // groups
    rng = np.random.default_rng(seed)
    rows = [np.arange(g * R, (g + 1) * R) if rows_per_group is None or rows_per_group >= R
            else np.sort(rng.choice(np.arange(g * R, (g + 1) * R), rows_per_group, replace=False))
            for g in range(groups)]
    Wh = W.double().cpu().numpy()
    Fh = [F[g].double().cpu().numpy() for g in range(groups)]
    Lh = []
    for g in range(groups):
        if chol is None:
            L, ok = orc.cholesky(Fh[g])
            assert ok
        else:
            L = chol(Fh[g])
        Lh.append(L)
    C, Q = lnq.lnq_init_codebook(W, m)
    J = torch.empty(d_out, dtype=torch.float64, device=W.device)
    st = torch.empty(d_out, dtype=torch.int32, device=W.device)
    summary = {"follows": 0, "changed": 0, "max_c_err": 0.0, "max_J_err": 0.0}
    for it in range(iters):
        C0, Q0 = C.double().cpu().numpy(), Q.cpu().numpy()
        lnq.lnq_ganq_rows(F, W, m, 1, C, Q, J, st)
        torch.cuda.synchronize()
        C1, Q1, J1, st1 = C.double().cpu().numpy(), Q.cpu().numpy(), J.cpu().numpy(), st.cpu().numpy()
        for g in range(groups):
            r = rows[g]
            Jw = np.einsum("ri,ik,rk->r", Wh[r], Fh[g], Wh[r])
            J0 = np.array([orc.objective_row(Fh[g], Wh[j], C0[j], Q0[j]) for j in r])
            band = TIE_TOL * J0 + SCALE_FLOOR * Jw
            Cf, Qf, Jf, stats, status = orc.ganq_iteration(Fh[g], Lh[g], Wh[r], m, C0[r], Q0[r],
                                                           Q_hint=Q1[r], band=band)
            assert int(stats[:, 2].sum()) == 0, \
                f"iteration {it} group {g}: {int(stats[:, 2].sum())} assignment mismatches"
            np.testing.assert_array_equal(Q1[r], Qf)
            np.testing.assert_array_equal(st1[r], status)
            cscale = np.abs(Cf).max(axis=1, keepdims=True)
            cerr = float((np.abs(C1[r] - Cf) / cscale).max())
            Js = np.array([orc.objective_row(Fh[g], Wh[jj], C1[jj], Q1[jj]) for jj in r])
            jerr = float((np.abs(J1[r] - Js) / (Js + SCALE_FLOOR * Jw / J_TOL)).max())
            assert cerr <= C_TOL, f"iteration {it} group {g}: codebook error {cerr:.3e}"
            assert jerr <= J_TOL, f"iteration {it} group {g}: objective error {jerr:.3e}"
            summary["follows"] += int(stats[:, 1].sum())
            summary["changed"] += int(stats[:, 0].sum())
            summary["max_c_err"] = max(summary["max_c_err"], cerr)
            summary["max_J_err"] = max(summary["max_J_err"], jerr)
    return summary, C, Q


@pytest.mark.parametrize("m", [2, 4, 8, 16])
def test_ganq_tiny_layer(orc, lnq, wl, m):
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    summary, _, _ = ganq_follow_parity(orc, lnq, F, W, m, 3)
    assert summary["changed"] > 0


@pytest.mark.parametrize("d_in,d_out,groups", [(1, 3, 1), (37, 8, 2), (300, 66, 3), (1027, 40, 2)])
def test_ganq_ragged_shapes(orc, lnq, d_in, d_out, groups):
    gen = torch.Generator().manual_seed(d_in)
    F = []
    for _ in range(groups):
        X = torch.randn(d_in + 64, d_in, generator=gen, dtype=torch.float64)
        F.append((X.T @ X / (d_in + 64)).float())
    F = torch.stack(F).contiguous().to(_dev())
    W = (torch.randn(d_out, d_in, generator=gen) * 0.02).to(_dev())
    ganq_follow_parity(orc, lnq, F, W, 8, 2)


def test_ganq_q_proj_sampled_rows_and_bit_identity(orc, lnq, wl):
    layer = wl.Q_PROJ
    X, G, W = wl.make_layer(layer, _dev())
    F = lnq.lnq_build_fisher(X, G, layer.groups)
    del X, G
    summary, C, Q = ganq_follow_parity(orc, lnq, F, W, 16, 2, rows_per_group=3,
                                       chol=np.linalg.cholesky)
    assert summary["changed"] > 0
    C2, Q2 = lnq.lnq_init_codebook(W, 16)
    lnq.lnq_ganq_rows(F, W, 16, 2, C2, Q2)
    torch.cuda.synchronize()
    assert torch.equal(C2, C) and torch.equal(Q2, Q)


def test_ganq_group_not_positive_definite(orc, lnq):
    """Group 1's F has a negative diagonal entry: its rows keep their codes and report
    LNQ_ROW_NOT_PD; group 0 is unaffected."""
    gen = torch.Generator().manual_seed(7)
    d, rows = 64, 8
    F = []
    for _ in range(2):
        X = torch.randn(3 * d, d, generator=gen, dtype=torch.float64)
        F.append((X.T @ X).float())
    F[1][10, 10] = -1.0
    F = torch.stack(F).contiguous().to(_dev())
    W = (torch.randn(rows, d, generator=gen) * 0.02).to(_dev())
    C, Q = lnq.lnq_init_codebook(W, 4)
    Q0 = Q.clone()
    st = torch.empty(rows, dtype=torch.int32, device=_dev())
    lnq.lnq_ganq_rows(F, W, 4, 1, C, Q, None, st)
    torch.cuda.synchronize()
    assert torch.all(st[4:] == lnq.LNQ_ROW_NOT_PD)
    assert torch.equal(Q[4:], Q0[4:])
    assert torch.all(st[:4] != lnq.LNQ_ROW_NOT_PD)
    assert not orc.cholesky(F[1].double().cpu().numpy())[1]
