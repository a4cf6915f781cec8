"""Comparison helpers for the GPU-versus-oracle parity tests.

Tolerances (per entry unless stated), from the accuracy targets of the hot path:
  F          |F_gpu - F_oracle| <= 1e-3 * sqrt(F_ii F_kk)  (bf16 operands, fp32 accumulation)
  codebook   |c_gpu - c_oracle| <= 1e-4 * max_q |c_oracle|  (per row)
  objective  |J_gpu - J_oracle(same state)| <= 1e-5 * J: the GPU's reported objective against
             the oracle's objective of the GPU's own (C, Q). Along the trajectory the oracle keeps
             its fp64 codebook, which may differ from the fp32 one within the codebook tolerance,
             and J follows that difference to first order: there J agrees within 1e-4.
  indices    identical, except where the oracle's best two candidates are within 1e-6 * J
             (the oracle then follows the GPU's choice and counts it; any other difference is a
             mismatch and fails)
LNQ parity feeds both sides the GPU's F (widened to fp64), so the F budget does not leak into the
LNQ budgets.
"""
from __future__ import annotations

import numpy as np
import torch

F_TOL = 1e-3
C_TOL = 1e-4
J_TOL = 1e-5
J_TRAJ_TOL = 1e-4
TIE_TOL = 1e-6
# Absolute floor of the tie band and of the objective tolerance, relative to the row's scale
# w^T F w. It only matters when a row's objective reaches ~0 (an exactly representable row), where
# equal-valued codewords make several assignments equally correct.
SCALE_FLOOR = 1e-12


def group_scales_oracle(orc, G: torch.Tensor, groups: int, g: int, chunk: int = 8192):
    """s_g over all tokens, from the oracle, reading G (on any device) one row chunk at a time."""
    n, d_out = G.shape
    R = d_out // groups
    out = np.empty(n)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        Gh = G[r0:r1, g * R:(g + 1) * R].double().cpu().numpy()
        out[r0:r1] = orc.group_scales(Gh, r1 - r0, R, 1)[0]
    return out


def check_fisher_full(orc, F: torch.Tensor, X: torch.Tensor, G, groups: int, alpha=1.0):
    Xh = X.double().cpu().numpy()
    Gh = None if G is None else G.double().cpu().numpy()
    Fo = orc.fisher_full(Xh, Gh, groups, alpha)
    Fg = F.double().cpu().numpy()
    worst = 0.0
    for g in range(groups):
        dg = np.sqrt(np.outer(np.diag(Fo[g]), np.diag(Fo[g])))
        dg[dg == 0] = 1e-300
        err = np.abs(Fg[g] - Fo[g]) / dg
        worst = max(worst, float(err.max()))
    assert worst <= F_TOL, f"F relative error {worst:.3e} > {F_TOL}"
    return worst


def check_fisher_sampled(orc, F: torch.Tensor, X: torch.Tensor, G, groups: int, alpha=1.0,
                         tiles_per_group=8, tile=64, seed=0, check_groups=None):
    """Full diagonal plus random tiles (always including one on the diagonal and one touching the
    last, possibly ragged, columns) of every group (or of the groups in check_groups)."""
    n, d = X.shape
    rng = np.random.default_rng(seed)
    worst = 0.0
    for g in (range(groups) if check_groups is None else check_groups):
        s = np.ones(n) if G is None else group_scales_oracle(orc, G, groups, g)
        diag = np.empty(d)
        for c0 in range(0, d, 512):
            c1 = min(d, c0 + 512)
            diag[c0:c1] = orc.fisher_diag(X[:, c0:c1].double().cpu().numpy(), s, alpha)
        Fd = torch.diagonal(F[g]).double().cpu().numpy()
        err = np.abs(Fd - diag) / diag
        worst = max(worst, float(err.max()))
        starts = [(0, 0), (max(0, d - tile), max(0, d - tile))]
        while len(starts) < tiles_per_group:
            starts.append((int(rng.integers(0, d - tile + 1)), int(rng.integers(0, d - tile + 1))))
        for i0, k0 in starts[:tiles_per_group]:
            I, K = slice(i0, min(d, i0 + tile)), slice(k0, min(d, k0 + tile))
            blk = orc.fisher_block(X[:, I].double().cpu().numpy(), X[:, K].double().cpu().numpy(),
                                   s, alpha)
            got = F[g, I, K].double().cpu().numpy()
            dg = np.sqrt(np.outer(diag[I], diag[K]))
            worst = max(worst, float((np.abs(got - blk) / dg).max()))
    assert worst <= F_TOL, f"F relative error {worst:.3e} > {F_TOL}"
    return worst


def lnq_follow_parity(orc, lnq, F: torch.Tensor, W: torch.Tensor, m: int, iters: int,
                      rows_per_group=None, seed=0, nthreads=0, diag=False):
    """Runs init and then `iters` single-iteration calls of the GPU path on every row, and checks
    sampled rows of each group against the oracle in follow mode after every step.
    diag=True: F is [groups][d] (the diagonals), the GPU step is lnq_quantize_rows_diag and the
    oracle runs its ordinary LNQ on the dense matrix diag(F[g]).
    Returns a summary dict."""
    groups, d = F.shape[0], F.shape[1]
    d_out = W.shape[0]
    R = d_out // groups
    rng = np.random.default_rng(seed)
    if rows_per_group is None or rows_per_group >= R:
        rows = [np.arange(g * R, (g + 1) * R) for g in range(groups)]
    else:
        rows = [np.sort(rng.choice(np.arange(g * R, (g + 1) * R), rows_per_group, replace=False))
                for g in range(groups)]
    Wh = W.double().cpu().numpy()
    C, Q = lnq.lnq_init_codebook(W, m)
    torch.cuda.synchronize()
    Ch, Qh = C.double().cpu().numpy(), Q.cpu().numpy()
    for g in range(groups):
        for j in rows[g]:
            c0, q0 = orc.init_row(Wh[j], m)
            np.testing.assert_array_equal(Ch[j], c0.astype(np.float32).astype(np.float64))
            np.testing.assert_array_equal(Qh[j], q0)
    J = torch.empty(d_out, dtype=torch.float64, device=W.device)
    st = torch.empty(d_out, dtype=torch.int32, device=W.device)
    summary = {"follows": 0, "moves": 0, "rows": int(sum(len(r) for r in rows)),
               "max_c_err": 0.0, "max_J_err": 0.0, "max_J_same_state_err": 0.0}
    Fh = [None] * groups
    for it in range(iters):
        C0, Q0 = C.double().cpu().numpy(), Q.cpu().numpy()
        if diag:
            lnq.lnq_quantize_rows_diag(F, W, m, 1, C, Q, J, st)
        else:
            lnq.lnq_quantize_rows(F, W, m, 1, C, Q, J, st)
        torch.cuda.synchronize()
        C1, Q1 = C.double().cpu().numpy(), Q.cpu().numpy()
        J1, st1 = J.cpu().numpy(), st.cpu().numpy()
        for g in range(groups):
            if Fh[g] is None:
                Fh[g] = F[g].double().cpu().numpy()
                if diag:
                    Fh[g] = np.diag(Fh[g])
            r = rows[g]
            Jw = np.einsum("ri,ik,rk->r", Wh[r], Fh[g], Wh[r])
            Cf, Qf, Jf, stats, status = orc.follow_iteration(Fh[g], Wh[r], m, C0[r], Q0[r], Q1[r],
                                                             TIE_TOL, nthreads,
                                                             tie_abs=SCALE_FLOOR * Jw)
            assert int(stats[:, 2].sum()) == 0, \
                f"iteration {it} group {g}: {int(stats[:, 2].sum())} assignment mismatches"
            np.testing.assert_array_equal(Q1[r], Qf)
            np.testing.assert_array_equal(st1[r], status)
            cscale = np.abs(Cf).max(axis=1, keepdims=True)
            cerr = float((np.abs(C1[r] - Cf) / cscale).max())
            jerr = float((np.abs(J1[r] - Jf) / (Jf + SCALE_FLOOR * Jw / J_TOL)).max())
            # the oracle's objective of the GPU's own state (its fp32 codebook and assignment)
            Js = np.array([orc.objective_row(Fh[g], Wh[jj], C1[jj], Q1[jj]) for jj in r])
            serr = float((np.abs(J1[r] - Js) / (Js + SCALE_FLOOR * Jw / J_TOL)).max())
            assert cerr <= C_TOL, f"iteration {it} group {g}: codebook error {cerr:.3e}"
            assert serr <= J_TOL, f"iteration {it} group {g}: objective error {serr:.3e}"
            assert jerr <= J_TRAJ_TOL, f"iteration {it} group {g}: trajectory objective {jerr:.3e}"
            summary["follows"] += int(stats[:, 1].sum())
            summary["moves"] += int(stats[:, 0].sum())
            summary["max_c_err"] = max(summary["max_c_err"], cerr)
            summary["max_J_err"] = max(summary["max_J_err"], jerr)
            summary["max_J_same_state_err"] = max(summary["max_J_same_state_err"], serr)
    return summary, C, Q
