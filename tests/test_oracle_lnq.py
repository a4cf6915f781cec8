"""Pins for the oracle's LNQ routines, each against something other than the oracle itself.

Passages: "GuidedQuant" blog post, LNQ section -- the per-row problem (one-hot P, codebook c,
objective ||Xw - XPc||^2 = (Pc - w)^T H (Pc - w)) and the iteration "repeat: codebook
c <- (P^T H P)^-1 P^T H w; for i = 1..d_in: assignment argmin over {c_1..c_m}"; the descent
claims in that section and in the GuidedQuant abstract (aitopics "squeezellm" tag page).
Readings where the pages are silent (initial codebook, tie-breaks, empty codewords) are the ones
stated in the oracle's header.
"""
import itertools

import numpy as np
import pytest

from conftest import golden
from post_weight_quantization_guided_b200 import workloads as wl


def _onehot(q, m):
    P = np.zeros((len(q), m))
    P[np.arange(len(q)), q] = 1.0
    return P


def _J(F, w, c, q):
    r = c[q] - w
    return float(r @ F @ r)


def _tiny_row_problem(orc, seed=0, d=128, m=8, groups=4, g=1):
    layer = wl.TINY
    X, G, W = wl.make_layer(layer, "cpu")
    X, G, W = X.double().numpy(), G.double().numpy(), W.double().numpy()
    F = orc.fisher_full(X, G, layer.groups)[g]
    return F, W[g * layer.rows_per_group:(g + 1) * layer.rows_per_group]


# ----------------------------------------------------------------------------------- goldens

def test_hand_worked_lnq_golden(orc):
    g = golden("lnq_hand_d3_m2.json")
    F, w, m = np.array(g["F"], float), np.array(g["w"]), g["m"]
    c, q = orc.init_row(w, m)
    np.testing.assert_array_equal(c, g["init"]["c"])
    np.testing.assert_array_equal(q, g["init"]["q"])
    assert orc.objective_row(F, w, c, q) == g["init"]["J"]
    cb = g["codebook_after_init"]
    c1, st = orc.codebook_row(F, w, q, c)
    assert st == 0
    np.testing.assert_allclose(c1, np.array(cb["c_num"]) / cb["c_den"], rtol=1e-15)
    assert abs(orc.objective_row(F, w, c1, q) - cb["J_num"] / cb["J_den"]) < 1e-15
    q1, J1, stats, _ = orc.sweep_row(F, w, c1, q)
    np.testing.assert_array_equal(q1, g["sweep_after_codebook"]["q"])
    assert stats["moves"] == g["sweep_after_codebook"]["moves"]
    sm = g["sweep_with_moves"]
    q2, J2, stats2, trace = orc.sweep_row(F, w, np.array(sm["c"]), np.array(sm["q_start"]),
                                          trace=True)
    np.testing.assert_array_equal(q2, sm["q_end"])
    np.testing.assert_allclose(trace, sm["J_trace"], rtol=0, atol=1e-12)
    C, Q, Jh, status = orc.lnq_rows(F, w[None], m, iters=3)
    assert abs(Jh[0, -1] - g["optimum_J_num"] / g["optimum_J_den"]) < 1e-14


# ----------------------------------------------------------------------------------- init

def test_init_is_sorted_quantiles_and_nearest(orc):
    rng = np.random.default_rng(5)
    for d, m in ((128, 8), (100, 16), (37, 4), (2, 2), (4096, 16)):
        w = rng.standard_normal(d) * 0.02
        c, q = orc.init_row(w, m)
        srt = np.sort(w)
        ref_c = np.array([srt[((2 * k + 1) * d) // (2 * m)] for k in range(m)])
        np.testing.assert_array_equal(c, ref_c)
        ref_q = np.argmin(np.abs(w[:, None] - ref_c[None, :]), axis=1)   # first minimum
        np.testing.assert_array_equal(q, ref_q)


def test_init_ties_go_to_lower_index(orc):
    w = np.array([0.0, 1.0, 2.0, 3.0])     # m=2: c = sorted[1], sorted[3] = 1, 3
    c, q = orc.init_row(w, 2)
    np.testing.assert_array_equal(c, [1.0, 3.0])
    np.testing.assert_array_equal(q, [0, 0, 0, 1])   # w=2 is equidistant -> index 0


# ----------------------------------------------------------------------------------- codebook

def test_codebook_satisfies_normal_equations(orc):
    F, W = _tiny_row_problem(orc)
    for j in range(4):
        w = W[j]
        c0, q = orc.init_row(w, 8)
        c, st = orc.codebook_row(F, w, q, c0)
        assert st == 0
        P = _onehot(q, 8)
        M, b = P.T @ F @ P, P.T @ F @ w
        nz = P.sum(0) > 0
        res = M[np.ix_(nz, nz)] @ c[nz] - b[nz]
        assert np.abs(res).max() <= 1e-12 * np.abs(b[nz]).max()


def test_codebook_identity_F_gives_cluster_means(orc):
    rng = np.random.default_rng(1)
    d, m = 64, 4
    w = rng.standard_normal(d)
    q = rng.integers(0, m, d).astype(np.uint8)
    c, st = orc.codebook_row(np.eye(d), w, q, np.zeros(m))
    assert st == 0
    for k in range(m):
        np.testing.assert_allclose(c[k], w[q == k].mean(), rtol=1e-13)


def test_codebook_diagonal_F_gives_weighted_means(orc):
    rng = np.random.default_rng(2)
    d, m = 50, 4
    w = rng.standard_normal(d)
    f = rng.uniform(0.5, 3.0, d)
    q = rng.integers(0, m, d).astype(np.uint8)
    c, st = orc.codebook_row(np.diag(f), w, q, np.zeros(m))
    for k in range(m):
        sel = q == k
        np.testing.assert_allclose(c[k], (f[sel] * w[sel]).sum() / f[sel].sum(), rtol=1e-13)


def test_codebook_single_codeword_closed_form(orc):
    rng = np.random.default_rng(3)
    A = rng.standard_normal((40, 12))
    F, w = A.T @ A, rng.standard_normal(12)
    c, st = orc.codebook_row(F, w, np.zeros(12, np.uint8), np.zeros(1))
    one = np.ones(12)
    np.testing.assert_allclose(c[0], (one @ F @ w) / (one @ F @ one), rtol=1e-13)


def test_codebook_empty_codeword_kept_and_singular_row(orc):
    rng = np.random.default_rng(4)
    A = rng.standard_normal((40, 10))
    F, w = A.T @ A, rng.standard_normal(10)
    q = np.array([0, 0, 2, 2, 0, 2, 0, 0, 2, 2], np.uint8)     # codewords 1 and 3 empty
    c0 = np.array([0.1, 7.0, 0.3, -5.0])
    c, st = orc.codebook_row(F, w, q, c0)
    assert st == 0 and c[1] == 7.0 and c[3] == -5.0
    # coordinates of codeword 2 see a zero block of F -> pivot 0 -> singular, codebook kept
    Fz = F.copy()
    z = q == 2
    Fz[z, :] = 0.0
    Fz[:, z] = 0.0
    c2, st2 = orc.codebook_row(Fz, w, q, c0)
    assert st2 == 1
    np.testing.assert_array_equal(c2, c0)


# ----------------------------------------------------------------------------------- sweep

def _sweep_by_enumeration(F, w, c, q):
    """Reference sweep: each coordinate takes the candidate with the smallest objective, found
    by recomputing (Pc - w)^T F (Pc - w) for every candidate (staying unless strictly lower,
    lowest index among equal minima)."""
    q = q.copy()
    gaps = []
    for i in range(len(w)):
        Js = []
        for a in range(len(c)):
            qq = q.copy()
            qq[i] = a
            Js.append(_J(F, w, c, qq))
        Js = np.array(Js)
        stay = Js[q[i]]
        best = int(np.argmin(Js))
        srt = np.sort(Js)
        gaps.append((srt[1] - srt[0]) / max(abs(stay), 1e-300))
        if Js[best] < stay:
            q[i] = best
    return q, np.array(gaps)


def test_sweep_matches_enumeration(orc):
    F, W = _tiny_row_problem(orc)
    for j in range(3):
        w = W[j]
        c0, q0 = orc.init_row(w, 8)
        c, _ = orc.codebook_row(F, w, q0, c0)
        q_or, J_or, st, _ = orc.sweep_row(F, w, c, q0)
        q_en, gaps = _sweep_by_enumeration(F, w, c, q0)
        diff = np.nonzero(q_or != q_en)[0]
        assert all(gaps[i] < 1e-9 for i in diff), (j, diff)
        assert st["moves"] > 0
        assert abs(J_or - _J(F, w, c, q_or)) <= 1e-10 * abs(J_or)


def test_sweep_identity_F_is_nearest_codeword(orc):
    rng = np.random.default_rng(9)
    d, m = 200, 8
    w = rng.standard_normal(d)
    c = np.sort(rng.standard_normal(m))
    q0 = rng.integers(0, m, d).astype(np.uint8)
    for F in (np.eye(d), np.diag(rng.uniform(0.1, 5.0, d))):
        q, J, st, _ = orc.sweep_row(F, w, c, q0)
        np.testing.assert_array_equal(q, np.argmin(np.abs(w[:, None] - c[None, :]), axis=1))


def test_descent_every_step(orc):
    """The objective never increases: codebook steps and every single coordinate step."""
    F, W = _tiny_row_problem(orc, g=2)
    for j in range(4):
        w = W[j]
        c, q = orc.init_row(w, 8)
        J_prev = _J(F, w, c, q)
        for it in range(4):
            c, st = orc.codebook_row(F, w, q, c)
            Jc = _J(F, w, c, q)
            assert Jc <= J_prev * (1 + 1e-12)
            q, Js, stt, trace = orc.sweep_row(F, w, c, q, trace=True)
            assert np.all(np.diff(trace) <= 1e-12 * abs(trace[0]))
            assert abs(trace[0] - Jc) <= 1e-10 * Jc
            J_prev = _J(F, w, c, q)
            assert J_prev <= Jc * (1 + 1e-12)
    C, Q, Jh, status = orc.lnq_rows(F, W, 8, iters=3)
    assert np.all(np.diff(Jh, axis=1) <= 1e-12 * Jh[:, :1])
    assert np.all(status == 0)


def test_follow_mode_near_ties_and_mismatches(orc):
    # F = I, current codeword far away; w exactly between c0 and c1 up to 1e-9.
    d = 4
    F = np.eye(d)
    c = np.array([0.0, 1.0, 10.0])
    w = np.array([0.5 + 1e-9, 0.1, 9.0, 0.9])
    q0 = np.array([2, 2, 2, 2], np.uint8)
    q_own, _, st0, _ = orc.sweep_row(F, w, c, q0)
    np.testing.assert_array_equal(q_own, [1, 0, 2, 1])
    hint = q_own.copy()
    hint[0] = 0                       # near-tie: gap 2e-9 against J ~ 250
    q_f, _, st, _ = orc.sweep_row(F, w, c, q0, hint=hint, tie_rel=1e-6)
    assert st["follows"] == 1 and st["mismatches"] == 0 and q_f[0] == 0
    hint[1] = 1                       # far from the best: a mismatch, not followed
    q_m, _, st2, _ = orc.sweep_row(F, w, c, q0, hint=hint, tie_rel=1e-6)
    assert st2["mismatches"] == 1 and q_m[1] == 0


def test_follow_iteration_reproduces_own_run(orc):
    F, W = _tiny_row_problem(orc, g=3)
    rows = W[:6]
    C0 = np.zeros((6, 8))
    Q0 = np.zeros((6, 128), np.uint8)
    for j in range(6):
        C0[j], Q0[j] = orc.init_row(rows[j], 8)
    C1, Q1, Jh, _ = orc.lnq_rows(F, rows, 8, iters=1, init=False, C=C0, Q=Q0)
    Cf, Qf, Jf, stats, status = orc.follow_iteration(F, rows, 8, C0, Q0, Q1, 1e-6)
    np.testing.assert_array_equal(Qf, Q1)
    np.testing.assert_allclose(Cf, C1, rtol=1e-15)
    np.testing.assert_allclose(Jf, Jh[:, -1], rtol=1e-13)
    assert np.all(stats[:, 1] == 0) and np.all(stats[:, 2] == 0)


# ----------------------------------------------------------------------------------- optimum

def _brute_force(F, w, m):
    """min over all assignments (up to relabelling) of the objective with the optimal codebook."""
    d = len(w)
    best = np.inf
    wFw = w @ F @ w
    for q in itertools.product(range(m), repeat=d):
        q = np.array(q)
        if q[0] != 0:
            continue
        P = _onehot(q, m)[:, np.bincount(q, minlength=m) > 0]
        M, b = P.T @ F @ P, P.T @ F @ w
        c = np.linalg.solve(M, b)
        best = min(best, wFw - b @ c)
    return best


@pytest.mark.parametrize("seed", range(6))
def test_never_below_brute_force_optimum(orc, seed):
    rng = np.random.default_rng(100 + seed)
    d = 6 + seed % 3
    m = 2 + seed % 2
    A = rng.standard_normal((3 * d, d))
    F, w = A.T @ A, rng.standard_normal(d)
    Jstar = _brute_force(F, w, m)
    C, Q, Jh, _ = orc.lnq_rows(F, w[None], m, iters=6)
    assert Jh[0, -1] >= Jstar * (1 - 1e-12)


@pytest.mark.parametrize("m", [2, 3])
def test_reaches_optimum_on_separated_clusters(orc, m):
    rng = np.random.default_rng(40 + m)
    d = 8
    centres = np.array([-1.0, 0.2, 1.5])[:m]
    w = centres[np.arange(d) % m] + 0.01 * rng.standard_normal(d)
    A = np.eye(d) + 0.05 * rng.standard_normal((d, d))
    F = A.T @ A
    Jstar = _brute_force(F, w, m)
    C, Q, Jh, _ = orc.lnq_rows(F, w[None], m, iters=6)
    assert abs(Jh[0, -1] - Jstar) <= 1e-9 * Jstar


# ----------------------------------------------------------------------------------- mutations

MUTATIONS = [
    # (anchor in lnq_oracle.c, planted mistake, pin that must fail)
    ("(2.0 * u[i] + (c[a] - cur) * Fii)", "(u[i] + (c[a] - cur) * Fii)", "sweep"),
    ("u[k] += dlt * F[k * d + i];", "u[k] -= dlt * F[k * d + i];", "sweep"),
    ("fw += F[i * d + k] * w[k];", "fw += F[i * d + k] * w[i];", "codebook"),
    ("M[q[i] * m + q[k]] += F[i * d + k];", "M[q[i] * m + q[i]] += F[i * d + k];", "codebook"),
    ("sum -= L[k * nn + a] * y[k];", "sum -= L[a * nn + k] * y[k];", "codebook"),
    ("const double xa = st * XA[t * na + a];", "const double xa = XA[t * na + a];", "fisher"),
    ("acc /= (double)R;", "acc /= (double)(R + 1);", "fisher"),
    ("c[j] = sorted[((int64_t)(2 * j + 1) * d) / (2 * (int64_t)m)];",
     "c[j] = sorted[((int64_t)(2 * j) * d) / (2 * (int64_t)m)];", "init"),
    ("acc += F[i * d + k] * (c[q[k]] - w[k]);\n        J += ri * acc;",
     "acc += F[i * d + i] * (c[q[k]] - w[k]);\n        J += ri * acc;", "objective"),
]


def _pins_pass(orc, which):
    try:
        if which == "sweep":
            test_sweep_matches_enumeration(orc)
        elif which == "codebook":
            test_codebook_satisfies_normal_equations(orc)
            test_hand_worked_lnq_golden(orc)
        elif which == "fisher":
            test_hand_worked_fisher_golden_local(orc)
        elif which == "init":
            test_init_is_sorted_quantiles_and_nearest(orc)
        elif which == "objective":
            test_hand_worked_lnq_golden(orc)
        return True
    except AssertionError:
        return False


def test_hand_worked_fisher_golden_local(orc):
    g = golden("fisher_hand_n3_d2.json")
    X, G = np.array(g["X"], float), np.array(g["G"], float)
    for key, groups in (("groups_1", 1), ("groups_2", 2)):
        np.testing.assert_array_equal(orc.fisher_full(X, G, groups), np.array(g[key]["F"]))


@pytest.mark.parametrize("anchor,mistake,pin", MUTATIONS)
def test_pins_catch_planted_mistakes(orc, tmp_path, anchor, mistake, pin):
    assert _pins_pass(orc, pin)
    with orc.mutated(anchor, mistake, str(tmp_path)):
        assert not _pins_pass(orc, pin), f"pin '{pin}' missed: {mistake}"
    assert _pins_pass(orc, pin)


def test_follow_mode_absolute_floor_for_exactly_representable_rows(orc):
    """A row the codebook represents exactly reaches J ~ 0; candidates among equal codewords then
    differ only by rounding noise. Without a floor every such difference is a 'mismatch'; with a
    floor tied to the row's scale w^T F w they are followed, and nothing else changes."""
    rng = np.random.default_rng(12)
    A = rng.standard_normal((20, 5))
    F = A.T @ A
    w = np.array([0.1, 0.1, 0.2, 0.2, 0.3])
    c0, q0 = orc.init_row(w, 8)
    c, _ = orc.codebook_row(F, w, q0, c0)
    assert orc.objective_row(F, w, c, q0) < 1e-28
    hint = q0.copy()
    q_strict, _, st, _ = orc.sweep_row(F, w, c, q0, hint=hint, tie_rel=1e-6, tie_abs=0.0)
    Jw = w @ F @ w
    q_floor, _, st2, _ = orc.sweep_row(F, w, c, q0, hint=hint, tie_rel=1e-6, tie_abs=1e-12 * Jw)
    assert st2["mismatches"] == 0
    np.testing.assert_array_equal(q_floor, hint)
    # a genuinely worse hint is still a mismatch with the floor
    bad = q0.copy()
    bad[4] = 0
    _, _, st3, _ = orc.sweep_row(F, w, c, q0, hint=bad, tie_rel=1e-6, tie_abs=1e-12 * Jw)
    assert st3["mismatches"] == 1


def _weighted_lloyd(f, w, c, q, iters):
    """Textbook weighted 1-D k-means (Lloyd): each non-empty cluster's centre becomes the f-weighted
    mean of its points, then every point takes its nearest centre (a point moves only to a
    strictly nearer centre; the lowest index wins among equally near ones)."""
    c, q = c.copy(), q.copy()
    for _ in range(iters):
        for a in range(len(c)):
            sel = q == a
            if sel.any():
                c[a] = np.sum(f[sel] * w[sel]) / np.sum(f[sel])
        dist = (w[:, None] - c[None, :]) ** 2
        best = np.argmin(dist, axis=1)
        stay = dist[np.arange(len(w)), q] <= dist[np.arange(len(w)), best]
        q = np.where(stay, q, best).astype(np.uint8)
    return c, q


def test_lnq_with_diagonal_F_is_weighted_lloyd(orc):
    """With F = diag(f) the LNQ iteration (codebook step, then the in-order sweep) is weighted
    1-D k-means: the normal equations are diagonal and moves do not interact. The diagonal-Fisher
    objective of the GuidedQuant post's opening list (SqueezeLLM's sensitivity-weighted
    clustering, aitopics tag page) is exactly this case."""
    rng = np.random.default_rng(21)
    for d, m in ((64, 4), (300, 8), (1000, 16)):
        W = rng.standard_t(5, (3, d)) * 0.02
        f = np.exp(rng.standard_normal(d))
        C, Q, _, st = orc.lnq_rows(np.diag(f), W, m, 4)
        for j in range(3):
            c0, q0 = orc.init_row(W[j], m)
            c, q = _weighted_lloyd(f, W[j], c0, q0, 4)
            np.testing.assert_array_equal(Q[j], q)
            np.testing.assert_allclose(C[j], c, rtol=1e-12, atol=1e-15)
        assert np.all(st == 0)
