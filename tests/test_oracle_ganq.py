"""Pins for the oracle's GANQ-style comparison solver, each against something other than the
oracle itself.

Passage: scime.ai summary of GANQ (GPU-adaptive non-uniform quantization), Approach paragraph:
the same per-row problem solved by alternating a Cholesky / back-substitution assignment of the
codebook indices with the closed-form least-squares codebook update. The reading (lower factor
F = L L^T, coordinates visited from the last to the first, each taking the codeword nearest to its
back-substituted target, ties to the lower index, no damping) is reading R7 of the oracle header.
"""
import itertools

import numpy as np
import pytest


def _pd(rng, d, n=None):
    X = rng.standard_normal((n or 3 * d, d))
    return X.T @ X


def test_cholesky_reconstructs_and_matches_numpy(orc):
    rng = np.random.default_rng(1)
    F = _pd(rng, 37)
    L, ok = orc.cholesky(F)
    assert ok
    assert np.all(np.triu(L, 1) == 0.0)
    np.testing.assert_allclose(L @ L.T, F, rtol=0, atol=1e-10 * np.abs(F).max())
    np.testing.assert_allclose(L, np.linalg.cholesky(F), rtol=0, atol=1e-10 * np.abs(L).max())


def test_cholesky_rejects_indefinite_and_singular(orc):
    rng = np.random.default_rng(2)
    F = _pd(rng, 12)
    F[5, 5] = -1.0
    assert not orc.cholesky(F)[1]
    F = _pd(rng, 12)
    F[:, 3] = 0.0
    F[3, :] = 0.0
    assert not orc.cholesky(F)[1]


def test_identity_fisher_gives_nearest_codewords(orc):
    """With F = I the back-substituted target is w_i itself: the nearest codeword."""
    rng = np.random.default_rng(3)
    d, m = 50, 8
    w = rng.standard_normal(d)
    c = np.sort(rng.standard_normal(m))
    q, _ = orc.ganq_assign_row(np.eye(d), w, c, np.zeros(d, np.uint8))
    np.testing.assert_array_equal(q, np.argmin(np.abs(c[None, :] - w[:, None]), axis=1))


@pytest.mark.parametrize("d,m,seed", [(4, 4, 0), (5, 3, 1), (6, 2, 2), (3, 8, 3)])
def test_brute_force_lexicographic_characterisation(orc, d, m, seed):
    """z = L^T r has z_i depending only on r_i..r_{d-1}, so visiting i = d-1 down to 0 and
    minimising |z_i| each time yields the assignment that minimises (|z_{d-1}|, ..., |z_0|)
    lexicographically. Enumerating all m^d assignments and taking that minimum (matrix products,
    no back-substitution) must give the oracle's codes."""
    rng = np.random.default_rng(seed)
    F = _pd(rng, d)
    w = rng.standard_normal(d)
    c = rng.standard_normal(m)
    L, ok = orc.cholesky(F)
    assert ok
    best, best_key = None, None
    for qs in itertools.product(range(m), repeat=d):
        q = np.array(qs)
        z = L.T @ (c[q] - w)
        key = tuple(np.round(np.abs(z[::-1]), 12))
        if best_key is None or key < best_key:
            best, best_key = q, key
    q, _ = orc.ganq_assign_row(L, w, c, np.zeros(d, np.uint8))
    np.testing.assert_array_equal(q, best)


def test_objective_is_sum_of_squared_plane_residuals(orc):
    """r^T F r = ||L^T r||^2 for any assignment, and the chosen codes make every |z_i| no larger
    than with any other codeword at i (given the later coordinates)."""
    rng = np.random.default_rng(4)
    d, m = 60, 8
    F = _pd(rng, d)
    w = rng.standard_normal(d) * 0.1
    c = np.sort(rng.standard_normal(m) * 0.1)
    L, _ = orc.cholesky(F)
    q, _ = orc.ganq_assign_row(L, w, c, np.zeros(d, np.uint8))
    r = c[q] - w
    z = L.T @ r
    np.testing.assert_allclose(r @ F @ r, z @ z, rtol=1e-10)
    for i in range(d):
        for a in range(m):
            r2 = r.copy()
            r2[i] = c[a] - w[i]
            assert abs(z[i]) <= abs((L.T @ r2)[i]) + 1e-12


def test_iteration_runs_the_codebook_step_then_the_assignment(orc):
    rng = np.random.default_rng(5)
    d, m, rows = 48, 4, 3
    F = _pd(rng, d)
    W = rng.standard_normal((rows, d))
    L, _ = orc.cholesky(F)
    C0 = np.stack([orc.init_row(W[j], m)[0] for j in range(rows)])
    Q0 = np.stack([orc.init_row(W[j], m)[1] for j in range(rows)])
    C, Q, J, stats, status = orc.ganq_iteration(F, L, W, m, C0, Q0)
    for j in range(rows):
        c, st = orc.codebook_row(F, W[j], Q0[j], C0[j])
        np.testing.assert_array_equal(C[j], c)
        q, _ = orc.ganq_assign_row(L, W[j], c, Q0[j])
        np.testing.assert_array_equal(Q[j], q)
        assert J[j] == pytest.approx(orc.objective_row(F, W[j], C[j], Q[j]), rel=1e-14)
        assert status[j] == st
    assert np.all(stats[:, 1:] == 0)


def test_follow_mode_takes_near_ties_only(orc):
    rng = np.random.default_rng(6)
    d, m = 30, 4
    F = _pd(rng, d)
    w = rng.standard_normal(d)
    c = np.sort(rng.standard_normal(m))
    L, _ = orc.cholesky(F)
    q, _ = orc.ganq_assign_row(L, w, c, np.zeros(d, np.uint8))
    q2, st = orc.ganq_assign_row(L, w, c, np.zeros(d, np.uint8), hint=q)
    np.testing.assert_array_equal(q, q2)
    assert st[1] == 0 and st[2] == 0
    # a hint that differs everywhere: with no band every difference is a mismatch, with an
    # unbounded band every hinted code is taken
    hint = (q + 1) % m
    _, st = orc.ganq_assign_row(L, w, c, np.zeros(d, np.uint8), hint=hint)
    assert st[2] > 0 and st[1] == 0
    q3, st = orc.ganq_assign_row(L, w, c, np.zeros(d, np.uint8), hint=hint, band=np.inf)
    np.testing.assert_array_equal(q3, hint)


MUTATIONS = [
    ("for (int64_t i = d - 1; i >= 0; --i) {\n        double s = 0.0;\n        for (int64_t k = i + 1; k < d; ++k)\n            s += L[k * d + i] * r[k];",
     "for (int64_t i = d - 1; i >= 0; --i) {\n        double s = 0.0;\n        for (int64_t k = i + 1; k < d; ++k)\n            s += L[i * d + k] * r[k];"),
    ("        const double t = w[i] - s / lii;", "        const double t = w[i] + s / lii;"),
    ("                L[i * d + j] = sum / L[j * d + j];", "                L[i * d + j] = sum / L[i * d + i];"),
]


@pytest.mark.parametrize("anchor,mistake", MUTATIONS)
def test_pins_catch_planted_mistakes(orc, tmp_path, anchor, mistake):
    def pins_pass():
        try:
            test_cholesky_reconstructs_and_matches_numpy(orc)
            test_brute_force_lexicographic_characterisation(orc, 4, 4, 0)
            test_objective_is_sum_of_squared_plane_residuals(orc)
        except AssertionError:
            return False
        return True
    assert pins_pass()
    with orc.mutated(anchor, mistake, str(tmp_path)):
        assert not pins_pass(), f"pins missed: {mistake}"
