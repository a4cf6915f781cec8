"""Python view of the FP64 CPU oracle in ``lnq_oracle.c``.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` are the only importers. The CUDA product path never imports this module.

This module only marshals numpy arrays into the C routines; all arithmetic is in the C file, whose
header lists the passages of the GuidedQuant / LNQ pages each routine transcribes and the readings
taken where the pages are silent.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lnq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblnq_oracle.so")
_lib = None

_DP = ctypes.POINTER(ctypes.c_double)
_U8P = ctypes.POINTER(ctypes.c_uint8)
_I64P = ctypes.POINTER(ctypes.c_int64)
_I32P = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (FP64, OpenMP) if the shared object is missing or stale."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.orc_group_scales.argtypes = [_DP, _I64, _I64, _I64, _DP]
    lib.orc_fisher_block.argtypes = [_DP, _I64, _DP, _I64, _DP, _I64, ctypes.c_double, _DP]
    lib.orc_fisher_diag.argtypes = [_DP, _I64, _I64, _DP, ctypes.c_double, _DP]
    lib.orc_objective_row.argtypes = [_DP, _I64, _DP, _DP, _U8P]
    lib.orc_objective_row.restype = ctypes.c_double
    lib.orc_init_row.argtypes = [_DP, _I64, ctypes.c_int, _DP, _U8P]
    lib.orc_codebook_row.argtypes = [_DP, _I64, _DP, ctypes.c_int, _U8P, _DP]
    lib.orc_codebook_row.restype = ctypes.c_int
    lib.orc_sweep_row.argtypes = [_DP, _I64, _DP, ctypes.c_int, _DP, _U8P, _U8P,
                                  ctypes.c_double, ctypes.c_double, _I64P, _DP]
    lib.orc_sweep_row.restype = ctypes.c_double
    lib.orc_lnq_rows.argtypes = [_DP, _I64, _DP, _I64, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, _DP, _U8P, _DP, _I32P, ctypes.c_int]
    lib.orc_cholesky.argtypes = [_DP, _I64, _DP]
    lib.orc_cholesky.restype = ctypes.c_int
    lib.orc_ganq_assign_row.argtypes = [_DP, _I64, _DP, ctypes.c_int, _DP, _U8P, _U8P,
                                        ctypes.c_double, _I64P]
    lib.orc_ganq_iteration.argtypes = [_DP, _DP, _I64, _DP, _I64, ctypes.c_int, _DP, _U8P, _U8P,
                                       _DP, _DP, _U8P, _DP, _I64P, _I32P, ctypes.c_int]
    lib.orc_follow_iteration.argtypes = [_DP, _I64, _DP, _I64, ctypes.c_int, _DP, _U8P,
                                         _U8P, ctypes.c_double, _DP, _DP, _U8P, _DP, _I64P,
                                         _I32P, ctypes.c_int]
    u32p = ctypes.POINTER(ctypes.c_uint32)
    lib.orc_pack_codes.argtypes = [_U8P, _I64, _I64, ctypes.c_int, u32p]
    lib.orc_unpack_codes.argtypes = [u32p, _I64, _I64, ctypes.c_int, _U8P]
    lib.orc_lut_gemv.argtypes = [_DP, _I64, _DP, ctypes.c_int, _U8P, _I64, _I64, _DP]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(_LIB_PATH)
    return _lib


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


@contextlib.contextmanager
def mutated(old: str, new: str, workdir: str):
    """Test helper: compile a copy of the oracle with one planted mistake (`old` replaced by
    `new`, which must occur exactly once) and route every call in this module to it."""
    global _lib
    text = source_text()
    assert text.count(old) == 1, f"mutation anchor not unique: {old!r}"
    src = os.path.join(workdir, "mutant.c")
    so = os.path.join(workdir, "libmutant.so")
    with open(src, "w") as f:
        f.write(text.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                           "-ffp-contract=off", src, "-o", so, "-lm"])
    saved = _load()
    _lib = _bind(so)
    try:
        yield
    finally:
        _lib = saved


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _u8(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint8)


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


# ---------------------------------------------------------------------------------------------
# Fisher blocks
# ---------------------------------------------------------------------------------------------

def group_scales(G, n: int, d_out: int, groups: int) -> np.ndarray:
    """S[g, t] = mean over rows j of group g of G[t, j]^2; G None means all ones."""
    S = np.empty((groups, n), dtype=np.float64)
    if G is None:
        _load().orc_group_scales(None, n, d_out, groups, _p(S, _DP))
    else:
        Gd = _f64(G)
        assert Gd.shape == (n, d_out)
        _load().orc_group_scales(_p(Gd, _DP), n, d_out, groups, _p(S, _DP))
    return S


def fisher_block(XA, XB, s, alpha: float = 1.0) -> np.ndarray:
    """alpha * XA^T diag(s) XB for column subsets XA (n x na), XB (n x nb) of X."""
    XA, XB, s = _f64(XA), _f64(XB), _f64(s)
    n, na = XA.shape
    nb = XB.shape[1]
    assert XB.shape[0] == n and s.shape == (n,)
    out = np.empty((na, nb), dtype=np.float64)
    _load().orc_fisher_block(_p(XA, _DP), na, _p(XB, _DP), nb, _p(s, _DP), n, alpha,
                             _p(out, _DP))
    return out


def fisher_full(X, G, groups: int, alpha: float = 1.0) -> np.ndarray:
    """All grouped Fisher blocks F[g] = alpha X^T diag(s_g) X (small problems only)."""
    X = _f64(X)
    n, d = X.shape
    d_out = G.shape[1] if G is not None else groups
    S = group_scales(G, n, d_out, groups)
    return np.stack([fisher_block(X, X, S[g], alpha) for g in range(groups)])


def fisher_diag(X, s, alpha: float = 1.0) -> np.ndarray:
    X, s = _f64(X), _f64(s)
    n, d = X.shape
    out = np.empty(d, dtype=np.float64)
    _load().orc_fisher_diag(_p(X, _DP), n, d, _p(s, _DP), alpha, _p(out, _DP))
    return out


# ---------------------------------------------------------------------------------------------
# LNQ per row
# ---------------------------------------------------------------------------------------------

def objective_row(F, w, c, q) -> float:
    F, w, c, q = _f64(F), _f64(w), _f64(c), _u8(q)
    d = w.shape[0]
    return _load().orc_objective_row(_p(F, _DP), d, _p(w, _DP), _p(c, _DP), _p(q, _U8P))


def init_row(w, m: int):
    w = _f64(w)
    d = w.shape[0]
    c = np.empty(m, dtype=np.float64)
    q = np.empty(d, dtype=np.uint8)
    _load().orc_init_row(_p(w, _DP), d, m, _p(c, _DP), _p(q, _U8P))
    return c, q


def codebook_row(F, w, q, c):
    """Returns (new codebook, status) with status 0 = ok, 1 = singular (codebook unchanged)."""
    F, w, q = _f64(F), _f64(w), _u8(q)
    c = _f64(c).copy()
    d = w.shape[0]
    st = _load().orc_codebook_row(_p(F, _DP), d, _p(w, _DP), c.shape[0], _p(q, _U8P),
                                  _p(c, _DP))
    return c, st


def sweep_row(F, w, c, q, hint=None, tie_rel: float = 0.0, trace: bool = False,
              tie_abs: float = 0.0):
    """Returns (q after the sweep, J after, stats dict, J trace or None)."""
    F, w, c = _f64(F), _f64(w), _f64(c)
    q = _u8(q).copy()
    d = w.shape[0]
    stats = np.zeros(4, dtype=np.int64)
    jt = np.empty(d + 1, dtype=np.float64) if trace else None
    hp = _p(_u8(hint), _U8P) if hint is not None else None
    J = _load().orc_sweep_row(_p(F, _DP), d, _p(w, _DP), c.shape[0], _p(c, _DP), _p(q, _U8P),
                              hp, tie_rel, tie_abs, _p(stats, _I64P),
                              _p(jt, _DP) if trace else None)
    st = {"moves": int(stats[0]), "follows": int(stats[1]), "mismatches": int(stats[2]),
          "min_gap": float(stats[3:4].view(np.float64)[0])}
    return q, J, st, jt


def lnq_rows(F, W, m: int, iters: int, init: bool = True, C=None, Q=None,
             nthreads: int = 0):
    """Full LNQ for rows sharing F. Returns (C, Q, J_hist [rows, 2*iters], status)."""
    F, W = _f64(F), _f64(W)
    nrows, d = W.shape
    C = np.zeros((nrows, m), dtype=np.float64) if C is None else _f64(C).copy()
    Q = np.zeros((nrows, d), dtype=np.uint8) if Q is None else _u8(Q).copy()
    J = np.zeros((nrows, max(2 * iters, 1)), dtype=np.float64)
    status = np.zeros(nrows, dtype=np.int32)
    _load().orc_lnq_rows(_p(F, _DP), d, _p(W, _DP), nrows, m, iters, int(init), _p(C, _DP),
                         _p(Q, _U8P), _p(J, _DP), _p(status, _I32P), nthreads)
    return C, Q, J[:, :2 * iters], status


def follow_iteration(F, W, m: int, C_start, Q_start, Q_hint, tie_rel: float,
                     nthreads: int = 0, tie_abs=None):
    """One oracle iteration from another solver's state, following its choices at near-ties.
    tie_abs: optional per-row absolute floor of the tie band.

    Returns (C_out, Q_out, J_out, stats [rows, 4] with the gap column as float64, status)."""
    F, W = _f64(F), _f64(W)
    nrows, d = W.shape
    C_start, Q_start, Q_hint = _f64(C_start), _u8(Q_start), _u8(Q_hint)
    C_out = np.empty((nrows, m), dtype=np.float64)
    Q_out = np.empty((nrows, d), dtype=np.uint8)
    J_out = np.empty(nrows, dtype=np.float64)
    stats = np.zeros((nrows, 4), dtype=np.int64)
    status = np.zeros(nrows, dtype=np.int32)
    ta = None if tie_abs is None else _f64(tie_abs)
    _load().orc_follow_iteration(_p(F, _DP), d, _p(W, _DP), nrows, m, _p(C_start, _DP),
                                 _p(Q_start, _U8P), _p(Q_hint, _U8P), tie_rel,
                                 None if ta is None else _p(ta, _DP), _p(C_out, _DP),
                                 _p(Q_out, _U8P), _p(J_out, _DP), _p(stats, _I64P),
                                 _p(status, _I32P), nthreads)
    return C_out, Q_out, J_out, stats, status


_U32P = ctypes.POINTER(ctypes.c_uint32)


def cholesky(F):
    """(L, ok): the lower Cholesky factor F = L L^T in FP64; ok is False at a non-positive
    pivot (reading R7)."""
    F = _f64(F)
    d = F.shape[0]
    L = np.zeros((d, d), dtype=np.float64)
    bad = _load().orc_cholesky(_p(F, _DP), d, _p(L, _DP))
    return L, bad == 0


def ganq_assign_row(L, w, c, q, hint=None, band: float = 0.0):
    """The back-substitution assignment of one row (reading R7); returns (q, stats) with stats
    [changed, tie-follows, mismatches]."""
    L, w, c = _f64(L), _f64(w), _f64(c)
    q = _u8(q).copy()
    stats = np.zeros(3, dtype=np.int64)
    hp = None if hint is None else _p(_u8(hint), _U8P)
    _load().orc_ganq_assign_row(_p(L, _DP), L.shape[0], _p(w, _DP), c.shape[0], _p(c, _DP),
                                _p(q, _U8P), hp, float(band), _p(stats, _I64P))
    return q, stats


def ganq_iteration(F, L, W, m: int, C_start, Q_start, Q_hint=None, band=None, nthreads: int = 0):
    """One GANQ-style iteration (codebook step, then back-substitution assignment) for rows
    sharing F; returns (C, Q, J, stats [rows x 3], status)."""
    F, L, W = _f64(F), _f64(L), _f64(W)
    nrows, d = W.shape
    C = np.empty((nrows, m), dtype=np.float64)
    Q = np.empty((nrows, d), dtype=np.uint8)
    J = np.empty(nrows, dtype=np.float64)
    stats = np.zeros((nrows, 3), dtype=np.int64)
    status = np.zeros(nrows, dtype=np.int32)
    hp = None if Q_hint is None else _p(_u8(Q_hint), _U8P)
    bp = None if band is None else _p(_f64(band), _DP)
    _load().orc_ganq_iteration(_p(F, _DP), _p(L, _DP), d, _p(W, _DP), nrows, m,
                               _p(_f64(C_start), _DP), _p(_u8(Q_start), _U8P), hp, bp,
                               _p(C, _DP), _p(Q, _U8P), _p(J, _DP), _p(stats, _I64P),
                               _p(status, _I32P), nthreads)
    return C, Q, J, stats, status


def packed_words(d_in: int, bits: int) -> int:
    """32-bit words per row of packed codes (reading R6 in lnq_oracle.c)."""
    per = 32 // bits
    return (d_in + per - 1) // per


def pack_codes(Q, bits: int):
    """Q [d_out][d_in] uint8 -> packed uint32 [d_out][packed_words(d_in, bits)]."""
    Q = _u8(Q)
    d_out, d_in = Q.shape
    P = np.empty((d_out, packed_words(d_in, bits)), dtype=np.uint32)
    _load().orc_pack_codes(_p(Q, _U8P), d_out, d_in, bits, _p(P, _U32P))
    return P


def unpack_codes(P, d_in: int, bits: int):
    P = np.ascontiguousarray(P, dtype=np.uint32)
    d_out = P.shape[0]
    Q = np.empty((d_out, d_in), dtype=np.uint8)
    _load().orc_unpack_codes(_p(P, _U32P), d_out, d_in, bits, _p(Q, _U8P))
    return Q


def lut_gemv(x, C, Q):
    """y [nb][d_out] = x [nb][d_in] times W^ = C[Q] (rows of W^ are the output channels)."""
    x, C, Q = _f64(x), _f64(C), _u8(Q)
    if x.ndim == 1:
        x = x[None, :]
    nb, d_in = x.shape
    d_out, m = C.shape
    y = np.empty((nb, d_out), dtype=np.float64)
    _load().orc_lut_gemv(_p(x, _DP), nb, _p(C, _DP), m, _p(Q, _U8P), d_out, d_in, _p(y, _DP))
    return y
