"""Thin ctypes binding of liblnq.so with the same entry-point names as include/lnq.h.

Argument marshalling only: every step of the path runs in the CUDA library. PyTorch supplies
device memory and the current stream. If the library is missing, the functions raise; there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblnq.so")

# Status codes and selectors (include/lnq.h).
LNQ_OK, LNQ_ERR_INVALID_ARG, LNQ_ERR_CUDA, LNQ_ERR_WORKSPACE, LNQ_ERR_UNSUPPORTED, \
    LNQ_ERR_TIMEOUT = range(6)
LNQ_ROW_OK, LNQ_ROW_SINGULAR, LNQ_ROW_NOT_PD = 0, 1, 2
(LNQ_OP_BUILD_FISHER, LNQ_OP_INIT_CODEBOOK, LNQ_OP_QUANTIZE_ROWS, LNQ_OP_OBJECTIVE,
 LNQ_OP_GANQ_ROWS) = range(5)

EXPORTED = ("lnq_workspace_size", "lnq_build_fisher", "lnq_init_codebook", "lnq_quantize_rows",
            "lnq_objective", "lnq_workspace_check", "lnq_set_wait_limit", "lnq_status_string",
            "lnq_profile_enable", "lnq_profile_read", "lnq_build_fisher_noalloc",
            "lnq_packed_words", "lnq_pack_codes", "lnq_lut_gemv", "lnq_quantize_rows_diag",
            "lnq_sweep_counters", "lnq_fp32_probe", "lnq_ganq_rows")

_lib = None
_VP, _I64, _INT, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t


class LnqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lnq_status_string(status)} (status {status})")


def lib():
    """The loaded library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        L.lnq_workspace_size.argtypes = [_INT, _I64, _I64, _I64, _INT, _INT]
        L.lnq_workspace_size.restype = _SZ
        L.lnq_build_fisher.argtypes = [_VP, _VP, _I64, _I64, _I64, _INT, ctypes.c_float, _VP,
                                       _VP, _SZ, _VP]
        L.lnq_build_fisher_noalloc.argtypes = [_VP, _VP, _I64, _I64, _I64, _INT, ctypes.c_float,
                                               _VP, _VP]
        L.lnq_init_codebook.argtypes = [_VP, _I64, _I64, _INT, _VP, _VP, _VP, _SZ, _VP]
        L.lnq_quantize_rows.argtypes = [_VP, _INT, _VP, _I64, _I64, _INT, _INT, _VP, _VP, _VP,
                                        _VP, _VP, _SZ, _VP]
        L.lnq_ganq_rows.argtypes = L.lnq_quantize_rows.argtypes
        L.lnq_objective.argtypes = [_VP, _INT, _VP, _VP, _VP, _I64, _I64, _INT, _VP, _VP, _SZ,
                                    _VP]
        L.lnq_workspace_check.argtypes = [_VP, _VP]
        L.lnq_set_wait_limit.argtypes = [_I64]
        L.lnq_set_wait_limit.restype = None
        L.lnq_profile_enable.argtypes = [_INT]
        L.lnq_profile_enable.restype = None
        L.lnq_profile_read.argtypes = [_INT, ctypes.POINTER(ctypes.c_char_p),
                                       ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int64)]
        L.lnq_profile_read.restype = _INT
        L.lnq_status_string.argtypes = [_INT]
        L.lnq_status_string.restype = ctypes.c_char_p
        L.lnq_packed_words.argtypes = [_I64, _INT]
        L.lnq_packed_words.restype = _I64
        L.lnq_pack_codes.argtypes = [_VP, _I64, _I64, _INT, _VP, _VP]
        L.lnq_lut_gemv.argtypes = [_VP, _I64, _VP, _VP, _I64, _I64, _INT, _VP, _VP]
        L.lnq_quantize_rows_diag.argtypes = [_VP, _INT, _VP, _I64, _I64, _INT, _INT, _VP, _VP,
                                             _VP, _VP, _VP]
        L.lnq_sweep_counters.argtypes = [_VP, _VP, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]
        L.lnq_fp32_probe.argtypes = [_I64, _VP, ctypes.POINTER(_I64), _VP]
        for name in ("lnq_build_fisher", "lnq_build_fisher_noalloc", "lnq_init_codebook",
                     "lnq_quantize_rows", "lnq_objective", "lnq_workspace_check",
                     "lnq_pack_codes", "lnq_lut_gemv", "lnq_quantize_rows_diag",
                     "lnq_sweep_counters", "lnq_fp32_probe", "lnq_ganq_rows"):
            getattr(L, name).restype = _INT
        _lib = L
    return _lib


def lnq_status_string(status: int) -> str:
    return lib().lnq_status_string(int(status)).decode()


def lnq_workspace_size(op: int, n: int = 0, d_in: int = 0, d_out: int = 0, groups: int = 1,
                       m: int = 2) -> int:
    return int(lib().lnq_workspace_size(op, n, d_in, d_out, groups, m))


def lnq_set_wait_limit(cycles: int) -> None:
    lib().lnq_set_wait_limit(int(cycles))


def lnq_profile_enable(on: bool = True) -> None:
    lib().lnq_profile_enable(1 if on else 0)


def lnq_profile_read(max_kernels: int = 64) -> dict:
    """{kernel name: (launches, total device ms)} since the last read; clears the records."""
    names = (ctypes.c_char_p * max_kernels)()
    ms = (ctypes.c_double * max_kernels)()
    cnt = (ctypes.c_int64 * max_kernels)()
    k = lib().lnq_profile_read(max_kernels, names, ms, cnt)
    return {names[i].decode(): (int(cnt[i]), float(ms[i])) for i in range(k)}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def workspace(op: int, n=0, d_in=0, d_out=0, groups=1, m=2, device="cuda") -> torch.Tensor:
    """A device workspace of the size the library asks for (torch's allocator aligns to 512 B)."""
    size = lnq_workspace_size(op, n, d_in, d_out, groups, m)
    return torch.empty(max(size, 256), dtype=torch.uint8, device=device)


def _check(status: int, where: str):
    if status != LNQ_OK:
        raise LnqError(status, where)


def lnq_build_fisher(X: torch.Tensor, G: Optional[torch.Tensor], groups: int, alpha: float = 1.0,
                     F: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    n, d_in = X.shape
    d_out = G.shape[1] if G is not None else groups
    _need(X, torch.bfloat16, (n, d_in), "X")
    if G is not None:
        _need(G, torch.bfloat16, (n, d_out), "G")
    if F is None:
        F = torch.empty((groups, d_in, d_in), dtype=torch.float32, device=X.device)
    _need(F, torch.float32, (groups, d_in, d_in), "F")
    if ws is None:
        ws = workspace(LNQ_OP_BUILD_FISHER, n, d_in, d_out, groups, device=X.device)
    _check(lib().lnq_build_fisher(_ptr(X), _ptr(G), n, d_in, d_out, groups, alpha, _ptr(F),
                                  _ptr(ws), ws.numel(), _stream(stream)), "lnq_build_fisher")
    return F


def lnq_build_fisher_noalloc(X: torch.Tensor, G: Optional[torch.Tensor], groups: int,
                             alpha: float = 1.0, F: Optional[torch.Tensor] = None,
                             stream=None) -> torch.Tensor:
    """lnq_build_fisher with the library's static scratch instead of a workspace (F is still
    caller memory; pass it in to keep the call free of any allocation)."""
    n, d_in = X.shape
    d_out = G.shape[1] if G is not None else groups
    _need(X, torch.bfloat16, (n, d_in), "X")
    if G is not None:
        _need(G, torch.bfloat16, (n, d_out), "G")
    if F is None:
        F = torch.empty((groups, d_in, d_in), dtype=torch.float32, device=X.device)
    _need(F, torch.float32, (groups, d_in, d_in), "F")
    _check(lib().lnq_build_fisher_noalloc(_ptr(X), _ptr(G), n, d_in, d_out, groups, alpha,
                                          _ptr(F), _stream(stream)), "lnq_build_fisher_noalloc")
    return F


def lnq_noalloc_check(stream=None) -> int:
    """Synchronises the stream and reports (LNQ_OK / LNQ_ERR_TIMEOUT) whether a bounded wait of the
    last lnq_build_fisher_noalloc call on the current device gave up; clears the flag."""
    return int(lib().lnq_workspace_check(None, _stream(stream)))


def lnq_init_codebook(W: torch.Tensor, m: int, C: Optional[torch.Tensor] = None,
                      Q: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      stream=None):
    d_out, d_in = W.shape
    _need(W, torch.float32, (d_out, d_in), "W")
    if C is None:
        C = torch.empty((d_out, m), dtype=torch.float32, device=W.device)
    if Q is None:
        Q = torch.empty((d_out, d_in), dtype=torch.uint8, device=W.device)
    _need(C, torch.float32, (d_out, m), "C")
    _need(Q, torch.uint8, (d_out, d_in), "Q")
    if ws is None:
        ws = workspace(LNQ_OP_INIT_CODEBOOK, 0, d_in, d_out, 1, m, device=W.device)
    _check(lib().lnq_init_codebook(_ptr(W), d_out, d_in, m, _ptr(C), _ptr(Q), _ptr(ws),
                                   ws.numel(), _stream(stream)), "lnq_init_codebook")
    return C, Q


def lnq_quantize_rows(F: torch.Tensor, W: torch.Tensor, m: int, iters: int, C: torch.Tensor,
                      Q: torch.Tensor, J_out: Optional[torch.Tensor] = None,
                      row_status: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None, stream=None):
    """Runs `iters` LNQ iterations in place on (C, Q); returns (C, Q, J_out, row_status)."""
    groups, d_in, _ = F.shape
    d_out = W.shape[0]
    _need(F, torch.float32, (groups, d_in, d_in), "F")
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(C, torch.float32, (d_out, m), "C")
    _need(Q, torch.uint8, (d_out, d_in), "Q")
    if J_out is not None:
        _need(J_out, torch.float64, (d_out,), "J_out")
    if row_status is not None:
        _need(row_status, torch.int32, (d_out,), "row_status")
    if ws is None:
        ws = workspace(LNQ_OP_QUANTIZE_ROWS, 0, d_in, d_out, groups, m, device=W.device)
    _check(lib().lnq_quantize_rows(_ptr(F), groups, _ptr(W), d_out, d_in, m, iters, _ptr(C),
                                   _ptr(Q), _ptr(J_out), _ptr(row_status), _ptr(ws), ws.numel(),
                                   _stream(stream)), "lnq_quantize_rows")
    return C, Q, J_out, row_status


def lnq_ganq_rows(F: torch.Tensor, W: torch.Tensor, m: int, iters: int, C: torch.Tensor,
                  Q: torch.Tensor, J_out: Optional[torch.Tensor] = None,
                  row_status: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None, stream=None):
    """`iters` GANQ-style iterations (codebook step, Cholesky / back-substitution assignment) in
    place on (C, Q); returns (C, Q, J_out, row_status)."""
    groups, d_in, _ = F.shape
    d_out = W.shape[0]
    _need(F, torch.float32, (groups, d_in, d_in), "F")
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(C, torch.float32, (d_out, m), "C")
    _need(Q, torch.uint8, (d_out, d_in), "Q")
    if J_out is not None:
        _need(J_out, torch.float64, (d_out,), "J_out")
    if row_status is not None:
        _need(row_status, torch.int32, (d_out,), "row_status")
    if ws is None:
        ws = workspace(LNQ_OP_GANQ_ROWS, 0, d_in, d_out, groups, m, device=W.device)
    _check(lib().lnq_ganq_rows(_ptr(F), groups, _ptr(W), d_out, d_in, m, iters, _ptr(C),
                               _ptr(Q), _ptr(J_out), _ptr(row_status), _ptr(ws), ws.numel(),
                               _stream(stream)), "lnq_ganq_rows")
    return C, Q, J_out, row_status


def lnq_quantize_rows_diag(Fd: torch.Tensor, W: torch.Tensor, m: int, iters: int,
                           C: torch.Tensor, Q: torch.Tensor, J_out: Optional[torch.Tensor] = None,
                           row_status: Optional[torch.Tensor] = None, stream=None):
    """`iters` LNQ iterations in place on (C, Q) with diagonal Fisher blocks Fd [groups][d_in];
    returns (C, Q, J_out, row_status)."""
    groups, d_in = Fd.shape
    d_out = W.shape[0]
    _need(Fd, torch.float32, (groups, d_in), "Fd")
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(C, torch.float32, (d_out, m), "C")
    _need(Q, torch.uint8, (d_out, d_in), "Q")
    if J_out is not None:
        _need(J_out, torch.float64, (d_out,), "J_out")
    if row_status is not None:
        _need(row_status, torch.int32, (d_out,), "row_status")
    _check(lib().lnq_quantize_rows_diag(_ptr(Fd), groups, _ptr(W), d_out, d_in, m, iters,
                                        _ptr(C), _ptr(Q), _ptr(J_out), _ptr(row_status),
                                        _stream(stream)), "lnq_quantize_rows_diag")
    return C, Q, J_out, row_status


def lnq_objective(F: torch.Tensor, W: torch.Tensor, C: torch.Tensor, Q: torch.Tensor,
                  J: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    groups, d_in, _ = F.shape
    d_out, m = C.shape
    _need(F, torch.float32, (groups, d_in, d_in), "F")
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(Q, torch.uint8, (d_out, d_in), "Q")
    if J is None:
        J = torch.empty(d_out, dtype=torch.float64, device=W.device)
    if ws is None:
        ws = workspace(LNQ_OP_OBJECTIVE, 0, d_in, d_out, groups, m, device=W.device)
    _check(lib().lnq_objective(_ptr(F), groups, _ptr(W), _ptr(C), _ptr(Q), d_out, d_in, m,
                               _ptr(J), _ptr(ws), ws.numel(), _stream(stream)), "lnq_objective")
    return J


def lnq_workspace_check(ws: Optional[torch.Tensor], stream=None) -> int:
    """Synchronises the stream and returns LNQ_OK or LNQ_ERR_TIMEOUT (see include/lnq.h); ws None
    checks the static scratch of lnq_build_fisher_noalloc on the current device."""
    return int(lib().lnq_workspace_check(_ptr(ws), _stream(stream)))


def lnq_sweep_counters(ws: torch.Tensor, stream=None):
    """(moves, tail) of the sweeps of the last lnq_quantize_rows call on `ws` (synchronises)."""
    mv, tl = ctypes.c_int64(0), ctypes.c_int64(0)
    _check(lib().lnq_sweep_counters(_ptr(ws), _stream(stream), ctypes.byref(mv),
                                    ctypes.byref(tl)), "lnq_sweep_counters")
    return int(mv.value), int(tl.value)


def lnq_fp32_probe(iters: int, sink: torch.Tensor, stream=None) -> int:
    """Enqueues the FP32 FFMA probe kernel; returns the number of FFMAs it performs."""
    ops = ctypes.c_int64(0)
    _check(lib().lnq_fp32_probe(int(iters), _ptr(sink), ctypes.byref(ops), _stream(stream)),
           "lnq_fp32_probe")
    return int(ops.value)


def lnq_packed_words(d_in: int, bits: int) -> int:
    """32-bit words per packed row (see include/lnq.h)."""
    return int(lib().lnq_packed_words(int(d_in), int(bits)))


def lnq_pack_codes(Q: torch.Tensor, bits: int, P: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Q [d_out][d_in] uint8 -> packed int32 words [d_out][lnq_packed_words(d_in, bits)]."""
    d_out, d_in = Q.shape
    _need(Q, torch.uint8, (d_out, d_in), "Q")
    words = lnq_packed_words(d_in, bits)
    if P is None:
        P = torch.empty((d_out, words), dtype=torch.int32, device=Q.device)
    _need(P, torch.int32, (d_out, words), "P")
    _check(lib().lnq_pack_codes(_ptr(Q), d_out, d_in, int(bits), _ptr(P), _stream(stream)),
           "lnq_pack_codes")
    return P


def lnq_lut_gemv(x: torch.Tensor, P: torch.Tensor, C: torch.Tensor, d_in: int,
                 y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y [nb][d_out] = x [nb][d_in] times W^ = C[codes] (packed codes P, codebooks C [d_out][m])."""
    d_out, m = C.shape
    bits = m.bit_length() - 1
    if x.dim() == 1:
        x = x.view(1, -1)
    nb = x.shape[0]
    _need(x, torch.float32, (nb, d_in), "x")
    _need(C, torch.float32, (d_out, m), "C")
    _need(P, torch.int32, (d_out, lnq_packed_words(d_in, bits)), "P")
    if y is None:
        y = torch.empty((nb, d_out), dtype=torch.float32, device=x.device)
    _need(y, torch.float32, (nb, d_out), "y")
    _check(lib().lnq_lut_gemv(_ptr(x), nb, _ptr(P), _ptr(C), d_out, int(d_in), bits, _ptr(y),
                              _stream(stream)), "lnq_lut_gemv")
    return y
