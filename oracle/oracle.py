"""ctypes front end of the fp64 oracle (``attention_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Inputs are numpy
arrays; bf16 tensors travel as their raw uint16 bit patterns so that the
oracle sees exactly the values the GPU sees.  Outputs are float64.
"""
import ctypes
import os

import numpy as np

from .build_oracle import build as _build

_lib = None


def library_path() -> str:
    return _build()


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIBRARY lets the mutation test point the pins at a copy of
        # the oracle with a planted mistake; normally the built library loads.
        lib = ctypes.CDLL(os.environ.get("ORACLE_LIBRARY") or _build())
        dp = ctypes.POINTER(ctypes.c_double)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.oracle_softmax_row.argtypes = [dp, i64, dp]
        lib.oracle_attend_scores.argtypes = [dp, dp, i64, i64, i64, dp, dp]
        lib.oracle_attention_f64.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64,
                                             i64, ctypes.c_int, ctypes.c_double,
                                             ctypes.c_int]
        lib.oracle_attention_rows_bf16.argtypes = [
            u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_int,
            ctypes.c_double, i64p, i64, dp, dp, ctypes.c_int]
        lib.oracle_attention_backward_f64.argtypes = [
            dp, dp, dp, dp, dp, dp, dp, i64, i64, i64, i64, ctypes.c_int,
            ctypes.c_double, ctypes.c_int]
        lib.oracle_attention_backward_f64.restype = ctypes.c_int
        lib.oracle_attention_blocked_f64.argtypes = [
            dp, dp, dp, dp, dp, i64, i64, i64, i64, ctypes.c_int,
            ctypes.c_double, i64, i64]
        for f in (lib.oracle_softmax_row, lib.oracle_attend_scores,
                  lib.oracle_attention_f64, lib.oracle_attention_rows_bf16,
                  lib.oracle_attention_blocked_f64, lib.oracle_max_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _threads(n):
    if n is None or n <= 0:
        return len(os.sched_getaffinity(0))
    return int(n)


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def bf16_bits(t) -> np.ndarray:
    """Raw uint16 bit patterns of a torch bfloat16 CPU tensor (same shape)."""
    import torch
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor")
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening: a bf16 pattern is the upper half of a binary32."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def softmax_row(s) -> np.ndarray:
    s = _f64(s)
    p = np.empty_like(s)
    _check(_load().oracle_softmax_row(_dptr(s), s.size, _dptr(p)), "softmax_row")
    return p


def attend_scores(S, V):
    """softmax_rows(S) @ V with -inf entries of S treated as masked keys."""
    S = _f64(S)
    V = _f64(V)
    rows, n_keys = S.shape
    d = V.shape[1]
    O = np.empty((rows, d))
    lse = np.empty(rows)
    _check(_load().oracle_attend_scores(_dptr(S), _dptr(V), rows, n_keys, d,
                                        _dptr(O), _dptr(lse)), "attend_scores")
    return O, lse


def attention(q, k, v, causal: bool, scale: float, threads=None):
    """Two-pass oracle on fp64 arrays shaped [B, H, N, d]; returns (O, lse)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    O = np.empty((B, H, N, d))
    lse = np.empty((B, H, N))
    _check(_load().oracle_attention_f64(
        _dptr(q), _dptr(k), _dptr(v), _dptr(O), _dptr(lse), B, H, N, d,
        int(bool(causal)), float(scale), _threads(threads)), "attention")
    return O, lse


def attention_blocked(q, k, v, causal: bool, scale: float, Br: int, Bc: int):
    """The pages' blocked online-softmax algorithm, fp64, single thread."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    O = np.empty((B, H, N, d))
    lse = np.empty((B, H, N))
    _check(_load().oracle_attention_blocked_f64(
        _dptr(q), _dptr(k), _dptr(v), _dptr(O), _dptr(lse), B, H, N, d,
        int(bool(causal)), float(scale), int(Br), int(Bc)), "attention_blocked")
    return O, lse


def attention_rows_bf16(qbits, kbits, vbits, causal: bool, scale: float,
                        rows, threads=None):
    """Oracle on selected flat rows (bh * N + i) of bf16 bit-pattern inputs
    shaped [B, H, N, d]; returns (O [len(rows), d], lse [len(rows)])."""
    qbits = np.ascontiguousarray(qbits, dtype=np.uint16)
    kbits = np.ascontiguousarray(kbits, dtype=np.uint16)
    vbits = np.ascontiguousarray(vbits, dtype=np.uint16)
    B, H, N, d = qbits.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.empty((rows.size, d))
    lse = np.empty(rows.size)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    _check(_load().oracle_attention_rows_bf16(
        qbits.ctypes.data_as(u16p), kbits.ctypes.data_as(u16p),
        vbits.ctypes.data_as(u16p), B, H, N, d, int(bool(causal)),
        float(scale), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        rows.size, _dptr(O), _dptr(lse), _threads(threads)),
        "attention_rows_bf16")
    return O, lse


def attention_backward(q, k, v, do, causal: bool, scale: float, threads=None):
    """Gradients (dQ, dK, dV) of the forward for upstream gradient dO; fp64
    arrays shaped [B, H, N, d]."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    dq = np.empty((B, H, N, d))
    dk = np.empty((B, H, N, d))
    dv = np.empty((B, H, N, d))
    _check(_load().oracle_attention_backward_f64(
        _dptr(q), _dptr(k), _dptr(v), _dptr(do), _dptr(dq), _dptr(dk),
        _dptr(dv), B, H, N, d, int(bool(causal)), float(scale),
        _threads(threads)), "attention_backward")
    return dq, dk, dv
