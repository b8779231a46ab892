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
        lib.oracle_attention_decode_f64.argtypes = [
            dp, dp, dp, dp, dp, i64, i64, i64, i64, ctypes.c_int,
            ctypes.c_double, ctypes.c_int]
        lib.oracle_attention_decode_rows_bf16.argtypes = [
            u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_int, ctypes.c_double,
            i64p, i64, dp, dp, ctypes.c_int]
        lib.oracle_attention_block_sparse_rows_bf16.argtypes = [
            u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_int, ctypes.c_double,
            ctypes.POINTER(ctypes.c_uint8), ctypes.c_int, i64p, i64, dp, dp,
            ctypes.c_int]
        lib.oracle_attention_block_sparse_rows_bf16.restype = ctypes.c_int
        lib.oracle_attention_backward_rows_bf16.argtypes = [
            u16p, u16p, u16p, u16p, i64, i64, ctypes.c_int, ctypes.c_double,
            i64p, i64, dp, i64p, i64, dp, dp, ctypes.c_int]
        for f in (lib.oracle_attention_decode_f64,
                  lib.oracle_attention_decode_rows_bf16,
                  lib.oracle_attention_backward_rows_bf16):
            f.restype = ctypes.c_int
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i8p = ctypes.POINTER(ctypes.c_int8)
        fp = ctypes.POINTER(ctypes.c_float)
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode_array.argtypes = [fp, i64, u8p]
        lib.oracle_hadamard_rotate.argtypes = [dp, i64, i64, i8p, dp]
        lib.oracle_fp8_quantize.argtypes = [u16p, i64, i64, i64, ctypes.c_int,
                                            i8p, i64, u8p, dp]
        lib.oracle_attention_fp8_rows.argtypes = [
            u8p, dp, u8p, dp, u8p, dp, i64, i64, i64, ctypes.c_int,
            ctypes.c_double, i64, i64, i64, ctypes.c_double, i64p, i64, dp, dp,
            ctypes.c_double, dp, ctypes.c_int]
        for f in (lib.oracle_e4m3_encode_array, lib.oracle_hadamard_rotate,
                  lib.oracle_fp8_quantize, lib.oracle_attention_fp8_rows):
            f.restype = ctypes.c_int
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


def attention_backward_rows_bf16(qbits, kbits, vbits, dobits, causal: bool,
                                 scale: float, qrows, krows, threads=None):
    """Backward on sampled rows of one head of bf16 bit patterns [N, d]:
    returns (dQ [len(qrows), d], dK [len(krows), d], dV [len(krows), d])."""
    qbits, kbits, vbits, dobits = (np.ascontiguousarray(a, dtype=np.uint16)
                                   for a in (qbits, kbits, vbits, dobits))
    N, d = qbits.shape[-2], qbits.shape[-1]
    if qbits.size != N * d:
        raise ValueError("one head: arrays shaped [N, d]")
    qrows = np.ascontiguousarray(qrows, dtype=np.int64)
    krows = np.ascontiguousarray(krows, dtype=np.int64)
    dQ = np.empty((qrows.size, d))
    dK = np.empty((krows.size, d))
    dV = np.empty((krows.size, d))
    u16p = ctypes.POINTER(ctypes.c_uint16)
    i64p = ctypes.POINTER(ctypes.c_int64)
    _check(_load().oracle_attention_backward_rows_bf16(
        qbits.ctypes.data_as(u16p), kbits.ctypes.data_as(u16p),
        vbits.ctypes.data_as(u16p), dobits.ctypes.data_as(u16p), N, d,
        int(bool(causal)), float(scale), qrows.ctypes.data_as(i64p), qrows.size,
        _dptr(dQ), krows.ctypes.data_as(i64p), krows.size, _dptr(dK), _dptr(dV),
        _threads(threads)), "attention_backward_rows_bf16")
    return dQ, dK, dV


def attention_decode(q, k, v, causal: bool, scale: float, threads=None):
    """Decode attention on fp64 arrays: q [..., Nq, d], k and v [..., Nk, d]
    (same leading dims); the queries are the last Nq positions, so the
    causal mask lets query i see keys 0 .. Nk - Nq + i.  Returns (O, lse)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Nq, d = q.shape[-2], q.shape[-1]
    Nk = k.shape[-2]
    BH = q.size // (Nq * d) if Nq else int(np.prod(q.shape[:-2]))
    O = np.empty(q.shape)
    lse = np.empty(q.shape[:-1])
    _check(_load().oracle_attention_decode_f64(
        _dptr(q), _dptr(k), _dptr(v), _dptr(O), _dptr(lse), BH, Nq, Nk, d,
        int(bool(causal)), float(scale), _threads(threads)), "attention_decode")
    return O, lse


def attention_decode_rows_bf16(qbits, kbits, vbits, causal: bool, scale: float,
                               rows, threads=None):
    """Decode attention on bf16 bit patterns for flat rows bh * Nq + i;
    returns (O [len(rows), d], lse [len(rows)])."""
    qbits, kbits, vbits = (np.ascontiguousarray(a, dtype=np.uint16)
                           for a in (qbits, kbits, vbits))
    Nq, d = qbits.shape[-2], qbits.shape[-1]
    Nk = kbits.shape[-2]
    BH = qbits.size // (Nq * d)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.empty((rows.size, d))
    lse = np.empty(rows.size)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    _check(_load().oracle_attention_decode_rows_bf16(
        qbits.ctypes.data_as(u16p), kbits.ctypes.data_as(u16p),
        vbits.ctypes.data_as(u16p), BH, Nq, Nk, d, int(bool(causal)),
        float(scale), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        rows.size, _dptr(O), _dptr(lse), _threads(threads)),
        "attention_decode_rows_bf16")
    return O, lse


# ---------------------------------------------------------------- FP8 path
# FP8 attention with incoherent processing (fp8_oracle.c): E4M3 codes,
# randomized Hadamard rotation of Q and K, power-of-two block scales, and the
# blocked online softmax with E4M3 probabilities.

def _u8ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes (round to nearest even, saturating) of float32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _check(_load().oracle_e4m3_encode_array(
        x.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), x.size, _u8ptr(out)),
        "e4m3_encode")
    return out


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of E4M3 codes."""
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([_load().oracle_e4m3_decode(c) for c in range(256)])
    return table[codes]


def _signs(signs, d):
    signs = np.ascontiguousarray(signs, dtype=np.int8)
    if signs.shape != (d,) or not np.all(np.abs(signs) == 1):
        raise ValueError("signs must be d entries of +-1")
    return signs


def hadamard_rotate(x, signs) -> np.ndarray:
    """x diag(signs) H (unscaled Sylvester Hadamard) for rows of x [..., d]."""
    x = _f64(x)
    d = x.shape[-1]
    signs = _signs(signs, d)
    y = np.empty_like(x)
    _check(_load().oracle_hadamard_rotate(
        _dptr(x), x.size // d, d,
        signs.ctypes.data_as(ctypes.POINTER(ctypes.c_int8)), _dptr(y)),
        "hadamard_rotate")
    return y


def fp8_quantize(bits, rotate: bool, signs=None, block_rows: int = 128):
    """Block quantization of bf16 bit patterns [B, H, N, d] (or [BH, N, d]):
    returns (codes uint8 same shape, scales float64 [BH, ceil(N/block_rows)])."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    N, d = bits.shape[-2], bits.shape[-1]
    BH = bits.size // (N * d)
    nblk = -(-N // int(block_rows))
    codes = np.empty(bits.shape, dtype=np.uint8)
    scales = np.empty((BH, nblk))
    sp = None
    if rotate:
        signs = _signs(signs, d)
        sp = signs.ctypes.data_as(ctypes.POINTER(ctypes.c_int8))
    _check(_load().oracle_fp8_quantize(
        bits.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)), BH, N, d,
        int(bool(rotate)), sp, int(block_rows), _u8ptr(codes), _dptr(scales)),
        "fp8_quantize")
    return codes, scales


# The base threshold of the FP8 kernel (log2 units): a row's base moves to a
# block maximum only when that exceeds it by more than this.
FP8_KERNEL_TAU = 4.0


def attention_fp8_rows(q8, q_scale, k8, k_scale, v8, v_scale, causal: bool,
                       scale: float, rows, block: int = 128, flip_delta=0.0,
                       threads=None, tau=0.0):
    """FP8 attention on codes [.., N, d] for flat rows (bh * N + i); Q and K
    scales per `block` rows, V one scale per head; the base of a row moves
    when a block maximum exceeds it by more than `tau` (log2 units; 0: the
    exact running maximum).  Returns (O, lse, flip_bound) with flip_bound
    None unless flip_delta > 0 (+inf for a row with a base decision within
    the score error of tau)."""
    q8, k8, v8 = (np.ascontiguousarray(a, dtype=np.uint8) for a in (q8, k8, v8))
    N, d = q8.shape[-2], q8.shape[-1]
    BH = q8.size // (N * d)
    qs, ks, vs = (_f64(a).reshape(BH, -1) for a in (q_scale, k_scale, v_scale))
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.empty((rows.size, d))
    lse = np.empty(rows.size)
    fb = np.empty(rows.size) if flip_delta > 0 else None
    _check(_load().oracle_attention_fp8_rows(
        _u8ptr(q8), _dptr(qs), _u8ptr(k8), _dptr(ks), _u8ptr(v8), _dptr(vs),
        BH, N, d, int(bool(causal)), float(scale), int(block), int(block), 128,
        float(tau), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), rows.size,
        _dptr(O), _dptr(lse), float(flip_delta),
        _dptr(fb) if fb is not None else None, _threads(threads)),
        "attention_fp8_rows")
    return O, lse, fb


def attention_fp8(q8, q_scale, k8, k_scale, v8, v_scale, causal: bool,
                  scale: float, block: int = 128, flip_delta=0.0, threads=None,
                  tau=0.0):
    """attention_fp8_rows over every row; O shaped like the codes."""
    shape = q8.shape
    N, d = shape[-2], shape[-1]
    rows = np.arange(q8.size // d, dtype=np.int64)
    O, lse, fb = attention_fp8_rows(q8, q_scale, k8, k_scale, v8, v_scale,
                                    causal, scale, rows, block, flip_delta,
                                    threads, tau)
    return (O.reshape(shape), lse.reshape(shape[:-1]),
            None if fb is None else fb.reshape(shape[:-1]))


def quantize_qkv_fp8(qbits, kbits, vbits, rotate: bool, signs=None):
    """The method's quantization of one problem: Q and K rotated (if asked)
    and quantized per 128-row tile, V per head.  Returns a dict of codes and
    scales plus the softmax-scale multiplier of the rotated problem."""
    d = qbits.shape[-1]
    q8, qs = fp8_quantize(qbits, rotate, signs, 128)
    k8, ks = fp8_quantize(kbits, rotate, signs, 128)
    v8, vs = fp8_quantize(vbits, False, None, vbits.shape[-2])
    return dict(q8=q8, qs=qs, k8=k8, ks=ks, v8=v8, vs=vs,
                gain=(1.0 / d) if rotate else 1.0)


def attention_full_bf16(qbits, kbits, vbits, causal: bool, scale: float,
                        threads=None, panel: int = 256):
    """The definition over EVERY row of bf16 bit-pattern inputs [B, H, N, d],
    with the score block of a panel of query rows formed by a library matrix
    product (float64 BLAS) instead of the C oracle's scalar loops; for the
    full-output checks of the largest workloads, where the row oracle would
    take many minutes.

    Per head and panel of `panel` query rows, the steps are those of the C
    oracle, in the same order ([MM] "Mengapa perhatian terikat pada
    memori"; the masked path of "Integrasinya delapan baris"):
        S = scale * Q_panel K^T          (keys up to the panel's last row
                                          when causal; later keys are masked)
        S[i, j] = -inf for j > i         (causal)
        m = rowmax S;  E = exp(S - m);  l = rowsum E
        O = (E V) / l;  lse = m + ln l
    Panels run on a thread pool with one BLAS thread each.  Returns float64
    (O [B, H, N, d], lse [B, H, N])."""
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits

    shape = tuple(qbits.shape)
    B, H, N, d = shape
    BH = B * H
    heads = [tuple(bf16_bits_to_f64(np.asarray(x).reshape(BH, N, d)[h])
                   for x in (qbits, kbits, vbits)) for h in range(BH)]
    O = np.empty((BH, N, d))
    lse = np.empty((BH, N))

    def one_panel(job):
        h, r0 = job
        q, k, v = heads[h]
        r1 = min(N, r0 + panel)
        n_keys = r1 if causal else N
        S = scale * (q[r0:r1] @ k[:n_keys].T)
        if causal:
            S[np.arange(n_keys)[None, :] > np.arange(r0, r1)[:, None]] = -np.inf
        m = S.max(axis=1)
        E = np.exp(S - m[:, None])
        l = E.sum(axis=1)
        O[h, r0:r1] = (E @ v[:n_keys]) / l[:, None]
        lse[h, r0:r1] = m + np.log(l)

    jobs = [(h, r0) for h in range(BH) for r0 in range(0, N, panel)]
    # heaviest panels first under the causal mask, so the pool ends together
    if causal:
        jobs.sort(key=lambda j: -j[1])
    with threadpool_limits(limits=1, user_api="blas"):
        with ThreadPoolExecutor(max_workers=_threads(threads)) as ex:
            for _ in ex.map(one_panel, jobs):
                pass
    return O.reshape(shape), lse.reshape(shape[:-1])


def attention_block_sparse_rows_bf16(qbits, kbits, vbits, causal: bool,
                                     scale: float, block_mask, rows,
                                     threads=None):
    """Block-sparse attention ([MM]'s definition with the scores of the
    (128-query, 128-key) blocks the mask leaves out set to -inf; rows with no
    key left give O = 0, lse = -inf) on selected flat rows (bh * N + i) of
    bf16 bit patterns [B, H, N, d].  block_mask: uint8 [T, T] shared by all
    heads or [B, H, T, T] (or [B * H, T, T]) per head, T = ceil(N / 128).
    Returns (O [len(rows), d], lse [len(rows)])."""
    qbits = np.ascontiguousarray(qbits, dtype=np.uint16)
    kbits = np.ascontiguousarray(kbits, dtype=np.uint16)
    vbits = np.ascontiguousarray(vbits, dtype=np.uint16)
    B, H, N, d = qbits.shape
    T = -(-N // 128)
    m = np.ascontiguousarray(block_mask, dtype=np.uint8)
    per_head = int(m.size != T * T)
    if m.size not in (T * T, B * H * T * T):
        raise ValueError("block_mask must hold T*T or B*H*T*T bytes")
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.empty((rows.size, d))
    lse = np.empty(rows.size)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    _check(_load().oracle_attention_block_sparse_rows_bf16(
        qbits.ctypes.data_as(u16p), kbits.ctypes.data_as(u16p),
        vbits.ctypes.data_as(u16p), B, H, N, d, int(bool(causal)),
        float(scale), m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
        per_head, rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        rows.size, _dptr(O), _dptr(lse), _threads(threads)),
        "attention_block_sparse_rows_bf16")
    return O, lse


def attention_block_sparse_bf16(qbits, kbits, vbits, causal: bool, scale: float,
                                block_mask, threads=None):
    """attention_block_sparse_rows_bf16 over every row; O [B, H, N, d],
    lse [B, H, N]."""
    B, H, N, d = qbits.shape
    rows = np.arange(B * H * N, dtype=np.int64)
    O, lse = attention_block_sparse_rows_bf16(qbits, kbits, vbits, causal, scale,
                                              block_mask, rows, threads)
    return O.reshape(B, H, N, d), lse.reshape(B, H, N)
