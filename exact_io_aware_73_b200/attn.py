"""Thin ctypes binding of ``libattn_b200.so`` (C ABI in ``include/attn_b200.h``).

Argument marshalling only: every step of the attention forward pass runs in
the library's sm_100a kernel.  There is no fallback of any kind -- if the
library is missing or refuses the call, these functions raise.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libattn_b200.so")
# the same library built with the kernels' index checks (ATTN_DEBUG_BOUNDS)
DEBUG_LIB_PATH = os.path.join(PKG, "libattn_b200_debug.so")

ATTN_OK = 0
ERROR_NAMES = {
    1: "ATTN_ERR_NULL_POINTER", 2: "ATTN_ERR_INVALID_SIZE",
    3: "ATTN_ERR_UNSUPPORTED_HEAD_DIM", 4: "ATTN_ERR_MISALIGNED",
    5: "ATTN_ERR_INVALID_SCALE", 6: "ATTN_ERR_ALIAS",
    7: "ATTN_ERR_UNSUPPORTED_DEVICE", 8: "ATTN_ERR_CUDA",
    9: "ATTN_ERR_TENSOR_MAP", 10: "ATTN_ERR_NOT_DEVICE_MEMORY",
    11: "ATTN_ERR_WORKSPACE", 12: "ATTN_ERR_NOALLOC_TOO_LARGE",
    16: "ATTN_ERR_DEVICE_TIMEOUT",
    17: "ATTN_ERR_DEVICE_BOUNDS",
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = lib().attn_strerror(code).decode()
        super().__init__(f"{what}: {ERROR_NAMES.get(code, code)} ({msg})")


def lib():
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m exact_io_aware_73_b200.build` (no fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i = ctypes.c_void_p, ctypes.c_int
        L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i,
                               ctypes.c_float, vp]
        L.attn_fwd.restype = i
        L.attn_fwd_host.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i,
                                    ctypes.c_float, vp, ctypes.c_size_t, vp]
        L.attn_fwd_host.restype = i
        L.attn_fwd_host_workspace_bytes.argtypes = [i, i, i, i]
        L.attn_fwd_host_workspace_bytes.restype = ctypes.c_size_t
        L.attn_status.argtypes = [vp]
        L.attn_status.restype = i
        L.attn_last_status_bits.argtypes = []
        L.attn_last_status_bits.restype = ctypes.c_uint32
        L.attn_strerror.argtypes = [i]
        L.attn_strerror.restype = ctypes.c_char_p
        L.attn_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        L.attn_set_wait_timeout_ns.restype = None
        L.attn_set_fault_injection.argtypes = [ctypes.c_uint32]
        L.attn_set_fault_injection.restype = None
        _lib = L
    return _lib


def _stream_handle(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(getattr(stream, "cuda_stream", stream))


def _check(rc: int, what: str):
    if rc != ATTN_OK:
        raise AttnError(rc, what)


def _expect(name, t, dtype, shape=None, cuda=True, device=None, numel=None):
    """Refuse a tensor the C ABI would misread: it sees only a pointer, so
    dtype, layout (contiguous) and shape are checked here (or only the
    element count, for arrays whose leading dimensions may be merged)."""
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.is_cuda != cuda:
        where = "CUDA" if cuda else "host"
        raise TypeError(f"{name} must be a {dtype} {where} tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, like the queries")


def _expect_qkv(q, k, v, cuda=True):
    """q, k, v: 4-D bf16 tensors of one shape [B, H, N, d] (on one device)."""
    import torch
    _expect("q", q, torch.bfloat16, cuda=cuda)
    if q.dim() != 4:
        raise ValueError("q must be 4-D [B, H, N, d]")
    dev = q.device if cuda else None
    _expect("k", k, torch.bfloat16, q.shape, cuda, dev)
    _expect("v", v, torch.bfloat16, q.shape, cuda, dev)


def attn_fwd_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, causal,
                 scale, stream_handle) -> int:
    """Direct call with integer pointers; returns the library's code."""
    return lib().attn_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, int(B), int(H),
                          int(N), int(d), int(bool(causal)), float(scale),
                          stream_handle)


def attn_fwd(q, k, v, causal: bool = False, scale: float | None = None,
             out=None, lse=None, stream=None):
    """O, lse = exact attention forward of bf16 CUDA tensors [B, H, N, d].

    Allocates O (bf16) and lse (fp32 [B, H, N]) with torch unless given.
    """
    import torch
    _expect_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _expect("out", out, torch.bfloat16, q.shape, device=q.device)
    _expect("lse", lse, torch.float32, (B, H, N), device=q.device)
    rc = attn_fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                      lse.data_ptr(), B, H, N, d, causal, scale,
                      _stream_handle(stream))
    _check(rc, "attn_fwd")
    return out, lse


def _sparse_fn():
    f = lib().attn_fwd_block_sparse
    if f.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        f.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, ctypes.c_float, vp, i, vp]
        f.restype = i
    return f


def attn_fwd_block_sparse_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d,
                              causal, scale, mask_ptr, mask_per_head,
                              stream_handle) -> int:
    """Direct call with integer pointers; returns the library's code."""
    return _sparse_fn()(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, int(B), int(H),
                        int(N), int(d), int(bool(causal)), float(scale),
                        mask_ptr, int(bool(mask_per_head)), stream_handle)


def attn_fwd_block_sparse(q, k, v, block_mask, causal: bool = False,
                          scale: float | None = None, out=None, lse=None,
                          stream=None):
    """O, lse of block-sparse attention: attn_fwd with the (128-query,
    128-key) blocks that block_mask zeroes left out.  block_mask: uint8 CUDA
    tensor [T, T] for every head, or [B, H, T, T] / [B*H, T, T] per head,
    T = ceil(N / 128).  Rows with no key left get O = 0, lse = -inf."""
    import torch
    _expect_qkv(q, k, v)
    B, H, N, d = q.shape
    T = -(-N // 128)
    if not isinstance(block_mask, torch.Tensor) or block_mask.dtype != torch.uint8:
        raise TypeError("block_mask must be a uint8 CUDA tensor")
    if block_mask.numel() not in (T * T, B * H * T * T):
        raise ValueError(f"block_mask must hold {T}x{T} bytes or one such mask per head")
    _expect("block_mask", block_mask, torch.uint8, device=q.device)
    per_head = block_mask.numel() != T * T
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _expect("out", out, torch.bfloat16, q.shape, device=q.device)
    _expect("lse", lse, torch.float32, (B, H, N), device=q.device)
    rc = attn_fwd_block_sparse_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                   out.data_ptr(), lse.data_ptr(), B, H, N, d,
                                   causal, scale, block_mask.data_ptr(), per_head,
                                   _stream_handle(stream))
    _check(rc, "attn_fwd_block_sparse")
    return out, lse


def attn_fwd_host(q, k, v, out, lse, causal: bool, scale: float, workspace,
                  stream=None):
    """End-to-end call on host (ideally pinned) bf16 tensors; `workspace` is a
    CUDA uint8 tensor of at least ``host_workspace_bytes`` bytes.  Queued on
    `stream`; synchronise before reading `out` / `lse`."""
    import torch
    _expect_qkv(q, k, v, cuda=False)
    B, H, N, d = q.shape
    _expect("out", out, torch.bfloat16, q.shape, cuda=False)
    _expect("lse", lse, torch.float32, (B, H, N), cuda=False)
    _expect("workspace", workspace, torch.uint8)
    rc = lib().attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                             out.data_ptr(), lse.data_ptr(), B, H, N, d,
                             int(bool(causal)), float(scale),
                             workspace.data_ptr(), workspace.numel(),
                             _stream_handle(stream))
    _check(rc, "attn_fwd_host")


def host_workspace_bytes(B, H, N, d) -> int:
    return int(lib().attn_fwd_host_workspace_bytes(B, H, N, d))


def status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status."""
    return int(lib().attn_status(_stream_handle(stream)))


def last_status_bits() -> int:
    return int(lib().attn_last_status_bits())


def strerror(code: int) -> str:
    return lib().attn_strerror(int(code)).decode()


def set_wait_timeout_ns(ns: int) -> None:
    lib().attn_set_wait_timeout_ns(int(ns))


def set_fault_injection(flags: int) -> None:
    lib().attn_set_fault_injection(int(flags))


# Scratch size of attn_fwd_host_noalloc's static device array (bytes).
NOALLOC_SCRATCH_BYTES = 32 << 20


def _noalloc_fn():
    f = lib().attn_fwd_host_noalloc
    if f.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        f.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, ctypes.c_float, vp]
        f.restype = i
    return f


def attn_fwd_host_noalloc(q, k, v, out, lse, causal: bool, scale: float,
                          stream=None):
    """Host-buffer attention that allocates no device memory: its scratch is
    a static 32 MiB device array inside the library, shared by every call on
    the device (so overlapping calls race).  Synchronous: `out` and `lse` are
    filled on return.  For callers without a device allocator of their own."""
    import torch
    _expect_qkv(q, k, v, cuda=False)
    B, H, N, d = q.shape
    _expect("out", out, torch.bfloat16, q.shape, cuda=False)
    _expect("lse", lse, torch.float32, (B, H, N), cuda=False)
    rc = _noalloc_fn()(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                       out.data_ptr(), lse.data_ptr(), B, H, N, d,
                       int(bool(causal)), float(scale), _stream_handle(stream))
    _check(rc, "attn_fwd_host_noalloc")


def selftest_exp2(x, mode: int, stream=None):
    """y = 2^x for a float32 CUDA tensor, evaluated as the kernel does:
    mode 0 = FMA-pipe polynomial, mode 1 = ex2.approx (test hook)."""
    import torch
    f = lib().attn_selftest_exp2
    if f.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        f.argtypes = [vp, vp, i, i, vp]
        f.restype = i
    x = x.contiguous()
    y = torch.empty_like(x)
    _check(f(x.data_ptr(), y.data_ptr(), x.numel(), int(mode),
             _stream_handle(stream)), "attn_selftest_exp2")
    return y


def _bwd_fns():
    L = lib()
    f, g = L.attn_bwd, L.attn_bwd_workspace_bytes
    if f.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        f.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                      i, i, i, i, i, ctypes.c_float, vp]
        f.restype = i
        g.argtypes = [i, i, i]
        g.restype = ctypes.c_size_t
    return f, g


def bwd_workspace_bytes(B, H, N) -> int:
    return int(_bwd_fns()[1](B, H, N))


def attn_bwd_raw(q, k, v, o, dout, lse, dq, dk, dv, ws, ws_bytes, B, H, N, d,
                 causal, scale, stream_handle) -> int:
    """Direct call with integer pointers; returns the library's code."""
    return _bwd_fns()[0](q, k, v, o, dout, lse, dq, dk, dv, ws, ws_bytes,
                         int(B), int(H), int(N), int(d), int(bool(causal)),
                         float(scale), stream_handle)


def attn_bwd(q, k, v, o, lse, dout, causal: bool = False,
             scale: float | None = None, stream=None, workspace=None):
    """dQ, dK, dV of attn_fwd for upstream gradient dout (bf16 CUDA tensors
    [B, H, N, d]; o and lse are attn_fwd's outputs)."""
    import torch
    _expect_qkv(q, k, v)
    B, H, N, d = q.shape
    _expect("o", o, torch.bfloat16, q.shape, device=q.device)
    _expect("dout", dout, torch.bfloat16, q.shape, device=q.device)
    _expect("lse", lse, torch.float32, (B, H, N), device=q.device)
    if scale is None:
        scale = d ** -0.5
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    need = bwd_workspace_bytes(B, H, N)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _expect("workspace", workspace, torch.uint8, device=q.device)
    rc = attn_bwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                      dout.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                      dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                      workspace.numel(), B, H, N, d, causal, scale,
                      _stream_handle(stream))
    _check(rc, "attn_bwd")
    return dq, dk, dv


# ------------------------------------------------------------------ FP8 path

def _fp8_fns():
    L = lib()
    if L.attn_fwd_fp8.argtypes is None:
        vp, i, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64
        L.attn_fp8_quantize.argtypes = [vp, vp, vp, vp, i, i, i, i, i, u64, u64,
                                        i, vp]
        L.attn_fp8_quantize.restype = i
        L.attn_fwd_fp8_quantized.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i,
                                             i, i, i, i, ctypes.c_float, vp]
        L.attn_fwd_fp8_quantized.restype = i
        L.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i,
                                   ctypes.c_float, i, u64, u64, vp,
                                   ctypes.c_size_t, vp]
        L.attn_fwd_fp8.restype = i
        L.attn_fwd_fp8_workspace_bytes.argtypes = [i, i, i, i]
        L.attn_fwd_fp8_workspace_bytes.restype = ctypes.c_size_t
        L.attn_fwd_fp8_host.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i,
                                        ctypes.c_float, i, u64, u64, vp,
                                        ctypes.c_size_t, vp]
        L.attn_fwd_fp8_host.restype = i
        L.attn_fwd_fp8_host_workspace_bytes.argtypes = [i, i, i, i]
        L.attn_fwd_fp8_host_workspace_bytes.restype = ctypes.c_size_t
    return L


def sign_mask(signs) -> tuple[int, int]:
    """(sign_lo, sign_hi) bit masks of a +-1 sequence of length <= 128:
    bit t set where signs[t] == -1."""
    lo = hi = 0
    for t, s in enumerate(int(x) for x in signs):
        if s not in (1, -1):
            raise ValueError("signs must be +-1")
        if s < 0:
            if t < 64:
                lo |= 1 << t
            else:
                hi |= 1 << (t - 64)
    return lo, hi


def fp8_workspace_bytes(B, H, N, d) -> int:
    return int(_fp8_fns().attn_fwd_fp8_workspace_bytes(B, H, N, d))


def fp8_quantize_raw(x, x8, scales, tile_amax, B, H, N, d, rotate, sign_lo,
                     sign_hi, per_head, stream_handle) -> int:
    return _fp8_fns().attn_fp8_quantize(x, x8, scales, tile_amax, int(B), int(H),
                                        int(N), int(d), int(bool(rotate)),
                                        int(sign_lo), int(sign_hi),
                                        int(bool(per_head)), stream_handle)


def fp8_quantize(x, rotate: bool, signs=None, per_head: bool = False,
                 stream=None):
    """E4M3 codes (uint8, same shape) and fp32 scales of a bf16 CUDA tensor
    [B, H, N, 128]: per 128-row tile ([B, H, ceil(N/128)]) or per head
    ([B, H]); Q and K rotated with the signs when `rotate`."""
    import torch
    _expect("x", x, torch.bfloat16)
    if x.dim() != 4:
        raise ValueError("x must be 4-D [B, H, N, d]")
    B, H, N, d = x.shape
    lo, hi = sign_mask(signs) if rotate else (0, 0)
    tiles = -(-N // 128)
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty((B, H) if per_head else (B, H, tiles),
                         dtype=torch.float32, device=x.device)
    amax = (torch.empty((B, H, tiles), dtype=torch.float32, device=x.device)
            if per_head else None)
    rc = fp8_quantize_raw(x.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                          amax.data_ptr() if amax is not None else None,
                          B, H, N, d, rotate, lo, hi, per_head,
                          _stream_handle(stream))
    _check(rc, "attn_fp8_quantize")
    return codes, scales


def attn_fwd_fp8_quantized(q8, q_scale, k8, k_scale, v8, v_scale, causal: bool,
                           scale: float, stream=None):
    """O (bf16), lse of the FP8 attention on quantized operands; `scale` is
    the softmax scale of the problem the codes encode."""
    import torch
    _expect("q8", q8, torch.uint8)
    if q8.dim() != 4:
        raise ValueError("q8 must be 4-D [B, H, N, d]")
    B, H, N, d = q8.shape
    tiles = -(-N // 128)
    dev = q8.device
    _expect("k8", k8, torch.uint8, q8.shape, device=dev)
    _expect("v8", v8, torch.uint8, q8.shape, device=dev)
    # scales: [B, H, tiles] and [B, H] in memory (any merging of B and H)
    _expect("q_scale", q_scale, torch.float32, device=dev, numel=B * H * tiles)
    _expect("k_scale", k_scale, torch.float32, device=dev, numel=B * H * tiles)
    _expect("v_scale", v_scale, torch.float32, device=dev, numel=B * H)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    rc = _fp8_fns().attn_fwd_fp8_quantized(
        q8.data_ptr(), q_scale.data_ptr(), k8.data_ptr(), k_scale.data_ptr(),
        v8.data_ptr(), v_scale.data_ptr(), o.data_ptr(), lse.data_ptr(),
        B, H, N, d, int(bool(causal)), float(scale), _stream_handle(stream))
    _check(rc, "attn_fwd_fp8_quantized")
    return o, lse


def attn_fwd_fp8_raw(q, k, v, o, lse, B, H, N, d, causal, scale, rotate,
                     sign_lo, sign_hi, ws, ws_bytes, stream_handle) -> int:
    return _fp8_fns().attn_fwd_fp8(q, k, v, o, lse, int(B), int(H), int(N),
                                   int(d), int(bool(causal)), float(scale),
                                   int(bool(rotate)), int(sign_lo),
                                   int(sign_hi), ws, ws_bytes, stream_handle)


def attn_fwd_fp8(q, k, v, causal: bool = False, scale: float | None = None,
                 signs=None, workspace=None, out=None, lse=None, stream=None):
    """FP8 attention forward of bf16 CUDA tensors [B, H, N, 128]: Q and K
    rotated with `signs` (+-1, length 128; None = no rotation, naive FP8)
    and block-quantized to E4M3 with V, then the FP8 kernel.  Returns
    (O bf16, lse fp32)."""
    import torch
    _expect_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = d ** -0.5
    lo, hi = sign_mask(signs) if signs is not None else (0, 0)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _expect("out", out, torch.bfloat16, q.shape, device=q.device)
    _expect("lse", lse, torch.float32, (B, H, N), device=q.device)
    need = fp8_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _expect("workspace", workspace, torch.uint8, device=q.device)
    rc = attn_fwd_fp8_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                          out.data_ptr(), lse.data_ptr(), B, H, N, d, causal,
                          scale, signs is not None, lo, hi,
                          workspace.data_ptr(), workspace.numel(),
                          _stream_handle(stream))
    _check(rc, "attn_fwd_fp8")
    return out, lse


def fp8_host_workspace_bytes(B, H, N, d) -> int:
    return int(_fp8_fns().attn_fwd_fp8_host_workspace_bytes(B, H, N, d))


def attn_fwd_fp8_host(q, k, v, out, lse, causal: bool, scale: float, workspace,
                      signs=None, stream=None):
    """attn_fwd_fp8 end to end on host (ideally pinned) bf16 tensors
    [B, H, N, 128]: copies in, rotation and quantization, the FP8 kernel and
    copies out, overlapped by head chunks; `workspace` is a CUDA uint8
    tensor of at least ``fp8_host_workspace_bytes`` bytes.  Queued on
    `stream`; synchronise before reading `out` / `lse`."""
    import torch
    _expect_qkv(q, k, v, cuda=False)
    B, H, N, d = q.shape
    _expect("out", out, torch.bfloat16, q.shape, cuda=False)
    _expect("lse", lse, torch.float32, (B, H, N), cuda=False)
    _expect("workspace", workspace, torch.uint8)
    lo, hi = sign_mask(signs) if signs is not None else (0, 0)
    rc = _fp8_fns().attn_fwd_fp8_host(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
        B, H, N, d, int(bool(causal)), float(scale), int(signs is not None), lo, hi,
        workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check(rc, "attn_fwd_fp8_host")


# ------------------------------------------------------------------ decode

def _decode_fns():
    L = lib()
    if L.attn_decode.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        L.attn_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                  ctypes.c_float, vp, ctypes.c_size_t, vp]
        L.attn_decode.restype = i
        L.attn_decode_workspace_bytes.argtypes = [i, i, i, i, i]
        L.attn_decode_workspace_bytes.restype = ctypes.c_size_t
        L.attn_set_decode_max_ctas.argtypes = [i]
        L.attn_set_decode_max_ctas.restype = None
        L.attn_set_decode_kernel.argtypes = [i]
        L.attn_set_decode_kernel.restype = None
        L.attn_decode_kernel_for.argtypes = [i, i]
        L.attn_decode_kernel_for.restype = i
    return L


DECODE_MAX_Q = 16   # queries per (batch, head) and call
DECODE_GROUP_Q = 4  # the CUDA-core kernel's queries per launch (the
                    # tensor-core kernel serves all of them in one)


def decode_workspace_bytes(B, H, Nq, Nk, d) -> int:
    return int(_decode_fns().attn_decode_workspace_bytes(B, H, Nq, Nk, d))


def set_decode_max_ctas(n: int) -> None:
    """Test hook: cap attn_decode's CTA count (0 restores the default)."""
    _decode_fns().attn_set_decode_max_ctas(int(n))


DECODE_AUTO, DECODE_CUDA_CORES, DECODE_TENSOR_CORES = 0, 1, 2


def set_decode_kernel(which: int) -> None:
    """Test hook: force the CUDA-core (1) or tensor-core (2) decode kernel;
    0 restores the library's choice."""
    _decode_fns().attn_set_decode_kernel(int(which))


def decode_kernel_for(Nq: int, d: int) -> int:
    """The decode kernel attn_decode would run: 1 CUDA cores, 2 tensor cores."""
    return int(_decode_fns().attn_decode_kernel_for(int(Nq), int(d)))


def attn_decode_raw(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, ws,
                    ws_bytes, stream_handle) -> int:
    return _decode_fns().attn_decode(q, k, v, o, lse, int(B), int(H), int(Nq),
                                     int(Nk), int(d), int(bool(causal)),
                                     float(scale), ws, ws_bytes, stream_handle)


def attn_decode(q, k, v, causal: bool = True, scale: float | None = None,
                workspace=None, out=None, lse=None, stream=None):
    """Split-KV decode: q bf16 [B, H, Nq, d] (the last Nq positions, Nq <= 16,
    all in one tensor-core launch unless set_decode_kernel forces the
    CUDA-core kernel) against k, v bf16 [B, H, Nk, d]; returns (O bf16, lse
    fp32 [B, H, Nq])."""
    import torch
    _expect("q", q, torch.bfloat16)
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be 4-D [B, H, Nq, d] and [B, H, Nk, d]")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    _expect("k", k, torch.bfloat16, (B, H, Nk, d), device=q.device)
    _expect("v", v, torch.bfloat16, (B, H, Nk, d), device=q.device)
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _expect("out", out, torch.bfloat16, q.shape, device=q.device)
    _expect("lse", lse, torch.float32, (B, H, Nq), device=q.device)
    need = decode_workspace_bytes(B, H, Nq, Nk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _expect("workspace", workspace, torch.uint8, device=q.device)
    rc = attn_decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                         out.data_ptr(), lse.data_ptr(), B, H, Nq, Nk, d,
                         causal, scale, workspace.data_ptr(), workspace.numel(),
                         _stream_handle(stream))
    _check(rc, "attn_decode")
    return out, lse


# ------------------------------------------------------------------ merge

def _merge_fns():
    L = lib()
    if L.attn_merge_fold.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        L.attn_merge_fold.argtypes = [vp, vp, vp, vp, ctypes.c_int64, i, i, vp]
        L.attn_merge_fold.restype = i
        L.attn_merge_finish.argtypes = [vp, vp, vp, vp, ctypes.c_int64, i, vp]
        L.attn_merge_finish.restype = i
    return L


def merge_fold(acc_o, acc_lse, part_o, part_lse, first: bool, stream=None):
    """Fold a partial result (part_o bf16 [..., d], part_lse fp32 [...]) into
    the fp32 accumulator (acc_o [..., d], acc_lse [...]) by the exact
    log-sum-exp merge; `first` initialises the accumulator."""
    import torch
    _expect("part_lse", part_lse, torch.float32)
    dev = part_lse.device
    d = part_o.shape[-1] if part_o.dim() else 0
    rows = part_lse.numel()
    _expect("part_o", part_o, torch.bfloat16, (*part_lse.shape, d), device=dev)
    _expect("acc_o", acc_o, torch.float32, (*part_lse.shape, d), device=dev)
    _expect("acc_lse", acc_lse, torch.float32, part_lse.shape, device=dev)
    rc = _merge_fns().attn_merge_fold(acc_o.data_ptr(), acc_lse.data_ptr(),
                                      part_o.data_ptr(), part_lse.data_ptr(),
                                      rows, d, int(bool(first)),
                                      _stream_handle(stream))
    _check(rc, "attn_merge_fold")


def merge_finish(acc_o, acc_lse, stream=None):
    """(O bf16, lse fp32) from a merge accumulator."""
    import torch
    _expect("acc_lse", acc_lse, torch.float32)
    d = acc_o.shape[-1] if acc_o.dim() else 0
    _expect("acc_o", acc_o, torch.float32, (*acc_lse.shape, d), device=acc_lse.device)
    o = torch.empty(acc_o.shape, dtype=torch.bfloat16, device=acc_o.device)
    lse = torch.empty_like(acc_lse)
    rc = _merge_fns().attn_merge_finish(acc_o.data_ptr(), acc_lse.data_ptr(),
                                        o.data_ptr(), lse.data_ptr(),
                                        acc_lse.numel(), acc_o.shape[-1],
                                        _stream_handle(stream))
    _check(rc, "attn_merge_finish")
    return o, lse


# modes of attn_fwd_merge
MERGE_FIRST, MERGE_INTO, MERGE_LAST = 1, 2, 3


def attn_fwd_merge(q, k, v, acc_o, acc_lse, mode: int, causal: bool = False,
                   scale: float | None = None, stream=None):
    """attn_fwd folded into the fp32 accumulator (acc_o [B, H, N, d],
    acc_lse [B, H, N]) in the kernel's epilogue.  mode MERGE_FIRST writes it,
    MERGE_INTO merges into it, MERGE_LAST returns the merged (O bf16, lse)."""
    import torch
    L = lib()
    f = L.attn_fwd_merge
    if f.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        f.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, ctypes.c_float, i, vp]
        f.restype = i
    _expect_qkv(q, k, v)
    B, H, N, d = q.shape
    _expect("acc_o", acc_o, torch.float32, q.shape, device=q.device)
    _expect("acc_lse", acc_lse, torch.float32, (B, H, N), device=q.device)
    if scale is None:
        scale = d ** -0.5
    o = lse = None
    if mode == MERGE_LAST:
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), acc_o.data_ptr(),
           acc_lse.data_ptr(), o.data_ptr() if o is not None else None,
           lse.data_ptr() if lse is not None else None, B, H, N, d,
           int(bool(causal)), float(scale), int(mode), _stream_handle(stream))
    _check(rc, "attn_fwd_merge")
    return (o, lse) if mode == MERGE_LAST else None
