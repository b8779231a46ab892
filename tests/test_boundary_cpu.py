"""The C-ABI library on the CPU: it loads, exports every function the header
declares, and rejects bad arguments before touching CUDA (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def attn():
    from exact_io_aware_73_b200 import build
    build.build()
    from exact_io_aware_73_b200 import attn as a
    return a


def _declared_functions():
    names = set()
    for f in os.listdir(HEADER_DIR):
        if not f.endswith(".h"):
            continue
        src = open(os.path.join(HEADER_DIR, f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", src,
                             flags=re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for required in ("attn_fwd", "attn_fwd_host", "attn_status",
                     "attn_strerror", "attn_fwd_host_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(attn):
    lib = attn.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", attn.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared_functions():
        assert name in exported, name
        assert hasattr(lib, name), name


def test_debug_library_exports_the_same_entry_points(attn):
    """The debug build (kernels' index checks compiled in) is the same ABI;
    built here if missing, as the build step does."""
    from exact_io_aware_73_b200 import build
    path = build.build(debug=True)
    assert path == attn.DEBUG_LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", path],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared_functions():
        assert name in exported, name
    dbg = ctypes.CDLL(path)
    dbg.attn_strerror.restype = ctypes.c_char_p
    dbg.attn_strerror.argtypes = [ctypes.c_int]
    assert b"index check" in dbg.attn_strerror(17)
    assert attn.ERROR_NAMES[17] == "ATTN_ERR_DEVICE_BOUNDS"


def test_build_targets_sm100a_only():
    from exact_io_aware_73_b200 import build
    f = build.flags()
    gencodes = [f[i + 1] for i, x in enumerate(f) if x == "-gencode"]
    assert gencodes == ["arch=compute_100a,code=sm_100a"]


def _call(attn, q=8, k=8, v=8, o=8, lse=8, B=1, H=1, N=16, d=64, causal=0,
          scale=0.125):
    # fake (non-null) pointers: every one of these cases must be refused
    # before any CUDA call, so nothing is ever dereferenced
    return attn.attn_fwd_raw(q, k, v, o, lse, B, H, N, d, causal, scale, None)


def test_argument_errors_need_no_device(attn):
    far = 1 << 40
    assert _call(attn, q=None) == 1
    assert _call(attn, lse=None) == 1
    assert _call(attn, B=-1) == 2
    assert _call(attn, N=(1 << 24) + 1, q=far, k=2 * far, v=3 * far,
                 o=4 * far, lse=5 * far) == 2
    assert _call(attn, d=96) == 3
    assert _call(attn, d=256) == 3
    assert _call(attn, q=far + 8, k=2 * far, v=3 * far, o=4 * far,
                 lse=5 * far) == 4
    assert _call(attn, q=far, k=2 * far, v=3 * far, o=4 * far,
                 lse=5 * far + 2) == 4
    assert _call(attn, scale=0.0) == 5
    assert _call(attn, scale=float("nan")) == 5
    assert _call(attn, scale=float("inf")) == 5
    assert _call(attn, scale=-0.5) == 5
    # o overlapping q
    assert _call(attn, q=far, k=2 * far, v=3 * far, o=far + 1024,
                 lse=5 * far) == 6
    # lse overlapping o
    assert _call(attn, q=far, k=2 * far, v=3 * far, o=4 * far,
                 lse=4 * far + 64) == 6


def test_empty_problem_is_a_no_op(attn):
    for B, H, N in ((0, 1, 16), (1, 0, 16), (1, 1, 0)):
        assert _call(attn, q=None, k=None, v=None, o=None, lse=None, B=B, H=H,
                     N=N) == 0


def test_no_device_is_reported_not_crashed(attn):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    far = 1 << 40
    assert _call(attn, q=far, k=2 * far, v=3 * far, o=4 * far,
                 lse=5 * far) == 7


def test_host_entry_workspace_checks(attn):
    assert attn.host_workspace_bytes(2, 3, 100, 64) == \
        4 * ((2 * 3 * 100 * 64 * 2 + 255) // 256 * 256) + \
        (2 * 3 * 100 * 4 + 255) // 256 * 256
    assert attn.host_workspace_bytes(1, 1, 16, 96) == 0
    lib = attn.lib()
    buf = ctypes.create_string_buffer(1 << 16)
    p = ctypes.addressof(buf)
    # workspace missing / too small are refused before any CUDA call
    rc = lib.attn_fwd_host(p, p + 4096, p + 8192, p + 12288, p + 16384, 1, 1,
                           16, 64, 0, 0.125, None, 0, None)
    assert rc == 11
    rc = lib.attn_fwd_host(p, p + 4096, p + 8192, p + 12288, p + 16384, 1, 1,
                           16, 64, 0, 0.125, 1 << 40, 16, None)
    assert rc == 11


def test_strerror_covers_every_code(attn):
    for code in list(attn.ERROR_NAMES) + [0]:
        text = attn.strerror(code)
        assert text and text != "unknown error code"
    assert attn.strerror(12345) == "unknown error code"


def test_python_binding_has_no_fallback(tmp_path, monkeypatch):
    """With the library missing, the binding raises instead of computing."""
    from exact_io_aware_73_b200 import attn as a
    monkeypatch.setattr(a, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(a, "_lib", None)
    with pytest.raises(ImportError):
        a.lib()


def test_fp8_entries_refuse_bad_arguments_without_a_device(attn):
    far = 1 << 40
    # d other than 128
    assert attn.fp8_quantize_raw(far, 2 * far, 3 * far, None, 1, 1, 16, 64, 1,
                                 0, 0, 0, None) == 3
    # per-head quantization needs the tile-amax scratch
    assert attn.fp8_quantize_raw(far, 2 * far, 3 * far, None, 1, 1, 16, 128, 0,
                                 0, 0, 1, None) == 1
    assert attn.fp8_quantize_raw(far + 8, 2 * far, 3 * far, None, 1, 1, 16, 128,
                                 0, 0, 0, 0, None) == 4
    # codes overlapping the input
    assert attn.fp8_quantize_raw(far, far + 64, 3 * far, None, 1, 1, 16, 128, 0,
                                 0, 0, 0, None) == 6
    # whole path: workspace missing or too small
    args = [far, 2 * far, 3 * far, 4 * far, 5 * far, 1, 1, 16, 128, 0, 0.125, 1,
            0, 0]
    assert attn.attn_fwd_fp8_raw(*args, None, 0, None) == 11
    assert attn.attn_fwd_fp8_raw(*args, 6 * far, 16, None) == 11
    assert attn.attn_fwd_fp8_raw(*(args[:8] + [64] + args[9:]), 6 * far,
                                 1 << 30, None) == 3
    # empty problems are no-ops
    assert attn.attn_fwd_fp8_raw(None, None, None, None, None, 0, 1, 16, 128, 0,
                                 0.125, 1, 0, 0, None, 0, None) == 0


def test_fp8_host_entry_refuses_bad_arguments_without_a_device(attn):
    far = 1 << 40
    L = attn._fp8_fns()
    args = [far, 2 * far, 3 * far, 4 * far, 5 * far, 1, 2, 1024, 128, 0, 0.125, 1,
            0, 0]
    assert L.attn_fwd_fp8_host(*args, None, 0, None) == 11          # no workspace
    assert L.attn_fwd_fp8_host(*args, 6 * far, 16, None) == 11      # too small
    assert L.attn_fwd_fp8_host(*args, 6 * far + 8, 1 << 40, None) == 11  # misaligned
    assert L.attn_fwd_fp8_host(*(args[:8] + [64] + args[9:]), 6 * far,
                               1 << 40, None) == 3                  # d != 128
    assert L.attn_fwd_fp8_host(None, *args[1:], 6 * far, 1 << 40, None) == 1
    assert L.attn_fwd_fp8_host(None, None, None, None, None, 0, 2, 1024, 128, 0,
                               0.125, 1, 0, 0, None, 0, None) == 0  # empty
    # staging for q, k, v, o, lse plus the FP8 scratch of the largest chunk
    r = lambda x: (x + 255) // 256 * 256
    B, H, N = 1, 32, 16384          # 32 heads of 4 MiB: chunks 6,6,6,6,4,2,1,1
    rows = B * H * N
    assert attn.fp8_host_workspace_bytes(B, H, N, 128) == \
        4 * r(rows * 128 * 2) + r(rows * 4) + attn.fp8_workspace_bytes(1, 6, N, 128)
    B, H, N = 1, 2, 64              # small: one chunk of both heads
    rows = B * H * N
    assert attn.fp8_host_workspace_bytes(B, H, N, 128) == \
        4 * r(rows * 128 * 2) + r(rows * 4) + attn.fp8_workspace_bytes(1, 2, N, 128)
    assert attn.fp8_host_workspace_bytes(1, 1, 16, 64) == 0


def test_fp8_workspace_and_sign_mask(attn):
    B, H, N = 2, 3, 300
    r = lambda x: (x + 255) // 256 * 256
    tiles = -(-N // 128)
    assert attn.fp8_workspace_bytes(B, H, N, 128) == \
        3 * r(B * H * N * 128) + 3 * r(B * H * tiles * 4) + r(B * H * 4)
    assert attn.fp8_workspace_bytes(B, H, N, 64) == 0
    lo, hi = attn.sign_mask([1, -1] + [1] * 62 + [-1] + [1] * 63)
    assert lo == 2 and hi == 1
    with pytest.raises(ValueError):
        attn.sign_mask([1, 0, 1])


def test_decode_entry_refuses_bad_arguments_without_a_device(attn):
    far = 1 << 40
    ws = 6 * far
    base = [far, 2 * far, 3 * far, 4 * far, 5 * far]
    def call(B=1, H=1, Nq=1, Nk=256, d=128, causal=1, scale=0.125, ptrs=None,
             wsp=ws, wsb=1 << 30):
        return attn.attn_decode_raw(*(ptrs or base), B, H, Nq, Nk, d, causal,
                                    scale, wsp, wsb, None)
    assert call(Nq=17) == 2                      # more than 16 queries
    assert call(Nq=5, Nk=4) == 2                 # causal needs Nq <= Nk
    assert call(d=96) == 3
    assert call(scale=0.0) == 5
    assert call(ptrs=[None] + base[1:]) == 1
    assert call(ptrs=[far + 8] + base[1:]) == 4
    assert call(wsp=None) == 11
    assert call(wsb=16) == 11
    assert call(ptrs=base[:3] + [far + 64, base[4]]) == 6   # o overlaps q
    assert call(Nq=0, ptrs=[None] * 5, wsp=None) == 0       # empty: no-op
    assert attn.decode_workspace_bytes(1, 1, 17, 10, 128) == 0
    B, H, Nq, d = 2, 3, 4, 64
    r = lambda x: (x + 255) // 256 * 256
    slots = B * H + 1024
    assert attn.decode_workspace_bytes(B, H, Nq, 1000, d) == \
        r(slots * Nq * d * 4) + r(slots * Nq * 4) + r(B * H * 4)
    # a part for every query (the tensor-core kernel serves them in one launch)
    for nq, dd in ((3, 64), (16, 64), (13, 128)):
        assert attn.decode_workspace_bytes(B, H, nq, 1000, dd) == \
            r(slots * nq * dd * 4) + r(slots * nq * 4) + r(B * H * 4)


def test_merge_entries_refuse_bad_arguments_without_a_device(attn):
    far = 1 << 40
    L = attn._merge_fns()
    assert L.attn_merge_fold(far, 2 * far, 3 * far, 4 * far, 10, 96, 1, None) == 3
    assert L.attn_merge_fold(far, 2 * far, 3 * far, 4 * far, -1, 128, 1, None) == 2
    assert L.attn_merge_fold(None, 2 * far, 3 * far, 4 * far, 10, 128, 1, None) == 1
    assert L.attn_merge_fold(far + 4, 2 * far, 3 * far, 4 * far, 10, 128, 1, None) == 4
    assert L.attn_merge_fold(far, 2 * far, far + 64, 4 * far, 10, 128, 1, None) == 6
    assert L.attn_merge_fold(None, None, None, None, 0, 128, 1, None) == 0
    assert L.attn_merge_finish(far, 2 * far, 3 * far, 4 * far, 10, 100, None) == 3
    assert L.attn_merge_finish(far, 2 * far, far + 16, 4 * far, 10, 64, None) == 6


def test_fwd_merge_refuses_bad_modes_without_a_device(attn):
    far = 1 << 40
    f = attn.lib().attn_fwd_merge
    import ctypes
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, ctypes.c_float, i, vp]
    f.restype = i
    args = [far, 2 * far, 3 * far, 4 * far, 5 * far, 6 * far, 7 * far, 1, 1, 64, 64, 0, 0.1]
    assert f(*args, 0, None) == 2              # no such mode
    assert f(*args, 4, None) == 2
    assert f(*(args[:3] + [None] + args[4:]), 2, None) == 1   # accumulator missing
    assert f(*(args[:3] + [4 * far + 8] + args[4:]), 2, None) == 4
    assert f(*(args[:3] + [far + 64] + args[4:]), 2, None) == 6  # acc over q


def test_decode_kernel_choice_without_a_device(attn):
    """The library's decode kernel choice and the test hook that forces one
    (host logic only, no CUDA call): tensor cores by default at both head
    sizes, either kernel when forced, the default back for any other value."""
    try:
        for nq in (1, 4, 16):
            for d in (64, 128):
                assert attn.decode_kernel_for(nq, d) == attn.DECODE_TENSOR_CORES
        attn.set_decode_kernel(attn.DECODE_CUDA_CORES)
        assert attn.decode_kernel_for(3, 64) == attn.DECODE_CUDA_CORES
        attn.set_decode_kernel(attn.DECODE_TENSOR_CORES)
        assert attn.decode_kernel_for(3, 64) == attn.DECODE_TENSOR_CORES
        attn.set_decode_kernel(7)  # not a kernel: the library's choice
        assert attn.decode_kernel_for(3, 64) == attn.DECODE_TENSOR_CORES
    finally:
        attn.set_decode_kernel(attn.DECODE_AUTO)


def test_block_sparse_refuses_bad_arguments_without_a_device(attn):
    """attn_fwd_block_sparse checks its arguments (those of attn_fwd, plus the
    mask pointer and the mask's overlap with the outputs) before any CUDA
    call; fake pointers are never dereferenced."""
    far = 1 << 40
    f = attn._sparse_fn()
    ok = dict(q=far, k=2 * far, v=3 * far, o=4 * far, lse=5 * far, B=1, H=2,
              N=300, d=64, causal=0, scale=0.125, mask=6 * far, per_head=0)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"],
                 a["d"], a["causal"], a["scale"], a["mask"], a["per_head"], None)

    assert call(mask=None) == 1                 # ATTN_ERR_NULL_POINTER
    assert call(N=-1) == 2                      # ATTN_ERR_INVALID_SIZE
    assert call(d=96) == 3                      # head size
    assert call(q=far + 8) == 4                 # misaligned
    assert call(scale=0.0) == 5
    assert call(o=far) == 6                     # o over q
    assert call(mask=4 * far + 64) == 6         # mask inside o
    assert call(mask=None, B=0) == 0            # empty problem: nothing to do
