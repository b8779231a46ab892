"""Failure detection on the GPU without a GPU fault.

The host asks the library to make the first CTA's loader skip its first Q
copy.  The MMA warp's wait for that copy can then never complete; with a
50 ms wait limit it must give up, flag the device status word, let the other
warps leave their loops, drain the copies that were issued, free its tensor
memory and exit.  The host reads ATTN_ERR_DEVICE_TIMEOUT from attn_status,
and the same CUDA context must then run a normal launch correctly.
Nothing traps, asserts or faults.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import attn
from exact_io_aware_73_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()
    assert attn.status() == 0


@pytest.mark.parametrize("d,causal", [(128, False), (64, True)])
def test_wait_timeout_is_reported_and_the_context_survives(d, causal):
    w = W.shape_case(1, 4, 1024, d, causal, seed=31)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    attn.set_wait_timeout_ns(50_000_000)
    attn.set_fault_injection(1)
    try:
        attn.attn_fwd(q, k, v, causal=causal)
        rc = attn.status()
    finally:
        attn.set_fault_injection(0)
        attn.set_wait_timeout_ns(0)
    assert rc == 16, attn.strerror(rc)
    bits = attn.last_status_bits()
    assert bits & 1                 # a wait ran out ...
    # ... in the MMA warp (its Q never came) or in a warp waiting on it
    # (whichever waiter looks at its clock first reports the timeout)
    assert bits & ((1 << 8) | (1 << 9) | (1 << 10) | (1 << 11))
    assert not bits & (1 << 12)     # every issued copy drained in time

    # the context is intact: a normal launch is correct
    o, lse = attn.attn_fwd(q, k, v, causal=causal)
    assert attn.status() == 0
    o2, lse2 = attn.attn_fwd(q, k, v, causal=causal)
    assert attn.status() == 0
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.isfinite(o.float()).all()
    # row 0 of each head: causal -> exactly V[0]; else a convex mix of V
    if causal:
        np.testing.assert_allclose(o[:, :, 0].float().cpu().numpy(),
                                   v[:, :, 0].float().cpu().numpy(), atol=2e-2)
    assert (o.float().abs().amax() <= v.float().abs().amax() * 1.01).item()


@pytest.mark.parametrize("kernel", [1, 2])
def test_decode_wait_timeout_is_reported_and_the_context_survives(kernel):
    """Decode: CTA 0's loader skips its first K/V tile.  On the CUDA-core
    kernel (1) its compute warps' bounded wait runs out; on the tensor-core
    kernel (2) the MMA thread's and the softmax warps' waits do.  The CTA
    leaves without writing and the loader drains what it did copy.  The
    status reports the timeout, no drain ran out, and the next launch is
    correct."""
    w = W.decode_case(1, 8, 6, 20000, 128, True, seed=32)
    q, k, v = (t.cuda() for t in W.make_decode_qkv(w))
    attn.set_decode_kernel(kernel)
    try:
        good, good_lse = attn.attn_decode(q, k, v, causal=True)
        assert attn.status() == 0
        attn.set_wait_timeout_ns(50_000_000)
        attn.set_fault_injection(2)
        try:
            attn.attn_decode(q, k, v, causal=True)
            rc = attn.status()
        finally:
            attn.set_fault_injection(0)
            attn.set_wait_timeout_ns(0)
        assert rc == 16, attn.strerror(rc)
        bits = attn.last_status_bits()
        assert bits & 1 and bits & ((1 << 8) | (1 << 9) | (1 << 10))
        assert not bits & (1 << 12)
        o, lse = attn.attn_decode(q, k, v, causal=True)
        assert attn.status() == 0
        assert torch.equal(o, good) and torch.equal(lse, good_lse)
    finally:
        attn.set_decode_kernel(0)


def _debug_lib():
    """The debug build of the library (kernels' index checks compiled in),
    loaded beside the release one; each keeps its own device state."""
    import ctypes
    import os
    if not os.path.exists(attn.DEBUG_LIB_PATH):
        pytest.fail(f"{attn.DEBUG_LIB_PATH} is missing: build it with "
                    "`python -m exact_io_aware_73_b200.build --debug`")
    L = ctypes.CDLL(attn.DEBUG_LIB_PATH)
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, ctypes.c_float, vp]
    L.attn_fwd.restype = i
    L.attn_status.argtypes = [vp]
    L.attn_status.restype = i
    L.attn_last_status_bits.restype = ctypes.c_uint32
    L.attn_set_fault_injection.argtypes = [ctypes.c_uint32]
    L.attn_set_fault_injection.restype = None
    return L


@pytest.mark.parametrize("d,causal,N", [(128, False, 1000), (64, True, 777)])
def test_debug_build_checks_indices_without_faulting(d, causal, N):
    """The debug build computes exactly what the release build does (its
    checks only read indices), and an index error injected into it (the first
    row CTA 0 stores points past the output) is caught before the store:
    attn_status reports ATTN_ERR_DEVICE_BOUNDS, nothing faults, the wrong
    address is never written, and the next launch is correct."""
    L = _debug_lib()
    w = W.shape_case(2, 3, N, d, causal, seed=57)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    o_rel, l_rel = attn.attn_fwd(q, k, v, causal=causal, scale=w.scale)
    assert attn.status() == 0
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream

    def run():
        return L.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                          lse.data_ptr(), w.B, w.H, w.N, w.d, int(causal), w.scale, s)

    assert run() == 0 and L.attn_status(s) == 0
    assert torch.equal(o, o_rel) and torch.equal(lse, l_rel)
    # a guard region after the output: the skipped store must not land there
    big = torch.zeros(2 * q.numel(), dtype=torch.bfloat16, device="cuda")
    o = big[: q.numel()].view_as(q)
    L.attn_set_fault_injection(4)
    try:
        assert run() == 0
        rc = L.attn_status(s)
    finally:
        L.attn_set_fault_injection(0)
    assert rc == 17, attn.strerror(rc)
    assert L.attn_last_status_bits() & 2
    assert torch.count_nonzero(big[q.numel():]) == 0
    # the context is intact and the debug build is exact again
    o = torch.empty_like(q)
    assert run() == 0 and L.attn_status(s) == 0
    assert torch.equal(o, o_rel) and torch.equal(lse, l_rel)
    # the release build ignores the injection bit
    attn.set_fault_injection(4)
    try:
        o2, l2 = attn.attn_fwd(q, k, v, causal=causal, scale=w.scale)
        rc = attn.status()
    finally:
        attn.set_fault_injection(0)
    assert rc == 0 and torch.equal(o2, o_rel) and torch.equal(l2, l_rel)
