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


def test_decode_wait_timeout_is_reported_and_the_context_survives():
    """Decode: CTA 0's producer skips its first K/V tile; its compute warps'
    bounded wait runs out, they agree to leave without writing, the producer
    drains what it did copy.  The status reports the timeout, no drain ran
    out, and the next launch is correct."""
    w = W.decode_case(1, 8, 2, 20000, 128, True, seed=32)
    q, k, v = (t.cuda() for t in W.make_decode_qkv(w))
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
    assert bits & 1 and bits & ((1 << 8) | (1 << 10))
    assert not bits & (1 << 12)
    o, lse = attn.attn_decode(q, k, v, causal=True)
    assert attn.status() == 0
    assert torch.equal(o, good) and torch.equal(lse, good_lse)
