"""attn_fwd_host_noalloc: the host-buffer entry point that allocates nothing.

It exists for callers that cannot allocate device memory themselves (host
programs without a device allocator, or processes whose device memory is
owned by an allocator that must not see untracked cudaMalloc calls).  Its
scratch is a static device array inside the library, so two calls in a row
reuse the same memory: the second call must not see anything of the first.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_73_b200 import attn
from exact_io_aware_73_b200 import workloads as W

O_TOL = 2e-2    # the parity tolerances used throughout the GPU tests
LSE_TOL = 5e-3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()


def _pinned_case(B, H, N, d, causal, seed):
    w = W.shape_case(B, H, N, d, causal, seed=seed)
    q, k, v = (t.pin_memory() for t in W.make_qkv(w))
    return w, q, k, v


def _with_existing_entry(w, q, k, v):
    """Reference: the existing host-buffer entry point with a torch-allocated
    workspace."""
    o = torch.empty_like(q).pin_memory()
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.host_workspace_bytes(w.B, w.H, w.N, w.d),
                     dtype=torch.uint8, device="cuda")
    attn.attn_fwd_host(q, k, v, o, lse, w.causal, w.scale, ws)
    torch.cuda.synchronize()
    assert attn.status() == 0
    return o, lse


def _with_noalloc_entry(w, q, k, v):
    o = torch.full_like(q, float("nan")).pin_memory()
    lse = torch.full((w.B, w.H, w.N), float("nan"),
                     dtype=torch.float32).pin_memory()
    attn.attn_fwd_host_noalloc(q, k, v, o, lse, w.causal, w.scale)
    return o, lse


def test_noalloc_matches_existing_entry_on_two_calls_in_a_row():
    # Both entries run the same kernel on the same bits, so the outputs must
    # agree bit for bit; the second call reuses the scratch the first left.
    cases = [_pinned_case(2, 3, 777, 128, True, seed=21),
             _pinned_case(1, 4, 1000, 64, False, seed=22)]
    refs = [_with_existing_entry(*c) for c in cases]
    for (w, q, k, v), (o_ref, l_ref) in zip(cases, refs):
        o, lse = _with_noalloc_entry(w, q, k, v)
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert torch.equal(o, o_ref), w.name
        assert torch.equal(lse, l_ref), w.name
        # and within the parity tolerances of the fp64 oracle
        O, L = oracle.attention(q.float().numpy(), k.float().numpy(),
                                v.float().numpy(), w.causal, w.scale)
        assert np.max(np.abs(o.float().numpy() - O)) <= O_TOL, w.name
        assert np.max(np.abs(lse.numpy() - L)) <= LSE_TOL, w.name


def test_noalloc_second_call_takes_no_device_memory():
    # The first call on a device may load the library's module (which holds
    # the static scratch array); from then on nothing is allocated.
    w, q, k, v = _pinned_case(1, 2, 640, 128, False, seed=23)
    o = torch.empty_like(q).pin_memory()
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    attn.attn_fwd_host_noalloc(q, k, v, o, lse, w.causal, w.scale)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        attn.attn_fwd_host_noalloc(q, k, v, o, lse, w.causal, w.scale)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after >= free_before, (free_before, free_after)


def test_noalloc_timeout_is_reported_and_the_next_call_is_exact():
    # A wait that nothing will satisfy (the first CTA's loader skips its
    # first Q copy) must run out within the limit and come back as
    # ATTN_ERR_DEVICE_TIMEOUT from the call itself; the status word lives in
    # the shared array, so the next call must start from a clean word.
    w, q, k, v = _pinned_case(1, 4, 1024, 128, False, seed=24)
    o = torch.empty_like(q).pin_memory()
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    attn.set_wait_timeout_ns(50_000_000)
    attn.set_fault_injection(1)
    try:
        with pytest.raises(attn.AttnError) as e:
            attn.attn_fwd_host_noalloc(q, k, v, o, lse, w.causal, w.scale)
    finally:
        attn.set_fault_injection(0)
        attn.set_wait_timeout_ns(0)
    assert e.value.code == 16, attn.strerror(e.value.code)
    assert attn.last_status_bits() & 1
    o, lse = _with_noalloc_entry(w, q, k, v)
    O, L = oracle.attention(q.float().numpy(), k.float().numpy(),
                            v.float().numpy(), w.causal, w.scale)
    assert np.max(np.abs(o.float().numpy() - O)) <= O_TOL
    assert np.max(np.abs(lse.numpy() - L)) <= LSE_TOL


def test_noalloc_refuses_problems_beyond_its_scratch():
    # d = 128: 4 * (rows * 256 B) + rows * 4 B > 32 MiB for 40,000 rows
    B, H, N, d = 1, 1, 40000, 128
    assert attn.host_workspace_bytes(B, H, N, d) > attn.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    lse = torch.zeros(B, H, N, dtype=torch.float32)
    o = torch.zeros_like(q)
    with pytest.raises(attn.AttnError) as e:
        attn.attn_fwd_host_noalloc(q, q.clone(), q.clone(), o, lse, False,
                                   0.088)
    assert e.value.code == 12
