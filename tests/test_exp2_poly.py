"""The kernel's FMA-pipe exp2: constants pinned to their fitting script (CPU)
and values checked against exact 2^x and CUDA's exp2f (GPU)."""
import math
import os
import re
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_73_b200", "csrc")


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "attn_fwd_kernel.cuh")).read()
    body = src[src.index("exp2_poly_x2"):src.index("struct FwdParams")]
    hexes = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    # each coefficient appears twice (both halves of a packed pair)
    uniq = []
    for h in hexes:
        if h not in uniq:
            uniq.append(h)
    return [float.fromhex(h) for h in uniq]  # c3, c2, c1, c0 (Horner order)


def test_kernel_constants_come_from_the_fit():
    sys.path.insert(0, CSRC)
    import gen_exp2_poly as g
    _, c32, err = g.coefficients()
    assert err < 1e-4
    c3, c2, c1, c0 = _kernel_coefficients()
    np.testing.assert_array_equal(np.float32([c0, c1, c2, c3]), c32)


def _poly_exp2_cpu(x):
    """The kernel's evaluation sequence in fp32 (fused steps emulated in fp64)."""
    c3, c2, c1, c0 = (np.float64(np.float32(c)) for c in _kernel_coefficients())
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    n = np.rint(x.astype(np.float64))
    f = (x.astype(np.float64) - n).astype(np.float32).astype(np.float64)
    q = np.float32(c3 * f + c2).astype(np.float64)
    q = np.float32(q * f + c1).astype(np.float64)
    q = np.float32(q * f + c0).astype(np.float64)
    return q * np.exp2(n)


def test_polynomial_relative_error_bound_cpu():
    x = np.linspace(-125, 8, 2_000_001).astype(np.float32)
    rel = np.abs(_poly_exp2_cpu(x) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 8e-5
    # well inside bf16's half ulp (2^-9), the precision P is stored in
    assert rel.max() < 2 ** -9 / 20


@pytest.mark.gpu
def test_polynomial_on_gpu_against_exact_and_cuda_exp2f():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_io_aware_73_b200 import attn
    x = torch.linspace(-125, 8, 1_000_003, dtype=torch.float32)
    special = torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 8.0, -124.5, -125.0,
                            -0.0, 2.5, -2.5], dtype=torch.float32)
    x = torch.cat([x, special])
    xd = x.cuda()
    y_poly = attn.selftest_exp2(xd, 0).cpu().double()
    y_mufu = attn.selftest_exp2(xd, 1).cpu().double()
    y_cuda = torch.exp2(xd).cpu().double()
    exact = torch.exp2(x.double())
    assert (y_poly / exact - 1).abs().max().item() < 8e-5
    assert (y_mufu / exact - 1).abs().max().item() < 1e-6
    assert (y_poly / y_cuda - 1).abs().max().item() < 8e-5
    # bit-faithful to the CPU model of the same sequence
    np.testing.assert_allclose(y_poly.numpy(), _poly_exp2_cpu(x.numpy()),
                               rtol=2e-7, atol=0)
    # below the clamp: tiny, never zero or garbage
    low = torch.tensor([-126.0, -200.0, -1e30, float("-inf")]).cuda()
    y_low = attn.selftest_exp2(low, 0).cpu().double()
    assert torch.all(y_low > 0) and torch.all(y_low <= 2.0 ** -124)
    assert attn.status() == 0
