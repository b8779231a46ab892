"""GPU parity of the backward pass (attn_bwd) against the fp64 oracle.

The kernel recomputes P from the forward's lse and rounds P and dS to bf16
for its tensor-core GEMMs; dQ, dK, dV are stored in bf16.  Each gradient is
compared element by element with the fp64 oracle's gradient on the same
bf16 inputs (Q, K, V, dO):

    max |g - g_ref| <= BWD_RTOL * max |g_ref| + BWD_ATOL

Reading of the tolerance (the pages and the target give none for the
backward): relative to the gradient's own scale, because gradient
magnitudes vary with N by orders of magnitude; 2^-6 covers bf16 rounding of
P and dS (2^-9 each, summed over up to N terms with random signs) plus the
bf16 output rounding (2^-9).
"""
import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import attn
from exact_io_aware_73_b200 import workloads as W

BWD_RTOL = 2.0 ** -6
BWD_ATOL = 1e-4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()
    yield
    assert attn.status() == 0


def _grad_case(B, H, N, d, causal, seed):
    w = W.shape_case(B, H, N, d, causal, seed=seed)
    q, k, v = W.make_qkv(w)
    g = torch.Generator().manual_seed(seed + 99)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    return w, q, k, v, do


def _run(w, q, k, v, do):
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = attn.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale)
    dq, dk, dv = attn.attn_bwd(qd, kd, vd, o, lse, dod, causal=w.causal,
                               scale=w.scale)
    rc = attn.status()
    assert rc == 0, attn.strerror(rc)
    return [t.float().cpu().numpy() for t in (dq, dk, dv)]


def _ref(oracle_mod, w, q, k, v, do):
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k, v, do)]
    return oracle_mod.attention_backward(*f, w.causal, w.scale)


def _compare(got, ref, what):
    errs = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.all(np.isfinite(g)), f"{what} {name} not finite"
        scale = float(np.abs(r).max())
        err = float(np.abs(g - r).max())
        errs[name] = (err, scale)
        assert err <= BWD_RTOL * scale + BWD_ATOL, \
            f"{what} {name}: max err {err:.3e} vs max|ref| {scale:.3e}"
    print(what, {k: f"{e:.2e}/{s:.2e}" for k, (e, s) in errs.items()})


SHAPES = [(1, 1, 1, 64), (1, 2, 128, 64), (2, 1, 129, 128), (1, 2, 255, 64),
          (1, 1, 300, 128), (2, 2, 1000, 64), (1, 2, 1000, 128),
          (3, 2, 200, 128), (1, 1, 2048, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", SHAPES)
def test_backward_parity_shapes(oracle_mod, B, H, N, d, causal):
    w, q, k, v, do = _grad_case(B, H, N, d, causal, seed=300 + N + d + B + H)
    got = _run(w, q, k, v, do)
    ref = _ref(oracle_mod, w, q, k, v, do)
    _compare(got, ref, w.name)


def test_backward_invariants_on_gpu():
    """Sum over keys of dK vanishes and sum over keys of dV equals the sum
    over queries of dO (properties of the exact gradients), up to rounding."""
    w, q, k, v, do = _grad_case(1, 4, 1024, 128, False, seed=77)
    dq, dk, dv = _run(w, q, k, v, do)
    dk_sum = np.abs(dk.astype(np.float64).sum(axis=2)).max()
    assert dk_sum <= 0.05 * np.abs(dk).max() * np.sqrt(1024)
    np.testing.assert_allclose(dv.astype(np.float64).sum(axis=2),
                               do.double().numpy().sum(axis=2),
                               atol=0.05 * np.abs(do.float().numpy()).max() * 8)


def test_backward_is_deterministic():
    w, q, k, v, do = _grad_case(2, 2, 777, 64, True, seed=78)
    a = _run(w, q, k, v, do)
    b = _run(w, q, k, v, do)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_argument_errors():
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 64, dtype=torch.float32, device="cuda")
    outs = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty(attn.bwd_workspace_bytes(1, 1, 64), dtype=torch.uint8,
                     device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    args = [q.data_ptr()] * 5 + [lse.data_ptr()] + [o.data_ptr() for o in outs]
    # workspace too small
    assert attn.attn_bwd_raw(*args, ws.data_ptr(), 16, 1, 1, 64, 64, 0, 0.125,
                             s) == 11
    # an output overlapping an input
    bad = args[:6] + [q.data_ptr()] + args[7:]
    assert attn.attn_bwd_raw(*bad, ws.data_ptr(), ws.numel(), 1, 1, 64, 64, 0,
                             0.125, s) == 6
    assert attn.attn_bwd_raw(*args, ws.data_ptr(), ws.numel(), 1, 1, 64, 96, 0,
                             0.125, s) == 3
    assert attn.status() == 0


@pytest.mark.parametrize("name", ["long_b1h32n16384d128", "b2h16n4096d128_causal"])
def test_backward_full_size_sampled_rows(oracle_mod, name):
    """The full-size configurations through the GPU forward and backward;
    dQ of sampled query rows and dK, dV of sampled key rows of the first and
    last head against the oracle (same tolerance as the shape sweep)."""
    w = W.WORKLOADS[name]
    q, k, v = W.make_qkv(w)
    g = torch.Generator().manual_seed(w.seed + 99)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv = _run(w, q, k, v, do)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N - 1], rng.integers(0, w.N, 11)]))
    BH = w.B * w.H
    for bh in (0, BH - 1):
        b, h = divmod(bh, w.H)
        bits = [oracle_mod.bf16_bits(t[b, h].contiguous()) for t in (q, k, v, do)]
        rq, rk, rv = oracle_mod.attention_backward_rows_bf16(*bits, w.causal, w.scale,
                                                             rows, rows)
        got = [dq[b, h][rows], dk[b, h][rows], dv[b, h][rows]]
        _compare(got, [rq, rk, rv], f"{name} head {bh}")
