"""GPU parity of the split-KV decode (attn_decode) against the decode oracle.

Source: the briefgpt.xyz summary page of FlashAttention-2 (arXiv
2307.08691), entry "LeanAttention".  The kernel computes exact attention with
fp32 scores and probabilities (no bf16 rounding of P); its outputs differ
from the fp64 oracle on the same bf16 inputs by the bf16 rounding of O
(2^-9 relative, taken as 2^-8) plus fp32 accumulation over up to Nk keys and
ex2.approx (bounded here by 2e-3 absolute, far above what is observed); lse
within 5e-3, the forward's bound.  With 5..16 queries at d = 128 the kernel
is the tensor-core one, which rounds P to bf16 for the P.V product as the
forward does while the row sum adds the unrounded p: each weight then moves
by at most 2^-9 of itself, so O moves by at most 2^-9 max|v| more, which is
added to the absolute bound (lse is unaffected).  Every shape runs with the default split (two CTAs
per SM over all key tiles) and with the CTA count forced low and high, so
that heads split over many CTAs (merged in-kernel) and heads inside one CTA
(written directly) are both exercised.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import attn
from exact_io_aware_73_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_RTOL, O_ATOL, LSE_ATOL = 2.0 ** -8, 2e-3, 5e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()
    yield
    attn.set_decode_max_ctas(0)
    attn.set_decode_kernel(attn.DECODE_AUTO)
    assert attn.status() == 0


def _ref(oracle_mod, w, q, k, v):
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k, v)]
    return oracle_mod.attention_decode(*f, w.causal, w.scale)


def _o_atol(Nq, d, v):
    """O_ATOL, plus the bf16 rounding of P where the tensor-core kernel runs."""
    if attn.decode_kernel_for(Nq, d) != attn.DECODE_TENSOR_CORES:
        return O_ATOL
    return O_ATOL + 2.0 ** -9 * float(v.float().abs().max())


KERNELS = (attn.DECODE_CUDA_CORES, attn.DECODE_TENSOR_CORES)


def _check(got, ref, what, atol=O_ATOL):
    o, lse = (t.float().cpu().numpy() for t in got)
    O_ref, l_ref = ref
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), what
    err = np.abs(o - O_ref)
    assert np.all(err <= O_RTOL * np.abs(O_ref) + atol), \
        f"{what}: O error {err.max():.3e}"
    lerr = np.abs(lse - l_ref).max()
    assert lerr <= LSE_ATOL, f"{what}: lse error {lerr:.3e}"
    return float(err.max()), float(lerr)


SHAPES = [(1, 1, 1, 1, 64), (1, 2, 1, 64, 128), (2, 1, 3, 65, 128),
          (1, 2, 4, 300, 64), (2, 3, 16, 1000, 128), (1, 1, 16, 16, 128),
          (3, 2, 7, 4097, 64), (1, 4, 1, 20000, 128),
          # 5..16 queries: ragged and exact key tiles, one key tile and many
          (1, 1, 5, 5, 128), (1, 3, 5, 129, 128), (2, 2, 8, 4096, 128),
          (1, 2, 13, 20000, 128), (3, 1, 12, 128, 128), (1, 1, 16, 300, 128),
          (2, 2, 16, 3000, 64), (1, 1, 9, 127, 64)]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Nq,Nk,d", SHAPES)
def test_decode_parity(oracle_mod, B, H, Nq, Nk, d, causal, kernel):
    """Each shape on both kernels (forced), each with the default split, 3
    CTAs and 1000 CTAs."""
    w = W.decode_case(B, H, Nq, Nk, d, causal, seed=500 + Nk + Nq + d)
    q, k, v = W.make_decode_qkv(w)
    ref = _ref(oracle_mod, w, q, k, v)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    attn.set_decode_kernel(kernel)
    try:
        for ctas in (0, 3, 1000):
            attn.set_decode_max_ctas(ctas)
            out = attn.attn_decode(qd, kd, vd, causal=causal, scale=w.scale)
            assert attn.status() == 0
            e = _check(out, ref, f"{w.name} kernel={kernel} ctas={ctas}",
                       _o_atol(Nq, d, v))
    finally:
        attn.set_decode_max_ctas(0)
        attn.set_decode_kernel(attn.DECODE_AUTO)
    print(w.name, kernel, "max|dO| %.2e max|dlse| %.2e" % e)


def test_decode_repeated_calls_are_bitwise_equal():
    """The per-head counters are zeroed by every call and the merge order
    is fixed, so two calls give identical bits."""
    w = W.decode_case(2, 4, 3, 5000, 128, True, seed=77)
    q, k, v = (t.cuda() for t in W.make_decode_qkv(w))
    ws = torch.empty(attn.decode_workspace_bytes(2, 4, 3, 5000, 128),
                     dtype=torch.uint8, device="cuda")
    a = attn.attn_decode(q, k, v, causal=True, workspace=ws)
    b = attn.attn_decode(q, k, v, causal=True, workspace=ws)
    assert attn.status() == 0
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_decode_zero_queries_give_prefix_means(oracle_mod):
    """Q = 0: every visible key has weight 1, so O is the mean of the visible
    values and lse = ln(visible keys) -- the mask's alignment, checked on
    the GPU."""
    B, H, Nq, Nk, d = 1, 2, 5, 3000, 64
    k = torch.randn(B, H, Nk, d).to(torch.bfloat16)
    v = torch.randn(B, H, Nk, d).to(torch.bfloat16)
    q = torch.zeros(B, H, Nq, d, dtype=torch.bfloat16)
    o, lse = attn.attn_decode(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert attn.status() == 0
    vf = v.double().numpy()
    for i in range(Nq):
        n = Nk - Nq + i + 1
        np.testing.assert_allclose(o.float().cpu().numpy()[:, :, i],
                                   vf[:, :, :n].mean(axis=2), rtol=2 ** -8, atol=1e-4)
        np.testing.assert_allclose(lse.cpu().numpy()[:, :, i], np.log(n), atol=1e-4)


@pytest.mark.parametrize("name", sorted(W.DECODE_WORKLOADS))
def test_decode_full_workloads_every_row(oracle_mod, name):
    """The decode configurations at full size, every query row against the
    oracle (Nq is small, so every row is affordable)."""
    w = W.DECODE_WORKLOADS[name]
    q, k, v = W.make_decode_qkv(w)
    o, lse = attn.attn_decode(q.cuda(), k.cuda(), v.cuda(), causal=w.causal,
                              scale=w.scale)
    assert attn.status() == 0
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    rows = np.arange(w.B * w.H * w.Nq)
    O_ref, l_ref = oracle_mod.attention_decode_rows_bf16(*bits, w.causal, w.scale, rows)
    e = _check((o.reshape(-1, w.d), lse.reshape(-1)), (O_ref, l_ref), name,
               _o_atol(w.Nq, w.d, v))
    print(name, "max|dO| %.2e max|dlse| %.2e" % e)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("nq,d", [(4, 128), (16, 128), (16, 64)])
def test_decode_rising_scores_move_the_reference_max(oracle_mod, nq, d, kernel):
    """Scores that grow along the keys (and differ per query) make the lazy
    reference maximum move many times inside every head part, and the parts
    of a head split over many CTAs start from different maxima: the O
    rescales and the merge are exercised, on both kernels."""
    B, H, Nk = 1, 2, 3000
    g = torch.Generator().manual_seed(91)
    q = (torch.randn(B, H, nq, d, generator=g) * 0.1).to(torch.bfloat16)
    q[..., 0] = torch.linspace(2.0, 6.0, nq).to(torch.bfloat16)
    k = (torch.randn(B, H, Nk, d, generator=g) * 0.1)
    k[..., 0] = torch.linspace(0.0, 48.0, Nk)
    k = k.to(torch.bfloat16)
    v = torch.randn(B, H, Nk, d, generator=g).to(torch.bfloat16)
    scale = 1.0 / np.sqrt(d)
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k, v)]
    ref = oracle_mod.attention_decode(*f, True, scale)
    attn.set_decode_kernel(kernel)
    try:
        for ctas in (0, 7, 1000):
            attn.set_decode_max_ctas(ctas)
            out = attn.attn_decode(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=scale)
            assert attn.status() == 0
            _check(out, ref, f"nq={nq} d={d} kernel={kernel} ctas={ctas}", _o_atol(nq, d, v))
    finally:
        attn.set_decode_max_ctas(0)
        attn.set_decode_kernel(attn.DECODE_AUTO)


def test_decode_argument_errors_on_device():
    q = torch.zeros(1, 1, 2, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.attn_decode(q, k, k.clone(), causal=True,
                         workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert attn.status() == 0
