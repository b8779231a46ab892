"""FP8 path against EXACT attention on the dequantized operands.

[MM] = marketmaker.cc post "Apakah Konteks Sehari Penuh Mengalahkan Konteks
Sepuluh Menit? ...", section "FA3: Mekanika hopper", item 3: rotate Q and K
at random, quantize in blocks, attend in FP8.

The reference here shares nothing with the kernel's design.  The operands
are the method's own quantized tensors, Q^ = E4M3(Q R) x 2^-e per block,
likewise K^, and V^ = E4M3(V) x 2^-e per head (oracle.quantize_qkv_fp8,
pinned bit for bit to the library conversion and the Hadamard matrix; the
kernel's codes equal them bit for bit in test_fp8_gpu.py).  On those
operands the plain fp64 two-pass oracle (oracle.attention) gives exact
attention.  What is left between the two is the FP8 representation of the
probabilities P, plus fp32 and output rounding; the tolerance below follows
from the E4M3 format alone, with nothing taken from the kernel's key-block
size or from how it scales P before encoding it.

Per output element (row i, column t), with p_j the exact probabilities of
row i (normalised so that the row maximum is 1) and l = sum_j p_j:

  * E4M3 keeps 3 mantissa bits: any value in its normal range is stored
    with relative error <= 2^-4.  The kernel carries a row's probabilities
    on a base that lags the row's running maximum by at most tau = 4 (log2
    units) and keeps the largest below 2^8 (the format's top binade holds up
    to 448), so its largest probability lies between 2^(8 - tau) and 2^8,
    and the normal range (down to 2^-6) reaches at least 2^-(14 - tau) =
    2^-10 below it.  This is the error contract of the threshold: every
    p_j >= 2^-(14 - tau) is carried within 2^-4 p_j, and a smaller one is
    off by at most p_j (subnormal or flushed to zero):
        |O - O*| <= 2^-4 A + U,
        A = sum_j p_j |v_jt| / l           (exact attention on |V^|)
        U = sum_{p_j < 2^-(14 - tau)} p_j |v_jt| / l.
  * The scores come from fp32 sums of exact E4M3 products; with the fp32
    multiplier, the FMA and ex2.approx that gives a relative error delta in
    every p before it is encoded (delta as in test_fp8_gpu.py): 2 delta A
    for the numerator and 2 delta |O*| for the row sum.
  * bf16 output rounding, 2^-8 |O*| (twice the half ulp), and fp32
    accumulation of P.V, (keys / 32 + 16) x 2^-24 x max|V^|.

lse does not depend on P's encoding (the row sum adds the unrounded p), so
it keeps the tight bound |lse - lse*| <= 1e-4 (1 + |lse*|).
"""
import math

import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import attn
from exact_io_aware_73_b200 import workloads as W

pytestmark = pytest.mark.gpu

D = 128
LOG2E = 1.4426950408889634
E4M3_REL = 2.0 ** -4          # half the relative step of 3 mantissa bits
TAU = 4.0                     # the kernel's base threshold (log2 units)
E4M3_RANGE = 2.0 ** -(14 - TAU)  # normal range below the row maximum


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()
    yield
    assert attn.status() == 0


def _case(B, H, N, causal, seed, outliers=False):
    w = W.shape_case(B, H, N, D, causal, seed=seed)
    q, k, v = W.make_qkv(w)
    if outliers:
        ch = W.outlier_channels(seed + 1, D, 2)
        q, k = (W.add_channel_outliers(t, ch, 8.0) for t in (q, k))
    signs = W.make_signs(seed + 2, D)
    return w, q, k, v, signs


def _dequantized(oracle_mod, z):
    """Q^, K^, V^ as fp64 [BH, N, d]: codes times their block scales."""
    N = z["q8"].shape[-2]
    BH = z["q8"].size // (N * D)
    per_row = lambda s: np.repeat(s.reshape(BH, -1), 128, axis=1)[:, :N, None]
    qh = oracle_mod.e4m3_decode(z["q8"]).reshape(BH, N, D) * per_row(z["qs"])
    kh = oracle_mod.e4m3_decode(z["k8"]).reshape(BH, N, D) * per_row(z["ks"])
    vh = oracle_mod.e4m3_decode(z["v8"]).reshape(BH, N, D) * z["vs"].reshape(BH, 1, 1)
    return qh, kh, vh


def _score_delta(qh, kh, rows, c):
    """Relative error bound of the kernel's p before encoding (fp32 scores of
    exact products, fp32 multiplier and FMA, ex2.approx)."""
    A = np.abs(qh[rows]) @ np.abs(kh).T
    S = qh[rows] @ kh.T
    return math.log(2.0) * (2 * 2.0 ** -20 * A.max() * c +
                            2.0 ** -22 * 2 * np.abs(S).max() * c) + 2.0 ** -21


def _low_mass(qh, kh, vh_abs, rows, causal, scale_qk):
    """U: the exact probability mass (weighted by |V^|) of keys more than
    E4M3's normal range below their row's maximum."""
    N = kh.shape[0]
    S = scale_qk * (qh[rows] @ kh.T)
    if causal:
        S = np.where(np.arange(N)[None, :] > np.asarray(rows)[:, None], -np.inf, S)
    P = np.exp(S - S.max(axis=1, keepdims=True))
    low = np.where(P < E4M3_RANGE, P, 0.0)
    return (low @ vh_abs) / P.sum(axis=1, keepdims=True)


def _check(got_o, got_lse, O_ex, L_ex, A, U, delta, vmax, nkeys, what):
    assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_lse)), what
    tol = ((E4M3_REL + 2 * delta) * A + U + (2 * delta + 2.0 ** -8) * np.abs(O_ex)
           + (nkeys / 32 + 16) * 2.0 ** -24 * vmax)
    err = np.abs(got_o - O_ex)
    bad = err > tol
    assert not bad.any(), (
        f"{what}: {bad.sum()} outputs beyond the E4M3 bound, worst excess "
        f"{(err - tol).max():.3e} (max err {err.max():.3e})")
    lerr = np.abs(got_lse - L_ex)
    assert np.all(lerr <= 1e-4 * (1 + np.abs(L_ex))), f"{what}: lse {lerr.max():.3e}"
    return float(err.max()), float((err / np.maximum(tol, 1e-30)).max())


SHAPES = [(1, 1, 1), (1, 2, 128), (2, 1, 129), (1, 2, 300), (1, 1, 1000),
          (2, 2, 517), (1, 1, 2048)]


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N", SHAPES)
def test_fp8_output_within_e4m3_bound_of_exact_attention(oracle_mod, B, H, N,
                                                         causal, rotate):
    w, q, k, v, signs = _case(B, H, N, causal, seed=160 + N + B + H,
                              outliers=(N % 2 == 0))
    scale32 = float(np.float32(w.scale))
    z = oracle_mod.quantize_qkv_fp8(*[oracle_mod.bf16_bits(t) for t in (q, k, v)],
                                    rotate, signs.numpy())
    scale_qk = scale32 * z["gain"]
    qh, kh, vh = _dequantized(oracle_mod, z)
    BH = B * H
    O_ex, L_ex = oracle_mod.attention(qh[None], kh[None], vh[None], causal, scale_qk)
    A, _ = oracle_mod.attention(qh[None], kh[None], np.abs(vh)[None], causal, scale_qk)
    O_ex, L_ex, A = O_ex[0], L_ex[0], A[0]
    rows = np.arange(N)
    U = np.stack([_low_mass(qh[h], kh[h], np.abs(vh[h]), rows, causal, scale_qk)
                  for h in range(BH)])
    delta = max(_score_delta(qh[h], kh[h], rows, scale_qk * LOG2E) for h in range(BH))
    vmax = float(np.abs(vh).max())
    o, lse = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                               scale=scale32, signs=signs.tolist() if rotate else None)
    assert attn.status() == 0
    err, used = _check(o.float().cpu().numpy().reshape(BH, N, D),
                       lse.cpu().numpy().reshape(BH, N), O_ex, L_ex, A, U, delta,
                       vmax, N, f"{w.name} rotate={rotate}")
    print(f"{w.name} rotate={rotate}: max err {err:.3e}, {used:.2f} of the bound")


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_full_size_sampled_rows_within_e4m3_bound(oracle_mod, causal):
    """B=1, H=32, N=16384, d=128 through the whole FP8 path; sampled rows of
    the first and last head against exact attention on Q^, K^, V^.  The
    dequantized operands are exactly representable in bf16 (3 mantissa bits
    times a power of two), so the row oracle takes them as bf16 patterns."""
    w = W.WORKLOADS["long_b1h32n16384d128"].with_(causal=causal)
    q, k, v = W.make_qkv(w)
    signs = W.make_signs(w.seed + 3, D)
    scale32 = float(np.float32(w.scale))
    o, lse = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                               scale=scale32, signs=signs.tolist())
    assert attn.status() == 0
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    rng = np.random.default_rng(7)

    def to_bits(x):
        f = np.ascontiguousarray(x, dtype=np.float32)
        assert np.array_equal(f.astype(np.float64), x)
        u = f.view(np.uint32)
        assert not np.any(u & 0xFFFF), "not exactly representable in bf16"
        return (u >> 16).astype(np.uint16)

    for h in (0, w.H - 1):
        sel = lambda t: t[:, h:h + 1].contiguous()
        z = oracle_mod.quantize_qkv_fp8(*[oracle_mod.bf16_bits(sel(t)) for t in (q, k, v)],
                                        True, signs.numpy())
        scale_qk = scale32 * z["gain"]
        qh, kh, vh = (x[0] for x in _dequantized(oracle_mod, z))
        rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N - 1],
                                         rng.integers(0, w.N, 60)]))
        bq, bk, bv, bva = (to_bits(x)[None, None] for x in (qh, kh, vh, np.abs(vh)))
        O_ex, L_ex = oracle_mod.attention_rows_bf16(bq, bk, bv, causal, scale_qk, rows)
        A, _ = oracle_mod.attention_rows_bf16(bq, bk, bva, causal, scale_qk, rows)
        U = _low_mass(qh, kh, np.abs(vh), rows, causal, scale_qk)
        delta = _score_delta(qh, kh, rows, scale_qk * LOG2E)
        err, used = _check(o[0, h, rows], lse[0, h, rows], O_ex, L_ex, A, U, delta,
                           float(np.abs(vh).max()), w.N,
                           f"{w.name} causal={causal} head {h}")
        print(f"head {h} causal={causal}: max err {err:.3e}, {used:.2f} of the bound")
