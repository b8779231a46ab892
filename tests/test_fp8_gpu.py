"""GPU parity of the FP8 path (attn_fp8_quantize, attn_fwd_fp8_quantized,
attn_fwd_fp8) against the FP8 oracle (oracle/fp8_oracle.c).

[MM] = marketmaker.cc post "Apakah Konteks Sehari Penuh Mengalahkan Konteks
Sepuluh Menit? ...", section "FA3: Mekanika hopper", item 3.

Quantization is integer work: codes and scales must be bit-identical to the
oracle's (both sides rotate exactly in fp64, round to fp32, scale by an exact
power of two and round to E4M3).

The attention is floating point.  Tolerance, derived from the arithmetic
(the target states none for this path):
  * the E4M3 codes of P are decisions taken in fp32 from the kernel's
    scores; wherever the oracle's P lies within relative distance delta of an
    E4M3 rounding boundary, the kernel may land on the neighbouring code.
    delta bounds the kernel's relative error in P: the tensor core's fp32
    accumulation of exact E4M3 products (<= 2^-20 of sum |q_t k_t| per dot
    product, for the score and for the running max), the fp32 rounding of
    the multiplier and of the FMA (2^-22 of |x|), and ex2.approx (2^-21).
    The oracle reports per row the most those
    one-step changes can move an output (flip_bound: code spacing x max|V|
    / l summed over such keys);
  * the kernel moves a row's base only when a key block's maximum exceeds
    it by more than tau = 4 (log2 units; the oracle runs the same rule); a
    row where some block's gap lies within the score error of tau could be
    decided the other way in fp32, so the oracle gives it an infinite flip
    bound and the comparison here skips it (test_fp8_exact_gpu.py still
    bounds it against exact attention);
  * bf16 rounding of the stored output: 2^-8 of |O| (twice the half-ulp);
  * fp32 accumulation of P.V and l: (keys / 32 + 16) x 2^-24 x max|V|.
lse is independent of P's rounding: |lse - lse_ref| <= 1e-4 (1 + |lse_ref|).
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
EXP2_REL = 2.0 ** -21   # ex2.approx


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()
    yield
    assert attn.status() == 0


def _case(B, H, N, causal, seed, outliers=False, q_std=1.0):
    w = W.shape_case(B, H, N, D, causal, seed=seed, q_std=q_std, k_std=q_std)
    q, k, v = W.make_qkv(w)
    if outliers:
        ch = W.outlier_channels(seed + 1, D, 2)
        q, k = (W.add_channel_outliers(t, ch, 8.0) for t in (q, k))
    signs = W.make_signs(seed + 2, D)
    return w, q, k, v, signs


def _oracle_quant(oracle_mod, q, k, v, rotate, signs):
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    return oracle_mod.quantize_qkv_fp8(*bits, rotate, signs.numpy())


def _flip_delta(oracle_mod, z, scale_qk, causal):
    """Bound on the kernel's relative error in P before rounding (see the
    module docstring), as one number for the whole case."""
    N = z["q8"].shape[-2]
    qs = np.repeat(z["qs"].reshape(-1, z["qs"].shape[-1]), 128, axis=-1)[:, :N, None]
    ks = np.repeat(z["ks"].reshape(-1, z["ks"].shape[-1]), 128, axis=-1)[:, :N, None]
    qh = oracle_mod.e4m3_decode(z["q8"]).reshape(-1, N, D) * qs
    kh = oracle_mod.e4m3_decode(z["k8"]).reshape(-1, N, D) * ks
    c = scale_qk * LOG2E
    worst = 0.0
    for h in range(qh.shape[0]):
        A = np.abs(qh[h]) @ np.abs(kh[h]).T          # sum_t |q_t k_t|
        S = qh[h] @ kh[h].T
        if causal:
            A = np.tril(A)
            S = np.tril(S)
        worst = max(worst, 2 * 2.0 ** -20 * A.max() * c + 2.0 ** -22 * 2 * np.abs(S).max() * c)
    return math.log(2.0) * worst + EXP2_REL


def _compare(got_o, got_lse, ref_o, ref_lse, flip, vmax, nkeys, what):
    got_o = got_o.reshape(ref_o.shape)
    got_lse = got_lse.reshape(ref_lse.shape)
    # rows whose base decision the oracle cannot predict (infinite flip
    # bound) are left to the exact-attention bound; they must stay rare
    assert np.isinf(flip).mean() <= 0.01, f"{what}: {np.isinf(flip).sum()} undecided rows"
    assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_lse)), what
    tol = (flip.reshape(ref_lse.shape)[..., None] + 2.0 ** -8 * np.abs(ref_o)
           + (nkeys / 32 + 16) * 2.0 ** -24 * vmax)
    err = np.abs(got_o - ref_o)
    bad = err > tol
    assert not bad.any(), (
        f"{what}: {bad.sum()} outputs beyond tolerance, worst excess "
        f"{(err - tol).max():.3e}")
    lerr = np.abs(got_lse - ref_lse)
    assert np.all(lerr <= 1e-4 * (1 + np.abs(ref_lse))), f"{what}: lse {lerr.max():.3e}"
    return err.max(), float(np.sqrt(np.mean(err ** 2)))


# ------------------------------------------------------------ quantizer

@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (1, 2, 128), (2, 1, 300), (1, 3, 1000)])
def test_quantizer_codes_and_scales_bit_exact(oracle_mod, rotate, B, H, N):
    w, q, k, v, signs = _case(B, H, N, False, seed=40 + N, outliers=True)
    bits = oracle_mod.bf16_bits(q)
    codes_ref, sc_ref = oracle_mod.fp8_quantize(bits, rotate, signs.numpy(), 128)
    codes, sc = attn.fp8_quantize(q.cuda(), rotate, signs.tolist())
    assert np.array_equal(codes.cpu().numpy(), codes_ref)
    assert np.array_equal(sc.cpu().numpy().astype(np.float64).reshape(sc_ref.shape),
                          sc_ref)
    # one scale per head (V)
    vb = oracle_mod.bf16_bits(v)
    codes_ref, sc_ref = oracle_mod.fp8_quantize(vb, False, None, N)
    codes, sc = attn.fp8_quantize(v.cuda(), False, per_head=True)
    assert np.array_equal(codes.cpu().numpy(), codes_ref)
    assert np.array_equal(sc.cpu().numpy().astype(np.float64).reshape(sc_ref.shape),
                          sc_ref)
    assert attn.status() == 0


def test_quantizer_zero_and_wide_range_blocks(oracle_mod):
    x = torch.zeros(1, 1, 256, D, dtype=torch.bfloat16)
    x[0, 0, 128:, :] = (torch.randn(128, D, generator=torch.Generator().manual_seed(3))
                        * torch.logspace(-30, 30, D, base=2.0)).to(torch.bfloat16)
    for rotate in (False, True):
        signs = W.make_signs(4, D)
        codes_ref, sc_ref = oracle_mod.fp8_quantize(oracle_mod.bf16_bits(x), rotate,
                                                    signs.numpy(), 128)
        codes, sc = attn.fp8_quantize(x.cuda(), rotate, signs.tolist())
        assert np.array_equal(codes.cpu().numpy(), codes_ref)
        assert np.array_equal(sc.cpu().numpy().astype(np.float64).reshape(sc_ref.shape),
                              sc_ref)
    assert sc_ref[0, 0] == 1.0  # the zero tile


# ------------------------------------------------------------ attention

SHAPES = [(1, 1, 1), (1, 2, 128), (2, 1, 129), (1, 2, 300), (1, 1, 1000),
          (2, 2, 517), (1, 1, 2048)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N", SHAPES)
def test_fp8_forward_parity(oracle_mod, B, H, N, causal):
    w, q, k, v, signs = _case(B, H, N, causal, seed=60 + N + B + H, outliers=(N % 2 == 0))
    scale32 = float(np.float32(w.scale))
    z = _oracle_quant(oracle_mod, q, k, v, True, signs)
    scale_qk = scale32 * z["gain"]
    delta = _flip_delta(oracle_mod, z, scale_qk, causal)
    O_ref, l_ref, flip = oracle_mod.attention_fp8(
        z["q8"], z["qs"], z["k8"], z["ks"], z["v8"], z["vs"], causal, scale_qk,
        flip_delta=delta, tau=oracle_mod.FP8_KERNEL_TAU)
    vmax = float(np.abs(oracle_mod.e4m3_decode(z["v8"])).max() * z["vs"].max())
    # the whole path from bf16
    o, lse = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                               scale=scale32, signs=signs.tolist())
    assert attn.status() == 0
    e1 = _compare(o.float().cpu().numpy(), lse.cpu().numpy(), O_ref, l_ref, flip,
                  vmax, N, f"fp8 path {w.name}")
    # the attention kernel alone on the oracle's codes
    dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    o2, lse2 = attn.attn_fwd_fp8_quantized(
        dev(z["q8"], torch.uint8), dev(z["qs"], torch.float32),
        dev(z["k8"], torch.uint8), dev(z["ks"], torch.float32),
        dev(z["v8"], torch.uint8), dev(z["vs"], torch.float32), causal, scale_qk)
    assert attn.status() == 0
    _compare(o2.float().cpu().numpy(), lse2.cpu().numpy(), O_ref, l_ref, flip, vmax,
             N, f"fp8 kernel {w.name}")
    print(w.name, "max err %.3e rms %.3e, delta %.2e, flip bound max %.3e" %
          (e1[0], e1[1], delta, flip.max()))


def test_fp8_naive_path_parity(oracle_mod):
    """No rotation (naive FP8): same kernel, scale not divided by d."""
    w, q, k, v, signs = _case(1, 2, 640, True, seed=90, outliers=True)
    scale32 = float(np.float32(w.scale))
    z = _oracle_quant(oracle_mod, q, k, v, False, signs)
    delta = _flip_delta(oracle_mod, z, scale32, True)
    O_ref, l_ref, flip = oracle_mod.attention_fp8(
        z["q8"], z["qs"], z["k8"], z["ks"], z["v8"], z["vs"], True, scale32,
        flip_delta=delta, tau=oracle_mod.FP8_KERNEL_TAU)
    vmax = float(np.abs(oracle_mod.e4m3_decode(z["v8"])).max() * z["vs"].max())
    o, lse = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=True,
                               scale=scale32, signs=None)
    assert attn.status() == 0
    _compare(o.float().cpu().numpy(), lse.cpu().numpy(), O_ref, l_ref, flip, vmax,
             640, "naive fp8")


def test_zero_queries_average_values_on_gpu(oracle_mod):
    """Q = 0: every probability is 2^4 exactly (no rounding anywhere), so O is
    the mean of the dequantized V rows (prefix mean when causal)."""
    N = 300
    w, _, k, v, signs = _case(1, 1, N, False, seed=91)
    q = torch.zeros_like(k)
    vh = None
    for causal in (False, True):
        o, lse = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                                   signs=signs.tolist())
        assert attn.status() == 0
        if vh is None:
            v8, vs = oracle_mod.fp8_quantize(oracle_mod.bf16_bits(v), False, None, N)
            vh = oracle_mod.e4m3_decode(v8)[0, 0] * vs[0, 0]
        want = (np.cumsum(vh, 0) / np.arange(1, N + 1)[:, None]) if causal else \
            np.broadcast_to(vh.mean(0), (N, D))
        got = o.float().cpu().numpy()[0, 0]
        assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)
        ln = np.log(np.arange(1, N + 1)) if causal else np.full(N, math.log(N))
        np.testing.assert_allclose(lse.cpu().numpy()[0, 0], ln, atol=2e-5)


def test_rotation_lowers_gpu_fp8_error_with_outliers(oracle_mod):
    """[MM] "FA3: Mekanika hopper" item 3 on the GPU path: with outlier
    channels in Q and K, the rotated FP8 output is closer to exact attention
    (fp64 oracle on the bf16 inputs) than naive FP8, by more than 2.6x."""
    w, q, k, v, signs = _case(1, 4, 1024, False, seed=92, outliers=True)
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k, v)]
    O_ex, _ = oracle_mod.attention(*f, False, w.scale)
    errs = []
    for s in (None, signs.tolist()):
        o, _ = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=False,
                                 signs=s)
        o = o.float().cpu().numpy()
        errs.append(float(np.sqrt(np.mean((o - O_ex) ** 2) / np.mean(O_ex ** 2))))
    assert attn.status() == 0
    print("relative RMS error naive %.4f rotated %.4f ratio %.2f" %
          (errs[0], errs[1], errs[0] / errs[1]))
    assert errs[0] / errs[1] > 2.6


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_full_size_sampled_rows(oracle_mod, causal):
    """B=1, H=32, N=16384, d=128 (the long configuration) through the whole
    FP8 path; sampled rows of two heads against the oracle."""
    w = W.WORKLOADS["long_b1h32n16384d128"].with_(causal=causal)
    q, k, v = W.make_qkv(w)
    signs = W.make_signs(w.seed + 3, D)
    scale32 = float(np.float32(w.scale))
    o, lse = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                               scale=scale32, signs=signs.tolist())
    assert attn.status() == 0
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    rng = np.random.default_rng(5)
    for h in (0, w.H - 1):
        sel = lambda t: t[:, h:h + 1].contiguous()
        z = _oracle_quant(oracle_mod, sel(q), sel(k), sel(v), True, signs)
        rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N - 1],
                                         rng.integers(0, w.N, 60)]))
        scale_qk = scale32 * z["gain"]
        # delta from the sampled rows' own dot products
        zq = dict(z)
        zq["q8"] = z["q8"][:, :, rows]
        zq["qs"] = np.repeat(z["qs"], 128, axis=-1)[..., rows]
        qh = oracle_mod.e4m3_decode(zq["q8"]).reshape(-1, D) * zq["qs"].reshape(-1, 1)
        kh = (oracle_mod.e4m3_decode(z["k8"]).reshape(-1, D) *
              np.repeat(z["ks"].reshape(-1), 128)[:w.N, None])
        A = np.abs(qh) @ np.abs(kh).T
        S = qh @ kh.T
        c = scale_qk * LOG2E
        delta = math.log(2.0) * (2 * 2.0 ** -20 * A.max() * c +
                                 2.0 ** -22 * 2 * np.abs(S).max() * c) + EXP2_REL
        O_ref, l_ref, flip = oracle_mod.attention_fp8_rows(
            z["q8"], z["qs"], z["k8"], z["ks"], z["v8"], z["vs"], causal,
            scale_qk, rows, flip_delta=delta, tau=oracle_mod.FP8_KERNEL_TAU)
        vmax = float(np.abs(oracle_mod.e4m3_decode(z["v8"])).max() * z["vs"].max())
        _compare(o[0, h, rows], lse[0, h, rows], O_ref, l_ref, flip, vmax, w.N,
                 f"{w.name} causal={causal} head {h}")


@pytest.mark.parametrize("B,H,N,causal", [(1, 13, 16384, False), (1, 2, 300, True)])
def test_fp8_host_entry_matches_device_entry(B, H, N, causal):
    """attn_fwd_fp8_host: copies in, rotation, quantization, the FP8 kernel
    and copies out.  13 heads of 4 MiB go through the chunked pipeline (a
    ragged set of head chunks), 2 heads of 300 rows through one chunk.  The
    block scales are per head and tile, so splitting by heads changes no
    code: the outputs equal attn_fwd_fp8's bit for bit."""
    w, q, k, v, signs = _case(B, H, N, causal, seed=70 + H)
    sl = signs.tolist()
    o_dev, l_dev = attn.attn_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                                     scale=w.scale, signs=sl)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    o_h = torch.empty_like(q).pin_memory()
    l_h = torch.empty(B, H, N, dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.fp8_host_workspace_bytes(B, H, N, 128), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        attn.attn_fwd_fp8_host(qp, kp, vp, o_h, l_h, causal, w.scale, ws, signs=sl,
                               stream=stream)
        done = torch.cuda.Event()
        done.record(stream)
    done.synchronize()
    assert attn.status() == 0
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(l_h, l_dev.cpu())
