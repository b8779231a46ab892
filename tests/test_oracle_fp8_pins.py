"""Pins for the FP8 oracle (oracle/fp8_oracle.c).

The FP8 path ([MM] = marketmaker.cc post "Apakah Konteks Sehari Penuh
Mengalahkan Konteks Sepuluh Menit? ...", section "FA3: Mekanika hopper",
item 3) rotates Q and K at random, block-quantizes Q, K, V to FP8 (E4M3) and
runs the blocked online softmax with E4M3 probabilities.  Each piece is
pinned to something other than the oracle itself:

  * E4M3 encoding and decoding: torch's float8_e4m3fn conversion (a library
    routine) over every code and over dense and tie-point samples;
  * the rotation: scipy's Hadamard matrix, H H^T = d I, and exact
    preservation of dot products up to the factor d;
  * block quantization: the scale is the largest power of two that keeps the
    block's maximum within 448, checked with exact comparisons; the codes are
    torch's E4M3 conversion of the scaled values; error bounds of the format;
  * the FP8 attention: closed forms (one key, zero queries, causal row 0),
    an exactly representable case where it must equal the fp64 two-pass
    oracle on the dequantized operands, lse that never depends on the
    rounding of P, and the rounding-error bound of E4M3 probabilities;
  * the accuracy claim of the section (rotation lowers FP8 error when Q and
    K carry outliers).
"""
import math

import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import workloads as W

TORCH_E4M3 = torch.float8_e4m3fn


def _torch_encode(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(TORCH_E4M3) \
        .view(torch.uint8).numpy()


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(TORCH_E4M3) \
        .to(torch.float64).numpy()


# ------------------------------------------------------------------ E4M3

def test_decode_matches_library_for_every_code(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle_mod.e4m3_decode(codes)
    ref = _torch_decode(codes)
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), ~finite)
    np.testing.assert_array_equal(ours[finite], ref[finite])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_encode_roundtrips_every_finite_code(oracle_mod):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle_mod.e4m3_decode(codes).astype(np.float32)
    back = oracle_mod.e4m3_encode(vals)
    # +0 and -0 both decode to 0; the sign bit is kept
    np.testing.assert_array_equal(back, codes)


def test_encode_matches_library_on_dense_samples_and_ties(oracle_mod):
    rng = np.random.default_rng(3)
    mags = np.exp2(rng.uniform(-14, 8.85, 200_000)).astype(np.float32)
    x = mags * rng.choice([-1.0, 1.0], mags.size).astype(np.float32)
    # every midpoint between adjacent codes (ties go to the even code)
    vals = oracle_mod.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.float32([0.0, 2.0 ** -10, 3 * 2.0 ** -11])])
    x = x[np.abs(x) < 464]  # the library turns larger values into NaN
    np.testing.assert_array_equal(oracle_mod.e4m3_encode(x), _torch_encode(x))


def test_encode_saturates(oracle_mod):
    c = oracle_mod.e4m3_encode(np.float32([464, 1e6, -500, 3.0e38]))
    np.testing.assert_array_equal(c, [0x7E, 0x7E, 0xFE, 0x7E])


# -------------------------------------------------------------- rotation

@pytest.mark.parametrize("d", [64, 128])
def test_rotation_is_signed_sylvester_hadamard(oracle_mod, d):
    from scipy.linalg import hadamard
    s = W.make_signs(11, d).numpy()
    R = oracle_mod.hadamard_rotate(np.eye(d), s)      # rows of diag(s) H
    np.testing.assert_array_equal(R, np.diag(s.astype(np.float64)) @ hadamard(d))
    np.testing.assert_array_equal(R @ R.T, d * np.eye(d))


def test_rotation_preserves_dot_products_up_to_d(oracle_mod):
    d = 128
    g = torch.Generator().manual_seed(5)
    q = torch.randn(16, d, generator=g).to(torch.bfloat16)
    k = torch.randn(16, d, generator=g).to(torch.bfloat16)
    qf, kf = (oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k))
    s = W.make_signs(12, d).numpy()
    qr, kr = oracle_mod.hadamard_rotate(qf, s), oracle_mod.hadamard_rotate(kf, s)
    np.testing.assert_allclose(qr @ kr.T, d * (qf @ kf.T), rtol=1e-13, atol=1e-12)


def test_rotation_rejects_bad_signs(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.hadamard_rotate(np.zeros((2, 8)), np.array([1, 0, 1, 1, 1, 1, 1, 1]))


# ----------------------------------------------------------- quantization

def _bits(t):
    import oracle
    return oracle.bf16_bits(t)


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("N,block", [(300, 128), (256, 128), (77, 1000)])
def test_block_quantization_scale_and_codes(oracle_mod, rotate, N, block):
    d = 128
    g = torch.Generator().manual_seed(N + block)
    x = (torch.randn(2, N, d, generator=g) * 3).to(torch.bfloat16)
    x = W.add_channel_outliers(x, [5, 90], 12.0)
    s = W.make_signs(13, d).numpy()
    bits = _bits(x)
    codes, scales = oracle_mod.fp8_quantize(bits, rotate, s, block)
    xf = oracle_mod.bf16_bits_to_f64(bits)
    y = oracle_mod.hadamard_rotate(xf, s) if rotate else xf
    yf = y.astype(np.float32)
    nblk = -(-N // block)
    assert scales.shape == (2, nblk)
    for bh in range(2):
        for b in range(nblk):
            blk = yf[bh, b * block:(b + 1) * block].astype(np.float64)
            amax = np.abs(blk).max()
            sc = scales[bh, b]
            e = -math.log2(sc)
            assert e == int(e)                          # a power of two
            assert amax / sc <= 448.0 < amax / sc * 2   # the largest such
            want = _torch_encode((blk / sc).astype(np.float32))
            np.testing.assert_array_equal(codes[bh, b * block:(b + 1) * block], want)
            deq = oracle_mod.e4m3_decode(codes[bh, b * block:(b + 1) * block]) * sc
            # E4M3: half a step, 2^-4 relative in the normal range,
            # 2^-10 * scale absolute among the subnormals
            bound = np.maximum(2.0 ** -4 * np.abs(blk), 2.0 ** -10 * sc)
            assert np.all(np.abs(deq - blk) <= bound)


def test_quantization_of_zero_block(oracle_mod):
    bits = np.zeros((1, 130, 64), dtype=np.uint16)
    codes, scales = oracle_mod.fp8_quantize(bits, False, None, 128)
    assert np.all(codes == 0) and np.all(scales == 1.0)


# ------------------------------------------------------- FP8 attention

def _codes_from_values(oracle_mod, vals):
    """Codes of values that E4M3 represents exactly (checked)."""
    c = oracle_mod.e4m3_encode(np.asarray(vals, dtype=np.float32))
    assert np.array_equal(oracle_mod.e4m3_decode(c), np.asarray(vals, np.float64))
    return c


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_gives_value_row(oracle_mod, causal):
    rng = np.random.default_rng(1)
    d = 16
    q8 = _codes_from_values(oracle_mod, rng.integers(-4, 5, (1, 1, d)))
    k8 = _codes_from_values(oracle_mod, rng.integers(-4, 5, (1, 1, d)))
    v8 = _codes_from_values(oracle_mod, rng.integers(-8, 9, (1, 1, d)) / 4)
    O, lse, _ = oracle_mod.attention_fp8(q8, [[0.5]], k8, [[2.0]], v8, [0.25],
                                         causal, 0.3)
    qv, kv = oracle_mod.e4m3_decode(q8) * 0.5, oracle_mod.e4m3_decode(k8) * 2.0
    np.testing.assert_array_equal(O, oracle_mod.e4m3_decode(v8) * 0.25)
    assert lse[0, 0] == pytest.approx(0.3 * float((qv * kv).sum()), abs=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_the_values(oracle_mod, causal):
    N, d = 300, 32
    rng = np.random.default_rng(2)
    q8 = np.zeros((1, N, d), np.uint8)
    k8 = oracle_mod.e4m3_encode(rng.standard_normal((1, N, d)).astype(np.float32))
    v8 = oracle_mod.e4m3_encode(rng.standard_normal((1, N, d)).astype(np.float32))
    ks = np.full((1, 3), 0.5)
    O, lse, _ = oracle_mod.attention_fp8(q8, np.ones((1, 3)), k8, ks, v8, [2.0],
                                         causal, 0.125)
    vhat = oracle_mod.e4m3_decode(v8)[0] * 2.0
    if causal:
        want = np.cumsum(vhat, axis=0) / np.arange(1, N + 1)[:, None]
        np.testing.assert_allclose(lse[0], np.log(np.arange(1, N + 1)), atol=1e-12)
    else:
        want = np.broadcast_to(vhat.mean(axis=0), (N, d))
        np.testing.assert_allclose(lse[0], math.log(N), atol=1e-12)
    np.testing.assert_allclose(O[0], want, rtol=0, atol=1e-13)


def _exact_case(oracle_mod, N, d, causal, seed):
    """Scores that are integer multiples of ln 2 with a spread up to 17:
    every probability 256 * 2^(s - m) / ln 2 is an exact E4M3 value, so the
    FP8 attention must equal exact attention on the dequantized operands."""
    rng = np.random.default_rng(seed)
    q = np.zeros((1, N, d))
    q[0, :, 0] = rng.choice([1.0, 0.0], N)
    k = oracle_mod.e4m3_decode(oracle_mod.e4m3_encode(
        rng.standard_normal((1, N, d)).astype(np.float32)))
    k[0, :, 0] = rng.integers(0, 9, N) * 2.0   # q . k in {0, 1, ..., 16}
    v = rng.integers(-16, 17, (1, N, d)) / 8.0
    # keys 17 below the largest possible score: p = 2^-9, the smallest code
    k[0, ::97, 0] = -1.0
    q8, k8, v8 = (_codes_from_values(oracle_mod, a) for a in (q, k, v))
    qh, kh, vh = (oracle_mod.e4m3_decode(c) for c in (q8, k8, v8))
    return q8, k8, v8, qh, kh, vh


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 129])
def test_exactly_representable_case_equals_exact_attention(oracle_mod, causal, N):
    d = 8
    q8, k8, v8, qh, kh, vh = _exact_case(oracle_mod, N, d, causal, N)
    tiles = -(-N // 128)
    O, lse, fb = oracle_mod.attention_fp8(q8, np.ones((1, tiles)), k8,
                                          np.ones((1, tiles)), v8, [1.0],
                                          causal, math.log(2.0), flip_delta=1e-6)
    Oe, le = oracle_mod.attention(qh[None], kh[None], vh[None], causal, math.log(2.0))
    np.testing.assert_allclose(O, Oe[0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, le[0], rtol=0, atol=1e-12)
    # every probability is an exact code: nowhere near a rounding boundary
    assert np.all(fb == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_lse_is_independent_of_probability_rounding(oracle_mod, causal):
    """l adds the unrounded probabilities, so lse is the exact log-sum-exp
    of the dequantized scores whatever E4M3 does to P."""
    N, d = 260, 64
    g = torch.Generator().manual_seed(9)
    q, k, v = ((torch.randn(1, 1, N, d, generator=g) * 2).to(torch.bfloat16)
               for _ in range(3))
    s = W.make_signs(14, d).numpy()
    z = oracle_mod.quantize_qkv_fp8(*(_bits(t) for t in (q, k, v)), True, s)
    O, lse, _ = oracle_mod.attention_fp8(z["q8"], z["qs"], z["k8"], z["ks"],
                                         z["v8"], z["vs"], causal,
                                         z["gain"] / 8.0)
    deq = lambda c, sc, blk: oracle_mod.e4m3_decode(c) * np.repeat(
        sc.reshape(-1), blk)[:N, None]
    qh = deq(z["q8"][0, 0], z["qs"], 128)
    kh = deq(z["k8"][0, 0], z["ks"], 128)
    vh = oracle_mod.e4m3_decode(z["v8"][0, 0]) * z["vs"][0, 0]
    Oe, le = oracle_mod.attention(qh[None, None], kh[None, None], vh[None, None],
                                  causal, z["gain"] / 8.0)
    np.testing.assert_allclose(lse[0, 0], le[0, 0], rtol=0, atol=1e-12)
    # and O differs from exact attention on the same operands only by the
    # E4M3 rounding of P: at most 2^-4 relative per probability in the
    # normal range plus 2^-10 absolute per subnormal one (l >= 256)
    bound = (2.0 ** -4 + N * 2.0 ** -10 / 256) * np.abs(vh).max()
    assert np.abs(O[0, 0] - Oe[0, 0]).max() <= bound
    assert np.abs(O[0, 0] - Oe[0, 0]).max() > 0  # the rounding is really there


def test_causal_row_zero(oracle_mod):
    N, d = 140, 16
    rng = np.random.default_rng(4)
    q8, k8, v8 = (oracle_mod.e4m3_encode(rng.standard_normal((1, N, d)).astype(np.float32))
                  for _ in range(3))
    O, lse, _ = oracle_mod.attention_fp8(q8, np.ones((1, 2)), k8, np.ones((1, 2)),
                                         v8, [0.5], True, 0.25)
    np.testing.assert_array_equal(O[0, 0], oracle_mod.e4m3_decode(v8[0, 0]) * 0.5)
    qk = (oracle_mod.e4m3_decode(q8[0, 0]) * oracle_mod.e4m3_decode(k8[0, 0])).sum()
    assert lse[0, 0] == pytest.approx(0.25 * qk, abs=1e-12)


def test_rows_subset_matches_full(oracle_mod):
    N, d = 200, 32
    rng = np.random.default_rng(6)
    q8, k8, v8 = (oracle_mod.e4m3_encode(rng.standard_normal((2, N, d)).astype(np.float32))
                  for _ in range(3))
    qs, ks, vs = np.ones((2, 2)), np.full((2, 2), 0.5), np.array([1.0, 2.0])
    O, lse, _ = oracle_mod.attention_fp8(q8, qs, k8, ks, v8, vs, True, 0.2)
    rows = np.array([0, 5, 199, 200, 333, 399])
    O2, l2, _ = oracle_mod.attention_fp8_rows(q8, qs, k8, ks, v8, vs, True, 0.2, rows)
    np.testing.assert_array_equal(O2, O.reshape(-1, d)[rows])
    np.testing.assert_array_equal(l2, lse.reshape(-1)[rows])


# ------------------------------------------------------ accuracy claim

def test_rotation_lowers_fp8_error_with_outlier_channels(oracle_mod):
    """[MM] "FA3: Mekanika hopper" item 3: rotating before block quantization
    spreads outliers and lowers the FP8 error.  Q and K with two outlier
    channels (x8): the rotated path's relative RMS error against exact
    attention must be well below the plain FP8 path's; without outliers the
    two are alike."""
    def errs(outliers):
        w = W.shape_case(1, 2, 512, 128, False, seed=5)
        q, k, v = W.make_qkv(w)
        if outliers:
            ch = W.outlier_channels(15, 128, 2)
            q, k = (W.add_channel_outliers(t, ch, 8.0) for t in (q, k))
        bits = [_bits(t) for t in (q, k, v)]
        f = [oracle_mod.bf16_bits_to_f64(b) for b in bits]
        Oe, _ = oracle_mod.attention(*f, False, w.scale)
        out = []
        for rot in (False, True):
            z = oracle_mod.quantize_qkv_fp8(*bits, rot, W.make_signs(25, 128).numpy())
            O, _, _ = oracle_mod.attention_fp8(z["q8"], z["qs"], z["k8"], z["ks"],
                                               z["v8"], z["vs"], False,
                                               w.scale * z["gain"])
            out.append(np.sqrt(np.mean((O - Oe) ** 2) / np.mean(Oe ** 2)))
        return out
    plain, rotated = errs(True)
    assert plain / rotated > 2.6
    plain0, rotated0 = errs(False)
    assert 0.8 < plain0 / rotated0 < 1.25
    assert rotated < 0.08 and rotated0 < 0.08


# ------------------------------------------------------------ lazy base

def _attend_log2_scores(oracle_mod, scores, v, tau):
    """FP8 oracle on one query whose scores (log2 units) against the keys are
    `scores` (scale ln 2, q = e0, k[:, 0] = scores), values v [N, d]."""
    N, d = len(scores), v.shape[1]
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    k = np.zeros((1, N, d))
    k[0, :, 0] = scores
    q8, k8, v8 = (_codes_from_values(oracle_mod, a) for a in (q, k, v[None]))
    tiles = -(-N // 128)
    # the query is row 0 of a one-row problem: pad Q to N rows of zeros
    q8 = np.concatenate([q8, np.zeros((1, N - 1, d), np.uint8)], axis=1)
    O, lse, _ = oracle_mod.attention_fp8_rows(
        q8, np.ones((1, tiles)), k8, np.ones((1, tiles)), v8, [1.0], False,
        math.log(2.0), [0], tau=tau)
    return O[0], lse[0]


@pytest.mark.parametrize("tau", [0.0, 4.0])
def test_probability_offset_follows_the_threshold(oracle_mod, tau):
    """p = 2^(8 - tau) exp(s - m): two keys at 0 and -14 (log2 units) below
    the base.  With tau = 0 the small one is 2^-6, an exact E4M3 normal; with
    tau = 4 it is 2^-10, half the smallest subnormal, which rounds to even:
    0.  lse adds the unrounded p either way."""
    v = np.array([[0.0, 1.0], [1.0, 0.0]])
    O, lse = _attend_log2_scores(oracle_mod, [0.0, -14.0], v, tau)
    want = 2.0 ** -14 / (1 + 2.0 ** -14) if tau == 0 else 0.0
    assert O[0] == pytest.approx(want, rel=1e-14, abs=0)
    assert O[1] == pytest.approx(1 / (1 + 2.0 ** -14), rel=1e-14)
    assert lse == pytest.approx(math.log1p(2.0 ** -14), rel=1e-12)


@pytest.mark.parametrize("tau", [0.0, 4.0])
def test_base_moves_only_past_the_threshold(oracle_mod, tau):
    """Three key blocks whose maxima are 0, 3 and 8 (log2 units).  With
    tau = 4 the base stays at 0 through the second block (gap 3) and moves
    to 8 at the third (gap 8); every p is then a power of two that E4M3
    holds exactly: 16 and 2^-9 in the first two blocks (the key at -13), 16
    in the third.  So the result equals exact attention; a base that moved
    at gap 3 would flush the -13 key (2^-12 -> 0), one that stayed at gap 8
    would saturate (2^12 -> 448).  tau = 0 is exact as well (256, 2^-8)."""
    N = 384
    scores = np.full(N, -30.0)
    v = np.zeros((N, 4))
    for col, (key, sc) in enumerate([(0, 0.0), (128, 3.0), (129, -13.0), (256, 8.0)]):
        scores[key] = sc
        v[key, col] = 1.0
    O, lse = _attend_log2_scores(oracle_mod, scores, v, tau)
    w = np.exp2(scores)
    exact = (w @ v) / w.sum()
    np.testing.assert_allclose(O, exact, rtol=1e-13, atol=0)
    assert lse == pytest.approx(math.log(w.sum()) * 1.0, rel=1e-13)


def test_kernel_threshold_is_within_e4m3_range(oracle_mod):
    """The kernel's threshold keeps p <= 2^8 < 448 and the normal range at
    2^-(14 - tau) of the row maximum."""
    assert 0 < oracle_mod.FP8_KERNEL_TAU <= 8
    assert 2.0 ** 8 < 448
