"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test fixes the oracle to a closed form, an invariant of the definition,
a brute-force expansion on tiny inputs, the hand-worked fixture in
``tests/golden/hand_worked.txt`` or the pages' own blocked algorithm.  The
definition is that of the marketmaker.cc post "Apakah Konteks Sehari Penuh
Mengalahkan Konteks Sepuluh Menit? ..." (sections "Mengapa perhatian terikat
pada memori", "Integrasinya delapan baris" for the causal mask,
"Pengulangan softmax online" for the claim that the blocked form is exact).
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.txt")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(shape, seed, std=1.0):
    return _rng(seed).standard_normal(shape) * std


# --------------------------------------------------------------------------
# closed forms and special cases
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_single_key_gives_v_and_dot_product_lse(oracle_mod, causal):
    """N = 1: softmax of one score is 1, so O = V exactly and lse = the score."""
    q, k, v = (_rand((2, 3, 1, 5), s) for s in (1, 2, 3))
    scale = 0.37
    O, lse = oracle_mod.attention(q, k, v, causal, scale)
    assert np.array_equal(O, v)
    dots = scale * np.einsum("bhnd,bhnd->bhn", q, k)
    np.testing.assert_allclose(lse, dots, rtol=1e-15, atol=1e-15)


def test_zero_queries_noncausal_average_all_values(oracle_mod):
    """Q = 0: every score is 0, the softmax is uniform: O = mean of V rows,
    lse = ln N."""
    B, H, N, d = 2, 2, 37, 6
    v = _rand((B, H, N, d), 4)
    k = _rand((B, H, N, d), 5)
    q = np.zeros((B, H, N, d))
    O, lse = oracle_mod.attention(q, k, v, False, 0.5)
    mean = v.mean(axis=2, keepdims=True)
    np.testing.assert_allclose(O, np.broadcast_to(mean, O.shape), rtol=0,
                               atol=1e-14)
    np.testing.assert_allclose(lse, np.full((B, H, N), math.log(N)), rtol=1e-15)


def test_zero_queries_causal_average_prefix(oracle_mod):
    """Q = 0 with the causal mask: row i averages V[0..i], lse = ln(i + 1)."""
    B, H, N, d = 1, 3, 41, 4
    v = _rand((B, H, N, d), 6)
    k = _rand((B, H, N, d), 7)
    q = np.zeros((B, H, N, d))
    O, lse = oracle_mod.attention(q, k, v, True, 1.0)
    counts = np.arange(1, N + 1).reshape(1, 1, N, 1)
    prefix_mean = np.cumsum(v, axis=2) / counts
    np.testing.assert_allclose(O, prefix_mean, rtol=0, atol=1e-14)
    np.testing.assert_allclose(
        lse, np.broadcast_to(np.log(np.arange(1, N + 1)), (B, H, N)), rtol=1e-15)


def test_causal_first_row_is_first_value(oracle_mod):
    """Causal row 0 sees only key 0: O[0] = V[0], lse[0] = scale * q0 . k0."""
    q, k, v = (_rand((2, 2, 19, 8), s) for s in (8, 9, 10))
    O, lse = oracle_mod.attention(q, k, v, True, 0.25)
    assert np.array_equal(O[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(
        lse[:, :, 0], 0.25 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]),
        rtol=1e-14, atol=1e-15)


def _parse_golden(path):
    cases, cur = {}, None
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        if line.startswith("[case"):
            cur = line[len("[case"):].rstrip("]").strip()
            cases[cur] = {}
            continue
        key, val = (x.strip() for x in line.split("=", 1))
        if key in ("causal",):
            cases[cur][key] = bool(int(val))
        elif key == "scale":
            cases[cur][key] = float(val)
        elif key == "lse":
            cases[cur][key] = np.array([float(x) for x in val.split()])
        else:
            cases[cur][key] = np.array(
                [[float(x) for x in row.split()] for row in val.split(";")])
    return cases


def test_hand_worked_fixture(oracle_mod):
    cases = _parse_golden(GOLDEN)
    assert len(cases) == 4
    for name, c in cases.items():
        shp = (1, 1) + c["Q"].shape
        O, lse = oracle_mod.attention(c["Q"].reshape(shp), c["K"].reshape(shp),
                                      c["V"].reshape(shp), c["causal"],
                                      c["scale"])
        np.testing.assert_allclose(O[0, 0], c["O"], rtol=0, atol=2e-16 * 8,
                                   err_msg=name)
        np.testing.assert_allclose(lse[0, 0], c["lse"], rtol=0, atol=4e-16 * 4,
                                   err_msg=name)
        # the blocked algorithm on the same fixture, blocks of one row/key
        Ob, lseb = oracle_mod.attention_blocked(
            c["Q"].reshape(shp), c["K"].reshape(shp), c["V"].reshape(shp),
            c["causal"], c["scale"], 1, 1)
        np.testing.assert_allclose(Ob[0, 0], c["O"], rtol=0, atol=1e-15,
                                   err_msg=name)
        np.testing.assert_allclose(lseb[0, 0], c["lse"], rtol=0, atol=1e-15,
                                   err_msg=name)


# --------------------------------------------------------------------------
# invariants of the definition
# --------------------------------------------------------------------------

def test_softmax_rows_sum_to_one(oracle_mod):
    rng = _rng(11)
    for n, spread in [(1, 1.0), (7, 1.0), (300, 5.0), (1000, 300.0),
                      (64, 1e4)]:
        s = rng.standard_normal(n) * spread
        p = oracle_mod.softmax_row(s)
        assert np.all(p >= 0) and np.all(np.isfinite(p))
        assert abs(p.sum() - 1.0) <= 1e-14 * max(1, n) ** 0.5
        assert int(np.argmax(p)) == int(np.argmax(s))
        # ratios of probabilities are exp of score differences
        j, k = int(np.argmax(s)), int(np.argmin(s))
        if s[j] - s[k] < 600:
            np.testing.assert_allclose(p[k] / p[j], math.exp(s[k] - s[j]),
                                       rtol=1e-12)


def test_row_shift_invariance(oracle_mod):
    """Adding c to every score of one row leaves that row of O unchanged and
    adds c to its lse; the other rows do not move."""
    rng = _rng(12)
    S = rng.standard_normal((5, 33)) * 3
    V = rng.standard_normal((33, 7))
    O0, l0 = oracle_mod.attend_scores(S, V)
    for c in (-1e3, -7.5, 0.125, 40.0, 650.0):
        S2 = S.copy()
        S2[2] += c
        O1, l1 = oracle_mod.attend_scores(S2, V)
        np.testing.assert_allclose(O1, O0, rtol=0, atol=5e-14)
        assert abs(l1[2] - (l0[2] + c)) <= 1e-12 * max(1.0, abs(c))
        np.testing.assert_array_equal(np.delete(l1, 2), np.delete(l0, 2))


def test_masked_scores_are_dropped(oracle_mod):
    """-inf scores (masked keys) are the same as removing those keys."""
    rng = _rng(13)
    S = rng.standard_normal((4, 10))
    V = rng.standard_normal((10, 3))
    keep = np.array([0, 2, 3, 7, 9])
    Sm = np.full_like(S, -np.inf)
    Sm[:, keep] = S[:, keep]
    O1, l1 = oracle_mod.attend_scores(Sm, V)
    O2, l2 = oracle_mod.attend_scores(S[:, keep], V[keep])
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(l1, l2)


def test_key_permutation_equivariance(oracle_mod):
    """Non-causal attention does not care about the order of key/value rows
    permuted together."""
    q, k, v = (_rand((1, 2, 29, 6), s) for s in (14, 15, 16))
    perm = _rng(17).permutation(29)
    O1, l1 = oracle_mod.attention(q, k, v, False, 0.4)
    O2, l2 = oracle_mod.attention(q, k[:, :, perm], v[:, :, perm], False, 0.4)
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-14)


def test_query_permutation_equivariance(oracle_mod):
    """Permuting query rows permutes output rows (non-causal)."""
    q, k, v = (_rand((1, 1, 23, 5), s) for s in (18, 19, 20))
    perm = _rng(21).permutation(23)
    O1, l1 = oracle_mod.attention(q, k, v, False, 0.7)
    O2, l2 = oracle_mod.attention(q[:, :, perm], k, v, False, 0.7)
    np.testing.assert_array_equal(O2, O1[:, :, perm])
    np.testing.assert_array_equal(l2, l1[:, :, perm])


def test_causal_row_equals_noncausal_on_prefix(oracle_mod):
    """Causal row i is plain attention of query i over keys 0..i: this pins
    the mask boundary (key i itself is visible, key i + 1 is not)."""
    B, H, N, d = 1, 2, 17, 4
    q, k, v = (_rand((B, H, N, d), s) for s in (22, 23, 24))
    O, lse = oracle_mod.attention(q, k, v, True, 0.6)
    for i in (0, 1, 5, 16):
        Op, lp = _prefix_row(oracle_mod, q, k, v, i, 0.6)
        np.testing.assert_allclose(O[:, :, i], Op[:, :, -1], rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse[:, :, i], lp[:, :, -1], rtol=0,
                                   atol=1e-15)


def _prefix_row(oracle_mod, q, k, v, i, scale):
    # attention of the single query i against the first i + 1 keys: build a
    # (i + 1)-row problem whose last query is query i, non-causal
    qq = np.concatenate([np.zeros_like(q[:, :, :i]), q[:, :, i:i + 1]], axis=2)
    return oracle_mod.attention(qq, k[:, :, :i + 1], v[:, :, :i + 1], False,
                                scale)


def test_scale_enters_once_multiplying_scores(oracle_mod):
    """attention(q, k, v, scale=s) == attention(s * q, k, v, scale=1)."""
    q, k, v = (_rand((2, 1, 21, 8), s) for s in (25, 26, 27))
    s = 0.125
    O1, l1 = oracle_mod.attention(q, k, v, False, s)
    O2, l2 = oracle_mod.attention(q * s, k, v, False, 1.0)
    np.testing.assert_allclose(O1, O2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-14, atol=1e-14)


def test_values_affine_equivariance(oracle_mod):
    """Softmax rows sum to one, so V -> a V + b maps O -> a O + b (a dropped
    normalisation would fail this for b != 0)."""
    q, k, v = (_rand((1, 2, 25, 3), s) for s in (28, 29, 30))
    for causal in (False, True):
        O1, l1 = oracle_mod.attention(q, k, v, causal, 0.5)
        O2, l2 = oracle_mod.attention(q, k, -2.5 * v + 3.0, causal, 0.5)
        np.testing.assert_allclose(O2, -2.5 * O1 + 3.0, rtol=0, atol=1e-13)
        np.testing.assert_array_equal(l1, l2)


def test_output_in_convex_hull_of_values(oracle_mod):
    q, k, v = (_rand((1, 3, 50, 4), s, std) for s, std in
               ((31, 4.0), (32, 4.0), (33, 1.0)))
    for causal in (False, True):
        O, _ = oracle_mod.attention(q, k, v, causal, 1.0)
        N = v.shape[2]
        for i in range(N):
            vis = v[:, :, : (i + 1 if causal else N)]
            assert np.all(O[:, :, i] >= vis.min(axis=2) - 1e-14)
            assert np.all(O[:, :, i] <= vis.max(axis=2) + 1e-14)


def test_large_scores_stay_finite(oracle_mod):
    """Scores of several hundred (N(0, 2^2) queries and keys, d = 128, scaled
    up further) overflow a naive exp; the max-subtracted oracle stays finite
    and inside the hull of V."""
    B, H, N, d = 1, 1, 96, 128
    q = _rand((B, H, N, d), 34, 2.0)
    k = _rand((B, H, N, d), 35, 2.0)
    v = _rand((B, H, N, d), 36)
    for scale in (1 / math.sqrt(d), 4.0):
        O, lse = oracle_mod.attention(q, k, v, False, scale)
        assert np.all(np.isfinite(O)) and np.all(np.isfinite(lse))
        assert np.all(O <= v.max(axis=2, keepdims=True) + 1e-12)
        assert np.all(O >= v.min(axis=2, keepdims=True) - 1e-12)
    # at scale 4 the scores reach hundreds: lse is then within ln N of the max
    s = 4.0 * np.einsum("bhid,bhjd->bhij", q, k)
    assert s.max() > 300
    smax = s.max(axis=3)
    assert np.all(lse >= smax - 1e-9) and np.all(lse <= smax + math.log(N) + 1e-9)


# --------------------------------------------------------------------------
# brute force and the pages' blocked algorithm
# --------------------------------------------------------------------------

def _brute(q, k, v, causal, scale):
    """Direct expansion with Python floats, no max subtraction (tiny inputs
    only): O_i = sum_j exp(s_ij) v_j / sum_j exp(s_ij)."""
    N, d = q.shape
    O = [[0.0] * d for _ in range(N)]
    lse = [0.0] * N
    for i in range(N):
        num = [0.0] * d
        den = 0.0
        for j in range(N):
            if causal and j > i:
                continue
            s = scale * sum(float(q[i][t]) * float(k[j][t]) for t in range(d))
            w = math.exp(s)
            den += w
            for t in range(d):
                num[t] += w * float(v[j][t])
        O[i] = [x / den for x in num]
        lse[i] = math.log(den)
    return np.array(O), np.array(lse)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_tiny(oracle_mod, seed):
    rng = _rng(100 + seed)
    N = int(rng.integers(1, 9))
    d = int(rng.integers(1, 5))
    q, k, v = (rng.standard_normal((1, 1, N, d)) for _ in range(3))
    scale = float(rng.uniform(0.1, 2.0))
    for causal in (False, True):
        O, lse = oracle_mod.attention(q, k, v, causal, scale)
        Ob, lb = _brute(q[0, 0], k[0, 0], v[0, 0], causal, scale)
        np.testing.assert_allclose(O[0, 0], Ob, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[0, 0], lb, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("Br,Bc", [(1, 1), (4, 4), (5, 3), (16, 16), (8, 64),
                                   (64, 7)])
@pytest.mark.parametrize("causal", [False, True])
def test_blocked_algorithm_equals_two_pass(oracle_mod, Br, Bc, causal):
    """The pages' blocked online softmax reproduces the two-pass definition
    to rounding (the exact-reassociation claim)."""
    q, k, v = (_rand((2, 2, 37, 8), s, 2.0) for s in (41, 42, 43))
    O, lse = oracle_mod.attention(q, k, v, causal, 0.35)
    Ob, lb = oracle_mod.attention_blocked(q, k, v, causal, 0.35, Br, Bc)
    np.testing.assert_allclose(Ob, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lb, lse, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# the bf16 row-sampled entry point
# --------------------------------------------------------------------------

def test_bf16_widening_is_exact(oracle_mod):
    x = torch.randn(4096, generator=torch.Generator().manual_seed(3)) * 100
    xb = x.to(torch.bfloat16)
    bits = oracle_mod.bf16_bits(xb)
    np.testing.assert_array_equal(oracle_mod.bf16_bits_to_f64(bits),
                                  xb.to(torch.float64).numpy())


@pytest.mark.parametrize("causal", [False, True])
def test_rows_bf16_matches_full_oracle(oracle_mod, causal):
    g = torch.Generator().manual_seed(5)
    shape = (2, 3, 45, 16)
    q, k, v = (torch.randn(shape, generator=g).to(torch.bfloat16)
               for _ in range(3))
    qb, kb, vb = (oracle_mod.bf16_bits(t) for t in (q, k, v))
    O, lse = oracle_mod.attention(oracle_mod.bf16_bits_to_f64(qb),
                                  oracle_mod.bf16_bits_to_f64(kb),
                                  oracle_mod.bf16_bits_to_f64(vb), causal, 0.25)
    rows = np.array([0, 1, 44, 45, 100, 2 * 3 * 45 - 1])
    Or, lr = oracle_mod.attention_rows_bf16(qb, kb, vb, causal, 0.25, rows)
    np.testing.assert_array_equal(Or, O.reshape(-1, 16)[rows])
    np.testing.assert_array_equal(lr, lse.reshape(-1)[rows])


def test_bad_arguments_are_rejected(oracle_mod):
    with pytest.raises(RuntimeError):
        oracle_mod.softmax_row(np.zeros(0))
    with pytest.raises(RuntimeError):
        oracle_mod.attend_scores(np.full((1, 3), -np.inf), np.zeros((3, 2)))
    qb = np.zeros((1, 1, 4, 2), dtype=np.uint16)
    with pytest.raises(RuntimeError):
        oracle_mod.attention_rows_bf16(qb, qb, qb, False, 1.0, np.array([4]))


# --------------------------------------------------------------------------
# the full-output entry point (score blocks by BLAS products)
# --------------------------------------------------------------------------

def _bf16(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,panel", [(1, 256), (45, 16), (300, 128), (777, 256)])
def test_full_bf16_matches_row_oracle(oracle_mod, causal, N, panel):
    """The panelled BLAS form of the definition equals the scalar C oracle to
    rounding on every row, with ragged last panels and panels that straddle
    the causal diagonal."""
    shape = (2, 2, N, 16)
    q, k, v = (_bf16(shape, s, 2.0) for s in (11, 12, 13))
    qb, kb, vb = (oracle_mod.bf16_bits(t) for t in (q, k, v))
    O, lse = oracle_mod.attention(oracle_mod.bf16_bits_to_f64(qb),
                                  oracle_mod.bf16_bits_to_f64(kb),
                                  oracle_mod.bf16_bits_to_f64(vb), causal, 0.3)
    Of, lf = oracle_mod.attention_full_bf16(qb, kb, vb, causal, 0.3, panel=panel)
    np.testing.assert_allclose(Of, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lf, lse, rtol=0, atol=1e-12)


def test_full_bf16_closed_forms(oracle_mod):
    """N = 1 gives V and the dot product; Q = 0 gives the (prefix) mean of V
    with lse = ln N (ln(i + 1) when causal)."""
    one = [oracle_mod.bf16_bits(_bf16((1, 3, 1, 8), s)) for s in (21, 22, 23)]
    for causal in (False, True):
        O, lse = oracle_mod.attention_full_bf16(*one, causal, 0.5)
        f = [oracle_mod.bf16_bits_to_f64(b) for b in one]
        assert np.array_equal(O, f[2])
        np.testing.assert_allclose(lse, 0.5 * np.einsum("bhnd,bhnd->bhn", f[0], f[1]),
                                   rtol=1e-15, atol=1e-15)
    N = 333
    k, v = (oracle_mod.bf16_bits(_bf16((1, 2, N, 8), s)) for s in (24, 25))
    q = np.zeros_like(k)
    vf = oracle_mod.bf16_bits_to_f64(v)
    O, lse = oracle_mod.attention_full_bf16(q, k, v, False, 1.0, panel=100)
    np.testing.assert_allclose(O, np.broadcast_to(vf.mean(axis=2, keepdims=True),
                                                  O.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(N), rtol=1e-15)
    O, lse = oracle_mod.attention_full_bf16(q, k, v, True, 1.0, panel=100)
    np.testing.assert_allclose(O, np.cumsum(vf, axis=2) /
                               np.arange(1, N + 1).reshape(1, 1, N, 1), atol=1e-14)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, N + 1)),
                                                    lse.shape), rtol=1e-15)
