"""Pins for the fp64 backward oracle.

The backward pass ([MM] = marketmaker.cc post "Apakah Konteks Sehari Penuh
Mengalahkan Konteks Sepuluh Menit? ...", section "Backward pass: menghitung
ulang, bukan menyimpan") is the gradient of the forward definition.  The
oracle's gradients are pinned to:
  * central finite differences of the (separately pinned) forward oracle,
    L = sum(dO * O(Q, K, V));
  * closed forms (one key: dV = dO, dQ = dK = 0);
  * identities that follow from softmax rows summing to one: the rows of dS
    sum to zero, so sum_j dK_j = 0 and equal keys give dQ = 0; the columns
    of P sum per row to one, so sum_j dV_j = sum_i dO_i;
  * causality (a key only receives gradient from queries at or after it)
    and linearity in dO.
"""
import numpy as np
import pytest


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def _loss(oracle_mod, q, k, v, do, causal, scale):
    O, _ = oracle_mod.attention(q, k, v, causal, scale, threads=1)
    return float(np.sum(O * do))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("seed", [0, 1])
def test_gradients_match_finite_differences(oracle_mod, causal, seed):
    rng = np.random.default_rng(200 + seed)
    B, H = 1, 2
    N = int(rng.integers(2, 7))
    d = int(rng.integers(1, 4))
    q, k, v, do = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    scale = float(rng.uniform(0.3, 1.5))
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, do, causal, scale)
    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(oracle_mod, args["q"], args["k"], args["v"], do, causal, scale)
            args[name] = xm
            lm = _loss(oracle_mod, args["q"], args["k"], args["v"], do, causal, scale)
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_closed_form(oracle_mod, causal):
    q, k, v, do = (_rand((2, 2, 1, 5), s) for s in (1, 2, 3, 4))
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, do, causal, 0.4)
    np.testing.assert_array_equal(dv, do)
    np.testing.assert_allclose(dq, 0, atol=1e-15)
    np.testing.assert_allclose(dk, 0, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_key_gradients_sum_to_zero(oracle_mod, causal):
    """Rows of dS sum to zero, so sum over keys of dK vanishes."""
    q, k, v, do = (_rand((1, 3, 40, 8), s, 2.0) for s in (5, 6, 7, 8))
    _, dk, _ = oracle_mod.attention_backward(q, k, v, do, causal, 0.3)
    scale_of = np.abs(dk).max()
    np.testing.assert_allclose(dk.sum(axis=2), 0, atol=1e-12 * max(1, scale_of))


@pytest.mark.parametrize("causal", [False, True])
def test_value_gradients_sum_to_output_gradients(oracle_mod, causal):
    """Each softmax row sums to one: sum_j dV_j = sum_i dO_i."""
    q, k, v, do = (_rand((2, 2, 33, 6), s) for s in (9, 10, 11, 12))
    _, _, dv = oracle_mod.attention_backward(q, k, v, do, causal, 0.5)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), rtol=0,
                               atol=1e-12)


def test_equal_keys_give_zero_query_gradient(oracle_mod):
    q, v, do = (_rand((1, 2, 17, 4), s) for s in (13, 14, 15))
    k = np.broadcast_to(_rand((1, 2, 1, 4), 16), (1, 2, 17, 4)).copy()
    for causal in (False, True):
        dq, _, _ = oracle_mod.attention_backward(q, k, v, do, causal, 0.7)
        np.testing.assert_allclose(dq, 0, atol=1e-13)


def test_causal_last_key_gets_only_last_query(oracle_mod):
    """With the causal mask key N-1 is seen only by query N-1, so
    dV_{N-1} = P_{N-1,N-1} dO_{N-1}."""
    B, H, N, d = 1, 1, 12, 3
    q, k, v, do = (_rand((B, H, N, d), s) for s in (17, 18, 19, 20))
    _, _, dv = oracle_mod.attention_backward(q, k, v, do, True, 0.9)
    s = 0.9 * q[0, 0, N - 1] @ k[0, 0].T
    p_last = np.exp(s - s.max())
    p_last /= p_last.sum()
    np.testing.assert_allclose(dv[0, 0, N - 1], p_last[-1] * do[0, 0, N - 1],
                               rtol=1e-13, atol=1e-15)


def test_linear_in_output_gradient(oracle_mod):
    q, k, v, do = (_rand((1, 2, 21, 5), s) for s in (21, 22, 23, 24))
    g1 = oracle_mod.attention_backward(q, k, v, do, True, 0.6)
    g2 = oracle_mod.attention_backward(q, k, v, -3.0 * do, True, 0.6)
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(b, -3.0 * a, rtol=1e-13, atol=1e-14)


def test_backward_rejects_bad_arguments(oracle_mod):
    with pytest.raises(RuntimeError):
        x = np.zeros((1, 1, 2, 0))
        oracle_mod.attention_backward(x, x, x, x, False, 1.0)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_equal_the_full_backward(oracle_mod, causal):
    """The sampled-row backward (for full-size checks) equals the full fp64
    backward at those rows, on bf16 inputs of one head."""
    import torch
    g = torch.Generator().manual_seed(41)
    N, d = 150, 16
    q, k, v, do = (torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
                   for _ in range(4))
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v, do)]
    f = [oracle_mod.bf16_bits_to_f64(b) for b in bits]
    dq, dk, dv = oracle_mod.attention_backward(*f, causal, 0.3)
    qrows = np.array([0, 1, 77, 149])
    krows = np.array([0, 5, 148, 149])
    sq, sk, sv = oracle_mod.attention_backward_rows_bf16(
        *(b.reshape(N, d) for b in bits), causal, 0.3, qrows, krows)
    np.testing.assert_allclose(sq, dq[0, 0, qrows], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(sk, dk[0, 0, krows], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(sv, dv[0, 0, krows], rtol=1e-11, atol=1e-13)
