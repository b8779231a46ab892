"""Pins for the decode oracle (oracle_attention_decode_f64 and its bf16 row
variant): few new queries against a long key/value sequence.

Source: the briefgpt.xyz summary page of FlashAttention-2 (arXiv 2307.08691),
entry "LeanAttention" (Feb 2024): attention for the decode phase of long
contexts, computed in parallel over the sequence.  The result is exact
attention; the queries are the last Nq positions of an Nk-long sequence, so
with the causal mask query i sees keys 0 .. Nk - Nq + i.  Pinned to:
  * the self-attention oracle when Nq = Nk (masks coincide);
  * closed forms: zero queries give the prefix mean of the values with
    lse = ln(visible keys) -- this fixes the mask's alignment exactly;
  * a single query sees every key with or without the mask;
  * the split identity the decode kernel relies on: attention over a
    sequence equals the lse-weighted merge of attention over its parts;
  * brute force on tiny inputs, expanded by hand in numpy;
  * the bf16 row variant equals the fp64 one on widened inputs.
"""
import math

import numpy as np
import pytest
import torch


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_reduce_to_self_attention(oracle_mod, causal):
    q, k, v = (_rand((2, 3, 37, 8), s) for s in (1, 2, 3))
    O, lse = oracle_mod.attention_decode(q, k, v, causal, 0.4)
    O2, lse2 = oracle_mod.attention(q, k, v, causal, 0.4)
    np.testing.assert_allclose(O, O2, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse, lse2, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("Nq,Nk", [(1, 50), (4, 50), (7, 7), (3, 130)])
def test_zero_queries_give_prefix_means(oracle_mod, Nq, Nk):
    v = _rand((1, 2, Nk, 5), 4)
    k = _rand((1, 2, Nk, 5), 5)
    q = np.zeros((1, 2, Nq, 5))
    O, lse = oracle_mod.attention_decode(q, k, v, True, 0.7)
    for i in range(Nq):
        n = Nk - Nq + i + 1        # keys 0 .. Nk - Nq + i
        np.testing.assert_allclose(O[:, :, i], v[:, :, :n].mean(axis=2),
                                   rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[:, :, i], math.log(n), rtol=1e-14)
    On, lsen = oracle_mod.attention_decode(q, k, v, False, 0.7)
    np.testing.assert_allclose(On, np.broadcast_to(v.mean(axis=2, keepdims=True), On.shape),
                               rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lsen, math.log(Nk), rtol=1e-14)


def test_single_query_sees_every_key(oracle_mod):
    q, k, v = _rand((3, 1, 1, 16), 6), _rand((3, 1, 200, 16), 7), _rand((3, 1, 200, 16), 8)
    a = oracle_mod.attention_decode(q, k, v, True, 0.25)
    b = oracle_mod.attention_decode(q, k, v, False, 0.25)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("cut", [1, 64, 100, 199])
def test_split_merge_identity(oracle_mod, cut):
    """softmax over the whole sequence = lse-weighted merge of the parts:
    lse = log(exp(lse_a) + exp(lse_b)), O = sum_p exp(lse_p - lse) O_p."""
    q, k, v = _rand((1, 2, 3, 8), 9, 2.0), _rand((1, 2, 200, 8), 10), _rand((1, 2, 200, 8), 11)
    O, lse = oracle_mod.attention_decode(q, k, v, False, 0.5)
    Oa, la = oracle_mod.attention_decode(q, k[:, :, :cut], v[:, :, :cut], False, 0.5)
    Ob, lb = oracle_mod.attention_decode(q, k[:, :, cut:], v[:, :, cut:], False, 0.5)
    m = np.maximum(la, lb)
    lm = m + np.log(np.exp(la - m) + np.exp(lb - m))
    Om = np.exp(la - lm)[..., None] * Oa + np.exp(lb - lm)[..., None] * Ob
    np.testing.assert_allclose(lm, lse, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Om, O, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    Nq = int(rng.integers(1, 4))
    Nk = int(rng.integers(Nq, 8))
    d = int(rng.integers(1, 5))
    q, k, v = (rng.standard_normal((1, 1, n, d)) for n in (Nq, Nk, Nk))
    scale = float(rng.uniform(0.2, 1.5))
    for causal in (False, True):
        O, lse = oracle_mod.attention_decode(q, k, v, causal, scale)
        for i in range(Nq):
            last = (Nk - Nq + i) if causal else (Nk - 1)
            w = [math.exp(scale * sum(q[0, 0, i, t] * k[0, 0, j, t] for t in range(d)))
                 for j in range(last + 1)]
            tot = sum(w)
            for t in range(d):
                want = sum(w[j] * v[0, 0, j, t] for j in range(last + 1)) / tot
                assert abs(O[0, 0, i, t] - want) <= 1e-12 * (1 + abs(want))
            assert abs(lse[0, 0, i] - math.log(tot)) <= 1e-12 * (1 + abs(math.log(tot)))


def test_bf16_rows_match_fp64(oracle_mod):
    g = torch.Generator().manual_seed(12)
    q = torch.randn(2, 2, 3, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(2, 2, 300, 64, generator=g).to(torch.bfloat16)
    v = torch.randn(2, 2, 300, 64, generator=g).to(torch.bfloat16)
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    f = [oracle_mod.bf16_bits_to_f64(b) for b in bits]
    for causal in (False, True):
        O, lse = oracle_mod.attention_decode(*f, causal, 0.125)
        rows = np.array([0, 4, 5, 11])
        O2, l2 = oracle_mod.attention_decode_rows_bf16(*bits, causal, 0.125, rows)
        np.testing.assert_allclose(O2, O.reshape(-1, 64)[rows], rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(l2, lse.reshape(-1)[rows], rtol=1e-14, atol=1e-15)


def test_rejects_more_queries_than_keys_when_causal(oracle_mod):
    with pytest.raises(RuntimeError):
        oracle_mod.attention_decode(np.zeros((1, 1, 5, 4)), np.zeros((1, 1, 4, 4)),
                                    np.zeros((1, 1, 4, 4)), True, 1.0)
