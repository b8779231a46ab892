"""Pins for the block-sparse oracle (oracle.attention_block_sparse_rows_bf16).

The block-sparse extension of the tiled method (briefgpt.xyz summary page of
FlashAttention-2, arXiv 2307.08691, FlashAttention entry) drops the keys of
the (128-query, 128-key) blocks a mask leaves out.  The pins fix it to
things other than itself: the dense row oracle (itself pinned in
test_oracle_pins.py) with every block kept, or on the keys a row keeps
gathered by plain indexing; the causal mask; per-head masks; and the
reading for rows with nothing left (O = 0, lse = -inf).
"""
import math

import numpy as np
import pytest
import torch


def _bits(oracle_mod, shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return oracle_mod.bf16_bits((torch.randn(shape, generator=g) * std).to(torch.bfloat16))


def _case(oracle_mod, B, H, N, d, seed):
    return [_bits(oracle_mod, (B, H, N, d), seed + s, 1.5) for s in range(3)]


def _mask(T, density, seed, heads=0):
    g = np.random.default_rng(seed)
    shape = (heads, T, T) if heads else (T, T)
    return (g.random(shape) < density).astype(np.uint8)


@pytest.mark.parametrize("causal", [False, True])
def test_every_block_kept_is_dense_attention(oracle_mod, causal):
    q, k, v = _case(oracle_mod, 1, 2, 300, 16, 1)
    T = 3
    rows = np.arange(2 * 300)
    O, L = oracle_mod.attention_block_sparse_rows_bf16(
        q, k, v, causal, 0.3, np.ones((T, T), np.uint8), rows)
    Od, Ld = oracle_mod.attention_rows_bf16(q, k, v, causal, 0.3, rows)
    assert np.array_equal(O, Od) and np.array_equal(L, Ld)


def test_causal_ignores_blocks_above_the_diagonal(oracle_mod):
    """Under the causal mask only blocks on or below the diagonal matter: a
    lower-triangular block mask and a full one give the causal result."""
    q, k, v = _case(oracle_mod, 1, 1, 400, 8, 4)
    T = 4
    rows = np.arange(400)
    tri = np.tril(np.ones((T, T), np.uint8))
    O1, L1 = oracle_mod.attention_block_sparse_rows_bf16(q, k, v, True, 0.5, tri, rows)
    O2, L2 = oracle_mod.attention_block_sparse_rows_bf16(
        q, k, v, True, 0.5, np.ones((T, T), np.uint8), rows)
    Od, Ld = oracle_mod.attention_rows_bf16(q, k, v, True, 0.5, rows)
    assert np.array_equal(O1, Od) and np.array_equal(O2, Od)
    assert np.array_equal(L1, Ld) and np.array_equal(L2, Ld)


@pytest.mark.parametrize("causal", [False, True])
def test_a_row_is_dense_attention_over_the_keys_it_keeps(oracle_mod, causal):
    """Each row equals dense attention of that query over the kept keys,
    gathered by plain indexing (the dense oracle on a problem whose every
    query is the row's query and whose keys are the kept ones)."""
    N, d = 520, 16
    q, k, v = _case(oracle_mod, 1, 1, N, d, 7)
    T = 5
    m = _mask(T, 0.5, 8)
    m[:, 0] = 1  # every row keeps a block (row 0 of the causal case too)
    rows = np.array([0, 1, 127, 128, 200, 255, 256, 300, 383, 384, 511, 519])
    O, L = oracle_mod.attention_block_sparse_rows_bf16(q, k, v, causal, 0.25, m, rows)
    for a, i in enumerate(rows):
        keep = [j for j in range(N) if m[i // 128, j // 128] and (not causal or j <= i)]
        n = len(keep)
        qq = np.repeat(q[:, :, i:i + 1], n, axis=2)
        Ok, Lk = oracle_mod.attention_rows_bf16(qq, k[:, :, keep], v[:, :, keep],
                                                False, 0.25, [0])
        np.testing.assert_allclose(O[a], Ok[0], rtol=0, atol=1e-14)
        np.testing.assert_allclose(L[a], Lk[0], rtol=0, atol=1e-13)


def test_rows_with_no_kept_key_give_zero_and_minus_infinity(oracle_mod):
    q, k, v = _case(oracle_mod, 1, 1, 300, 8, 11)
    m = np.ones((3, 3), np.uint8)
    m[1, :] = 0                         # query tile 1 keeps nothing
    m[2, 2] = 0
    rows = np.arange(300)
    O, L = oracle_mod.attention_block_sparse_rows_bf16(q, k, v, False, 0.4, m, rows)
    assert np.all(O[128:256] == 0) and np.all(L[128:256] == -np.inf)
    assert np.all(np.isfinite(O[:128])) and np.all(np.isfinite(L[256:]))
    # causal, diagonal block removed: row 0 sees nothing
    m = np.ones((3, 3), np.uint8)
    m[0, 0] = 0
    O, L = oracle_mod.attention_block_sparse_rows_bf16(q, k, v, True, 0.4, m, rows)
    assert np.all(O[:128] == 0) and np.all(L[:128] == -np.inf)


def test_per_head_masks_follow_the_head(oracle_mod):
    """A per-head mask is the shared-mask result of each head's own mask."""
    B, H, N, d = 2, 2, 260, 8
    q, k, v = _case(oracle_mod, B, H, N, d, 21)
    T = 3
    m = _mask(T, 0.6, 22, heads=B * H)
    m[:, :, 0] = 1
    rows = np.arange(B * H * N)
    O, L = oracle_mod.attention_block_sparse_rows_bf16(q, k, v, False, 0.3, m, rows)
    for h in range(B * H):
        b, hh = divmod(h, H)
        sel = lambda x: x[b:b + 1, hh:hh + 1]
        Oh, Lh = oracle_mod.attention_block_sparse_rows_bf16(
            sel(q), sel(k), sel(v), False, 0.3, m[h], np.arange(N))
        assert np.array_equal(O[h * N:(h + 1) * N], Oh)
        assert np.array_equal(L[h * N:(h + 1) * N], Lh)


def test_block_boundaries_are_128_keys_and_queries(oracle_mod):
    """Keys 127 and 128 fall in different blocks, and so do queries 127 and
    128: dropping key block 1 changes query 127's result only by key 128 on,
    and dropping query block 1's keys leaves query 127 untouched."""
    N, d = 256, 4
    q, k, v = _case(oracle_mod, 1, 1, N, d, 31)
    m = np.ones((2, 2), np.uint8)
    m[1, 1] = 0
    O, L = oracle_mod.attention_block_sparse_rows_bf16(q, k, v, False, 1.0, m,
                                                       [127, 128])
    Od, Ld = oracle_mod.attention_rows_bf16(q, k, v, False, 1.0, [127])
    assert np.array_equal(O[0], Od[0]) and L[0] == Ld[0]
    Ok, Lk = oracle_mod.attention_rows_bf16(q[:, :, :128], k[:, :, :128], v[:, :, :128],
                                            False, 1.0, [0])
    qq = np.repeat(q[:, :, 128:129], 128, axis=2)
    Ok, Lk = oracle_mod.attention_rows_bf16(qq, k[:, :, :128], v[:, :, :128],
                                            False, 1.0, [0])
    np.testing.assert_allclose(O[1], Ok[0], rtol=0, atol=1e-14)
    assert math.isclose(L[1], Lk[0], rel_tol=0, abs_tol=1e-13)


def test_bad_masks_are_rejected(oracle_mod):
    q, k, v = _case(oracle_mod, 1, 1, 130, 4, 41)
    with pytest.raises(ValueError):
        oracle_mod.attention_block_sparse_rows_bf16(q, k, v, False, 1.0,
                                                    np.ones((3, 3), np.uint8), [0])
    with pytest.raises(RuntimeError):
        oracle_mod.attention_block_sparse_rows_bf16(q, k, v, False, 1.0,
                                                    np.ones((2, 2), np.uint8), [130])
