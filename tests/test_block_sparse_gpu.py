"""GPU parity of block-sparse attention (attn_fwd_block_sparse) against the
fp64 block-sparse oracle.

The block-sparse extension of the tiled method (briefgpt.xyz summary page of
FlashAttention-2, arXiv 2307.08691, FlashAttention entry): the (128-query,
128-key) blocks a mask leaves out are skipped, which is the same as setting
their scores to -inf.  Tolerances are the forward's: max |O - O_ref| <= 2e-2,
max |lse - lse_ref| <= 5e-3; rows that keep no key must be exactly O = 0 and
lse = -inf.  With every block kept (or, under the causal mask, every block
on and below the diagonal) the result must equal attn_fwd's bit for bit: the
kernel is the forward kernel walking a list of K tiles.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import attn
from exact_io_aware_73_b200 import workloads as W

O_TOL = 2e-2
LSE_TOL = 5e-3

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


def _compare(o, lse, o_ref, lse_ref, what):
    o = o.reshape(o_ref.shape)
    lse = lse.reshape(lse_ref.shape)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), what
    assert np.all(o[empty] == 0), what
    keep = ~empty
    assert np.all(np.isfinite(o[keep])) and np.all(np.isfinite(lse[keep])), what
    eo = float(np.max(np.abs(o[keep] - o_ref[keep]))) if keep.any() else 0.0
    el = float(np.max(np.abs(lse[keep] - lse_ref[keep]))) if keep.any() else 0.0
    assert eo <= O_TOL, f"{what}: max|dO| {eo}"
    assert el <= LSE_TOL, f"{what}: max|dlse| {el}"
    return eo, el


SHAPES = [(1, 1, 1, 128), (1, 3, 129, 64), (1, 2, 300, 64), (2, 1, 1000, 128),
          (1, 1, 1536, 128), (2, 2, 777, 64)]


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", SHAPES)
def test_block_sparse_parity(oracle_mod, B, H, N, d, causal, per_head):
    w = W.shape_case(B, H, N, d, causal, seed=300 + N + d + B + H)
    q, k, v = W.make_qkv(w)
    T = (N + 127) // 128
    m = W.make_block_mask(17 + N, T, 0.5, heads=B * H if per_head else 0)
    if T > 1:
        # one query tile keeps no block at all (its rows: O = 0, lse = -inf)
        m.reshape(-1, T, T)[:, 1, :] = 0
    o, lse = attn.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(), m.cuda(),
                                        causal=causal, scale=w.scale)
    assert attn.status() == 0
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    o_ref, l_ref = oracle_mod.attention_block_sparse_bf16(*bits, causal, w.scale,
                                                          m.numpy())
    _compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, w.name)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(300, 64), (1000, 128), (1536, 128)])
def test_full_mask_equals_dense_forward_bit_for_bit(N, d, causal):
    w = W.shape_case(2, 3, N, d, causal, seed=400 + N)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    T = (N + 127) // 128
    full = torch.ones(T, T, dtype=torch.uint8)
    if causal:
        full = torch.tril(full)   # blocks above the diagonal never count
    o, lse = attn.attn_fwd_block_sparse(q, k, v, full.cuda(), causal=causal,
                                        scale=w.scale)
    od, ld = attn.attn_fwd(q, k, v, causal=causal, scale=w.scale)
    assert attn.status() == 0
    assert torch.equal(o, od) and torch.equal(lse, ld)


def test_empty_mask_gives_zero_and_minus_infinity():
    w = W.shape_case(1, 2, 400, 128, False, seed=51)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    m = torch.zeros(4, 4, dtype=torch.uint8, device="cuda")
    o = torch.full_like(q, 7.0)
    lse = torch.zeros(1, 2, 400, device="cuda")
    attn.attn_fwd_block_sparse(q, k, v, m, out=o, lse=lse)
    assert attn.status() == 0
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def _mask_patterns(T):
    """Masks whose pairs of consecutive query tiles keep very different key
    tiles: alternating parity (disjoint lists), one tile keeping only the
    last key tile while its partner keeps all, and the first tile of every
    pair keeping nothing."""
    kj = np.arange(T)
    alt = ((kj[None, :] % 2) == (np.arange(T)[:, None] % 2)).astype(np.uint8)
    lone = np.ones((T, T), np.uint8)
    lone[0::2, :] = 0
    lone[0::2, T - 1] = 1
    first_empty = np.ones((T, T), np.uint8)
    first_empty[0::2, :] = 0
    return {"alternating": alt, "lone_last": lone, "first_empty": first_empty}


@pytest.mark.parametrize("pattern", ["alternating", "lone_last", "first_empty"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(2048, 64), (1900, 128)])
def test_pairs_with_different_key_lists(oracle_mod, pattern, causal, N, d):
    """A unit is two consecutive query tiles that load the union of their
    lists; each computes only its own key tiles (one issuing thread per
    tile), so these masks make the tiles of a pair skip many of the ring's
    slots."""
    w = W.shape_case(1, 2, N, d, causal, seed=500 + N + d)
    q, k, v = W.make_qkv(w)
    T = (N + 127) // 128
    m = torch.from_numpy(_mask_patterns(T)[pattern])
    o, lse = attn.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(), m.cuda(),
                                        causal=causal, scale=w.scale)
    assert attn.status() == 0
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    o_ref, l_ref = oracle_mod.attention_block_sparse_bf16(*bits, causal, w.scale,
                                                          m.numpy())
    _compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref,
             f"{pattern} {w.name}")


@pytest.mark.parametrize("d", [64, 128])
def test_block_sparse_forced_rescale_over_many_units(oracle_mod, d):
    """Scores that grow along the key axis force the output correction on
    every kept K tile; 40 heads of 4 pairs put several units on each CTA,
    and the alternating-parity mask gives the two tiles of a pair disjoint
    key lists."""
    B, H, N = 1, 40, 1024
    q = torch.zeros(B, H, N, d)
    q[..., 0] = 1.0
    k = torch.zeros(B, H, N, d)
    k[..., 0] = torch.linspace(0, 400, N)
    g = torch.Generator().manual_seed(17)
    v = torch.randn(B, H, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    T = N // 128
    m = _mask_patterns(T)["alternating"].copy()
    m[:, 0] = 1  # every row keeps K tile 0 too
    for causal in (False, True):
        o, lse = attn.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(),
                                            torch.from_numpy(m).cuda(), causal=causal,
                                            scale=1.0)
        assert attn.status() == 0
        bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
        o_ref, l_ref = oracle_mod.attention_block_sparse_bf16(*bits, causal, 1.0, m)
        _compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref,
                 f"forced rescale d={d} causal={causal}")


@pytest.mark.parametrize("name", sorted(W.SPARSE_WORKLOADS))
def test_block_sparse_workloads_sampled_rows(oracle_mod, name):
    """The benchmark's block-sparse workloads, in the launch the benchmark
    times, on sampled rows (first, tile edges, last, ragged tail, random)."""
    w, _, _ = W.SPARSE_WORKLOADS[name]
    q, k, v = W.make_qkv(w)
    m = W.block_mask_for(name)
    o, lse = attn.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(), m.cuda(),
                                        causal=w.causal, scale=w.scale)
    assert attn.status() == 0
    rows = np.array(W.sample_rows(w, 256))
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    o_ref, l_ref = oracle_mod.attention_block_sparse_rows_bf16(
        *bits, w.causal, w.scale, m.numpy(), rows)
    _compare(o.float().cpu().numpy().reshape(-1, w.d)[rows],
             lse.cpu().numpy().reshape(-1)[rows], o_ref, l_ref, name)


@pytest.mark.parametrize("seed", range(12))
def test_random_masks_and_shapes(oracle_mod, seed):
    """Random shapes (ragged N, d = 64 or 128, causal or not) with random
    per-head masks of random density: pairs of query tiles whose key lists
    overlap anywhere from fully to not at all, empty rows included."""
    rng = np.random.default_rng(900 + seed)
    d = 64 if seed % 2 else 128
    B, H = 1, int(rng.integers(1, 4))
    N = int(rng.integers(129, 1800))
    causal = bool(rng.integers(0, 2))
    w = W.shape_case(B, H, N, d, causal, seed=950 + seed)
    q, k, v = W.make_qkv(w)
    T = (N + 127) // 128
    density = float(rng.uniform(0.05, 0.95))
    m = (rng.random((B * H, T, T)) < density).astype(np.uint8)
    o, lse = attn.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(),
                                        torch.from_numpy(m).cuda(), causal=causal,
                                        scale=w.scale)
    assert attn.status() == 0
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    o_ref, l_ref = oracle_mod.attention_block_sparse_bf16(*bits, causal, w.scale, m)
    _compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref,
             f"seed {seed}: {w.name} density {density:.2f}")
