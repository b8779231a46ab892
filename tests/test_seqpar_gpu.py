"""GPU parity of sequence-sharded attention (seqpar) and of the merge
kernels (attn_merge_fold / attn_merge_finish) against the fp64 oracle.

Only one GPU is available, so the ring of P ranks runs emulated: rank after
rank on one device, each computing exactly the blocks the distributed run
computes (its query shard against key shard (r - t) mod P, causal on its
own shard, skipped for later shards under the mask) with the CUDA kernels,
and folding them with the merge kernels.  Tolerance: the forward's
(max |O - O_ref| <= 2e-2, |lse - lse_ref| <= 5e-3); the partial outputs are
bf16, the merge fp32.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import attn, seqpar
from exact_io_aware_73_b200 import workloads as W

pytestmark = pytest.mark.gpu
O_TOL, LSE_TOL = 2e-2, 5e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()
    yield
    assert attn.status() == 0


def _oracle(oracle_mod, q, k, v, causal, scale):
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k, v)]
    return oracle_mod.attention(*f, causal, scale)


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", [(1, 2, 1536, 128), (2, 1, 768, 64)])
def test_emulated_ring_matches_full_attention(oracle_mod, world, causal, B, H, N, d):
    w = W.shape_case(B, H, N, d, causal, seed=40 + world + N)
    q, k, v = W.make_qkv(w)
    stats = seqpar.RingStats()
    outs, lses = seqpar.ring_attention_emulated(
        *(seqpar.shard(t.cuda(), world) for t in (q, k, v)), causal, w.scale,
        stats=stats)
    o, lse = torch.cat(outs, dim=2), torch.cat(lses, dim=2)
    assert attn.status() == 0
    O_ref, l_ref = _oracle(oracle_mod, q, k, v, causal, w.scale)
    eo = float(np.abs(o.float().cpu().numpy() - O_ref).max())
    el = float(np.abs(lse.cpu().numpy() - l_ref).max())
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
    assert stats.blocks == (world * (world + 1) // 2 if causal else world * world)
    print(w.name, world, "max|dO| %.2e max|dlse| %.2e" % (eo, el))


def test_one_shard_is_the_plain_forward_bit_for_bit():
    w = W.shape_case(1, 3, 1000, 128, True, seed=44)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    (o1,), (l1,) = seqpar.ring_attention_emulated([q], [k], [v], True, w.scale)
    o2, l2 = attn.attn_fwd(q, k, v, causal=True, scale=w.scale)
    assert attn.status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_merge_of_disjoint_key_sets(oracle_mod):
    """Parts computed by the oracle over disjoint key sets (given to the
    kernels as bf16 O and fp32 lse) merge to attention over their union;
    a part whose lse is -inf for a row contributes nothing to that row."""
    g = torch.Generator().manual_seed(5)
    B, H, n, N, d = 1, 2, 64, 300, 128
    q = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k, v)]
    cuts = [0, 70, 200, 300]
    acc_o = torch.empty(B, H, n, d, dtype=torch.float32, device="cuda")
    acc_l = torch.empty(B, H, n, dtype=torch.float32, device="cuda")
    for i in range(3):
        a, b = cuts[i], cuts[i + 1]
        Op, lp = oracle_mod.attention_decode(f[0], f[1][:, :, a:b], f[2][:, :, a:b],
                                             False, 0.1)
        lp = lp.copy()
        if i == 1:
            lp[0, 0, 5] = -np.inf  # this row sees no key of part 1
            Op[0, 0, 5] = 0.0
        attn.merge_fold(acc_o, acc_l, torch.from_numpy(Op).to(torch.bfloat16).cuda(),
                        torch.from_numpy(lp).float().cuda(), i == 0)
    o, lse = attn.merge_finish(acc_o, acc_l)
    assert attn.status() == 0
    O_ref, l_ref = oracle_mod.attention_decode(f[0], f[1], f[2], False, 0.1)
    mask = np.ones(n, dtype=bool)
    mask[5] = False
    eo = np.abs(o.float().cpu().numpy() - O_ref)[0, 0, mask].max()
    assert eo <= O_TOL and np.abs(lse.cpu().numpy() - l_ref)[0, 1].max() <= 1e-4
    # row 5 of head 0: the merge of parts 0 and 2 only
    keep = np.r_[0:70, 200:300]
    O5, l5 = oracle_mod.attention_decode(f[0][:, :1, 5:6], f[1][:, :1, keep],
                                         f[2][:, :1, keep], False, 0.1)
    assert np.abs(o.float().cpu().numpy()[0, 0, 5] - O5[0, 0, 0]).max() <= O_TOL
    assert abs(float(lse[0, 0, 5]) - l5[0, 0, 0]) <= 1e-4


@pytest.mark.parametrize("name,world", [("long_b1h32n16384d128", 4),
                                        ("b2h16n4096d128_causal", 4)])
def test_emulated_ring_full_size_sampled_rows(oracle_mod, name, world):
    """Full-size configurations sharded over 4 emulated ranks; sampled rows
    (both ends of every shard boundary included) against the oracle."""
    w = W.WORKLOADS[name]
    q, k, v = W.make_qkv(w)
    outs, lses = seqpar.ring_attention_emulated(
        *(seqpar.shard(t.cuda(), world) for t in (q, k, v)), w.causal, w.scale)
    assert attn.status() == 0
    o = torch.cat(outs, dim=2).float().cpu().numpy().reshape(-1, w.d)
    lse = torch.cat(lses, dim=2).cpu().numpy().reshape(-1)
    n = w.N // world
    rows = set(W.sample_rows(w, 48))
    for bh in (0, w.B * w.H - 1):
        for r in range(world):
            rows.update({bh * w.N + r * n, bh * w.N + r * n + n - 1})
    rows = np.array(sorted(rows))
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    O_ref, l_ref = oracle_mod.attention_rows_bf16(*bits, w.causal, w.scale, rows)
    eo = float(np.abs(o[rows] - O_ref).max())
    el = float(np.abs(lse[rows] - l_ref).max())
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
    print(name, "max|dO| %.2e max|dlse| %.2e" % (eo, el))


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_merge_modes_fold_in_the_epilogue(oracle_mod, d):
    """attn_fwd_merge over three key blocks (first, into, last) equals
    attention over all their keys; only the final output is rounded to bf16,
    so the bound is that of a plain forward."""
    g = torch.Generator().manual_seed(8 + d)
    B, H, n = 2, 2, 700
    q = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    ks = [torch.randn(B, H, n, d, generator=g).to(torch.bfloat16) for _ in range(3)]
    vs = [torch.randn(B, H, n, d, generator=g).to(torch.bfloat16) for _ in range(3)]
    acc_o = torch.empty(B, H, n, d, dtype=torch.float32, device="cuda")
    acc_l = torch.empty(B, H, n, dtype=torch.float32, device="cuda")
    modes = [attn.MERGE_FIRST, attn.MERGE_INTO, attn.MERGE_LAST]
    for kb, vb, mode in zip(ks, vs, modes):
        out = attn.attn_fwd_merge(q.cuda(), kb.cuda(), vb.cuda(), acc_o, acc_l, mode,
                                  causal=False, scale=0.09)
    o, lse = out
    assert attn.status() == 0
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t))
         for t in (q, torch.cat(ks, dim=2), torch.cat(vs, dim=2))]
    O_ref, l_ref = oracle_mod.attention_decode(*f, False, 0.09)
    err = np.abs(o.float().cpu().numpy() - O_ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(O_ref) + 2e-3), err.max()
    assert np.abs(lse.cpu().numpy() - l_ref).max() <= 1e-4
