"""The seeded input recipe: deterministic, shaped and distributed as stated."""
import math

import torch

from exact_io_aware_73_b200 import workloads as W


def test_named_workloads_match_their_shapes():
    w = W.WORKLOADS
    assert (w["small_b1h1n256d64"].B, w["small_b1h1n256d64"].N) == (1, 256)
    assert w["tradingday_b1h12n23400d64_causal"].N == 23400
    assert w["tradingday_b1h12n23400d64_causal"].N % 128 != 0
    assert w["long_b1h32n16384d128"].q_std == 2.0
    assert w["b2h16n4096d128_causal"].v_dist == "uniform"
    assert W.HEADLINE in w and not w[W.HEADLINE].causal
    for x in w.values():
        assert math.isclose(x.scale, 1 / math.sqrt(x.d))
    f = w["long_b1h32n16384d128"].flops()
    assert f == 4 * 32 * 16384 ** 2 * 128
    assert w["gpt2s_b4h12n1024d64_causal"].flops() * 2 == \
        w["gpt2s_b4h12n1024d64"].flops()


def test_inputs_are_deterministic_and_bf16():
    w = W.shape_case(2, 3, 129, 64, True, seed=5)
    a = W.make_qkv(w)
    b = W.make_qkv(w)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (2, 3, 129, 64)
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    c = W.make_qkv(w, seed=6)
    assert not torch.equal(a[0], c[0])
    # Q, K and V come from different streams
    assert not torch.equal(a[0], a[1]) and not torch.equal(a[1], a[2])


def test_distributions():
    w = W.shape_case(1, 4, 4096, 64, False, seed=9, q_std=2.0, k_std=2.0,
                     v_dist="uniform")
    q, k, v = (t.float() for t in W.make_qkv(w))
    assert abs(q.std().item() - 2.0) < 0.02
    assert abs(k.mean().item()) < 0.02
    assert v.min().item() >= -1.0 and v.max().item() <= 1.0
    assert abs(v.std().item() - 1 / math.sqrt(3)) < 0.01


def test_sample_rows_cover_edges():
    w = W.WORKLOADS["tradingday_b1h12n23400d64_causal"]
    rows = W.sample_rows(w, 256)
    assert len(rows) >= 256 - 12
    assert 0 in rows and 23399 in rows and 23400 * 12 - 1 in rows
    assert all(0 <= r < 12 * 23400 for r in rows)
    assert rows == W.sample_rows(w, 256)
