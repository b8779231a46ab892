"""Seeded synthetic inputs for the attention forward pass.

This module is the one thing the CUDA path and the fp64 oracle share: it
makes Q, K and V and nothing else.  It holds none of the attention
arithmetic.  Every tensor is sampled in fp32 on the CPU from a seeded
``torch.Generator`` and rounded to bfloat16 (round-to-nearest-even), so the
same bits go to the GPU and to the oracle.

The named workloads are the shapes the method is measured on: a small
single-head case, a GPT-2-small-shaped layer (12 heads of 64), a d=128
causal case, one full trading day at one-second resolution (23,400 steps,
12 heads; the score-matrix size quoted in the marketmaker.cc post "Apakah
Konteks Sehari Penuh Mengalahkan Konteks Sepuluh Menit? ...", introduction)
and a long non-causal d=128 case with wide score spread.  No dataset is
involved: the post's BTC one-second series is replaced by these synthetic
draws.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    q_std: float = 1.0
    k_std: float = 1.0
    v_dist: str = "normal"  # "normal" (std 1) or "uniform" (U(-1, 1))
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """Metric FLOPs: the two GEMMs, 4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "small_b1h1n256d64": Workload("small_b1h1n256d64", 1, 1, 256, 64, False,
                                  seed=1001),
    "gpt2s_b4h12n1024d64": Workload("gpt2s_b4h12n1024d64", 4, 12, 1024, 64,
                                    False, seed=1002),
    "gpt2s_b4h12n1024d64_causal": Workload("gpt2s_b4h12n1024d64_causal", 4, 12,
                                           1024, 64, True, seed=1002),
    "b2h16n4096d128_causal": Workload("b2h16n4096d128_causal", 2, 16, 4096,
                                      128, True, v_dist="uniform", seed=1003),
    "tradingday_b1h12n23400d64_causal": Workload(
        "tradingday_b1h12n23400d64_causal", 1, 12, 23400, 64, True, seed=1004),
    "long_b1h32n16384d128": Workload("long_b1h32n16384d128", 1, 32, 16384,
                                     128, False, q_std=2.0, k_std=2.0,
                                     seed=1005),
    # profiling case: the headline's per-head shape with half the heads
    # (Q/K/V still 201 MB, above the 126 MB L2), for full counter captures
    "prof_b1h16n16384d128": Workload("prof_b1h16n16384d128", 1, 16, 16384,
                                     128, False, q_std=2.0, k_std=2.0,
                                     seed=1006),
}

# The non-causal N >= 4096, d = 128 case the throughput target is set on.
HEADLINE = "long_b1h32n16384d128"


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal(shape, std: float, seed: int) -> torch.Tensor:
    x = torch.randn(shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def _uniform(shape, seed: int) -> torch.Tensor:
    x = torch.rand(shape, generator=_gen(seed), dtype=torch.float32)
    x.mul_(2.0).sub_(1.0)
    return x.to(torch.bfloat16)


def make_qkv(w: Workload, seed: int | None = None):
    """(q, k, v) bf16 CPU tensors shaped [B, H, N, d].  Q uses ``seed``, K
    ``seed + 1`` and V ``seed + 2`` (default: the workload's seed)."""
    s = w.seed if seed is None else int(seed)
    shape = (w.B, w.H, w.N, w.d)
    q = _normal(shape, w.q_std, s)
    k = _normal(shape, w.k_std, s + 1)
    if w.v_dist == "normal":
        v = _normal(shape, 1.0, s + 2)
    elif w.v_dist == "uniform":
        v = _uniform(shape, s + 2)
    else:
        raise ValueError(f"unknown value distribution {w.v_dist!r}")
    return q, k, v


def shape_case(B: int, H: int, N: int, d: int, causal: bool, seed: int,
               q_std: float = 1.0, k_std: float = 1.0,
               v_dist: str = "normal") -> Workload:
    """An ad-hoc workload for parity sweeps over shapes."""
    return Workload(f"case_b{B}h{H}n{N}d{d}{'_causal' if causal else ''}",
                    B, H, N, d, causal, q_std, k_std, v_dist, seed)


def sample_rows(w: Workload, count: int, seed: int = 7):
    """Flat row indices (bh * N + i) for sampled parity checks: always the
    first and last row of every (b, h) head block that is sampled, the ragged
    tail rows, plus uniform draws."""
    g = _gen(seed)
    total = w.B * w.H * w.N
    picks = set()
    for bh in (0, w.B * w.H - 1):
        base = bh * w.N
        for i in (0, 1, 127, 128, w.N - 1, w.N - 2):
            if 0 <= i < w.N:
                picks.add(base + i)
    r = torch.randint(0, total, (max(0, count - len(picks)),), generator=g)
    picks.update(int(x) for x in r)
    return sorted(picks)


# ------------------------------------------------------------ block masks

def make_block_mask(seed: int, T: int, density: float, heads: int = 0,
                    local: int = 0) -> torch.Tensor:
    """A block mask for the block-sparse variant: uint8 [T, T] (or
    [heads, T, T] when heads > 0), 1 = the (128-query, 128-key) block is kept.
    Each block is kept with probability ``density`` (seeded draw), and the
    ``local`` blocks on and below the diagonal of every row are always kept
    (a sliding window of local * 128 keys)."""
    shape = (heads, T, T) if heads > 0 else (T, T)
    m = (torch.rand(shape, generator=_gen(seed)) < float(density)).to(torch.uint8)
    if local > 0:
        i = torch.arange(T)[:, None]
        j = torch.arange(T)[None, :]
        m |= ((j <= i) & (j > i - int(local))).to(torch.uint8)
    return m


# Block-sparse workloads: the long headline shape with a sliding window of
# 8 key tiles (1,024 keys) plus 25 % of the other key tiles at random, one
# mask for every head, and the trading day with a 30-minute window (15 key
# tiles of 128 one-second steps) plus 10 % random tiles, causal.
SPARSE_WORKLOADS = {
    "sparse_long_b1h32n16384d128": (WORKLOADS["long_b1h32n16384d128"], 0.25, 8),
    "sparse_tradingday_b1h12n23400d64_causal": (
        WORKLOADS["tradingday_b1h12n23400d64_causal"], 0.10, 15),
}


def block_mask_for(name: str) -> torch.Tensor:
    """The [T, T] mask of a named block-sparse workload (seed 4242)."""
    w, density, local = SPARSE_WORKLOADS[name]
    return make_block_mask(4242, (w.N + 127) // 128, density, local=local)


def sparse_flops(w: Workload, mask: torch.Tensor) -> float:
    """FLOPs of the two GEMMs over the computed blocks only: 4 d per visible
    score, with the causal mask and the ragged last key tile counted
    exactly (scores of masked-out blocks are not computed)."""
    T = (w.N + 127) // 128
    m = mask.reshape(-1, T, T).to(torch.int64)
    qlen = torch.full((T,), 128, dtype=torch.int64)
    qlen[-1] = w.N - 128 * (T - 1)
    klen = qlen.clone()
    pairs = qlen[:, None] * klen[None, :]
    if w.causal:
        # rows of tile i see keys <= row: full tiles below the diagonal, and
        # r + 1 keys of the diagonal tile for its row r
        i = torch.arange(T)[:, None]
        j = torch.arange(T)[None, :]
        diag = qlen * (qlen + 1) // 2
        pairs = torch.where(j < i, pairs, torch.zeros_like(pairs))
        pairs = pairs + torch.diag(diag)
    per_head = (m * pairs[None]).sum(dim=(1, 2)).to(torch.float64)
    heads = w.B * w.H
    total = per_head.sum() * (heads if m.shape[0] == 1 else 1)
    return float(4.0 * w.d * total)


# ------------------------------------------------------------ FP8 inputs

def make_signs(seed: int, d: int) -> torch.Tensor:
    """The random signs of the randomized Hadamard rotation: d entries of
    +-1 (int8), drawn from a seeded generator.  They are an input of the FP8
    path (both sides receive the same draw)."""
    bits = torch.randint(0, 2, (d,), generator=_gen(seed), dtype=torch.int64)
    return (1 - 2 * bits).to(torch.int8)


def add_channel_outliers(x: torch.Tensor, channels, factor: float) -> torch.Tensor:
    """Outlier features: the given coordinates of every row multiplied by
    ``factor`` (in fp32, then rounded to bf16 again).  Large, persistent
    per-channel magnitudes are the pattern that spoils plain FP8
    quantization of Q and K."""
    y = x.float()
    y[..., list(channels)] *= float(factor)
    return y.to(torch.bfloat16)


def outlier_channels(seed: int, d: int, count: int):
    """``count`` distinct coordinates in [0, d), drawn from a seeded generator."""
    return sorted(int(c) for c in torch.randperm(d, generator=_gen(seed))[:count])


# ------------------------------------------------------------ decode inputs

@dataclass(frozen=True)
class DecodeWorkload:
    """Nq new queries (the last Nq positions) against an Nk-long key/value
    sequence per (batch, head)."""
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """The two GEMMs over visible keys: 4 d per (query, key) pair."""
        if self.causal:
            keys = sum(self.Nk - self.Nq + i + 1 for i in range(self.Nq))
        else:
            keys = self.Nq * self.Nk
        return 4.0 * self.B * self.H * keys * self.d

    def kv_bytes(self) -> int:
        """K and V read once: the bytes a decode step must stream."""
        return 2 * self.B * self.H * self.Nk * self.d * 2


DECODE_WORKLOADS = {
    # few heads, very long context: a grid over (batch, head) alone would
    # occupy 8 of 148 SMs
    "decode_b1h8nq1nk262144d128": DecodeWorkload(
        "decode_b1h8nq1nk262144d128", 1, 8, 1, 262144, 128, True, seed=2001),
    # a batch of sequences, one new token each
    "decode_b8h32nq1nk32768d128": DecodeWorkload(
        "decode_b8h32nq1nk32768d128", 8, 32, 1, 32768, 128, True, seed=2002),
    # one trading day of one-second steps as context, 12 heads of 64,
    # four new steps at once
    "decode_tradingday_b16h12nq4nk23400d64": DecodeWorkload(
        "decode_tradingday_b16h12nq4nk23400d64", 16, 12, 4, 23400, 64, True,
        seed=2003),
    # sixteen new positions per sequence at once (a chunk of new queries):
    # one pass over K/V on the tensor cores serves all sixteen
    "decode_b4h16nq16nk32768d128": DecodeWorkload(
        "decode_b4h16nq16nk32768d128", 4, 16, 16, 32768, 128, True, seed=2004),
}

DECODE_HEADLINE = "decode_b1h8nq1nk262144d128"


def make_decode_qkv(w: DecodeWorkload, seed: int | None = None):
    """(q [B, H, Nq, d], k, v [B, H, Nk, d]) bf16 CPU tensors, N(0, 1),
    seeds seed, seed + 1, seed + 2 (default: the workload's seed)."""
    s = w.seed if seed is None else int(seed)
    q = _normal((w.B, w.H, w.Nq, w.d), 1.0, s)
    k = _normal((w.B, w.H, w.Nk, w.d), 1.0, s + 1)
    v = _normal((w.B, w.H, w.Nk, w.d), 1.0, s + 2)
    return q, k, v


def decode_case(B, H, Nq, Nk, d, causal, seed) -> DecodeWorkload:
    return DecodeWorkload(f"decode_case_b{B}h{H}nq{Nq}nk{Nk}d{d}"
                          f"{'_causal' if causal else ''}", B, H, Nq, Nk, d,
                          causal, seed)
