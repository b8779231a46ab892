"""GPU parity: the sm_100a kernel (through the C ABI) against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation): max |O - O_ref| <= 2e-2 and
max |lse - lse_ref| <= 5e-3, element by element on the same seeded bf16
inputs.  Small shapes are compared in full; the full-size workloads are run
exactly as the benchmark launches them and compared on sampled rows the
oracle computes one by one.
"""
import math

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
    cap = torch.cuda.get_device_capability()
    if cap != (10, 0):
        pytest.skip(f"needs a B200 (sm_100), found sm_{cap[0]}{cap[1]}")
    attn.lib()  # raises if the library is missing: no fallback
    yield
    assert attn.status() == 0


def _run(q, k, v, causal, scale):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = attn.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    rc = attn.status()
    assert rc == 0, attn.strerror(rc)
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _oracle_full(oracle_mod, q, k, v, causal, scale):
    f = [oracle_mod.bf16_bits_to_f64(oracle_mod.bf16_bits(t)) for t in (q, k, v)]
    return oracle_mod.attention(*f, causal, scale)


def _compare(o, lse, o_ref, lse_ref, what):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), what
    eo = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    el = float(np.max(np.abs(lse - lse_ref))) if lse.size else 0.0
    assert eo <= O_TOL, f"{what}: max|O-O_ref| = {eo}"
    assert el <= LSE_TOL, f"{what}: max|lse-lse_ref| = {el}"
    return eo, el


SHAPES = [
    # (B, H, N, d): single tile, tile boundaries, ragged tails, empty second
    # Q tile of a unit (N mod 256 in (0, 128]), several units per head
    (1, 1, 1, 64), (1, 2, 2, 128), (2, 1, 127, 64), (1, 2, 128, 128),
    (2, 2, 129, 64), (1, 1, 255, 128), (1, 3, 256, 64), (2, 1, 257, 128),
    (1, 2, 300, 64), (1, 1, 384, 128), (2, 3, 1000, 64), (1, 2, 1000, 128),
    (1, 1, 1536, 128), (3, 5, 200, 64),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", SHAPES)
def test_parity_shapes(oracle_mod, B, H, N, d, causal):
    w = W.shape_case(B, H, N, d, causal, seed=100 + N + d + 7 * B + H)
    q, k, v = W.make_qkv(w)
    o, lse = _run(q, k, v, causal, w.scale)
    o_ref, lse_ref = _oracle_full(oracle_mod, q, k, v, causal, w.scale)
    _compare(o, lse, o_ref, lse_ref, w.name)


@pytest.mark.parametrize("name", ["small_b1h1n256d64", "gpt2s_b4h12n1024d64",
                                  "gpt2s_b4h12n1024d64_causal"])
def test_parity_workloads_full(oracle_mod, name):
    w = W.WORKLOADS[name]
    q, k, v = W.make_qkv(w)
    o, lse = _run(q, k, v, w.causal, w.scale)
    o_ref, lse_ref = _oracle_full(oracle_mod, q, k, v, w.causal, w.scale)
    _compare(o, lse, o_ref, lse_ref, name)


@pytest.mark.parametrize("name", ["b2h16n4096d128_causal",
                                  "tradingday_b1h12n23400d64_causal",
                                  "long_b1h32n16384d128"])
def test_parity_workloads_sampled(oracle_mod, name):
    w = W.WORKLOADS[name]
    q, k, v = W.make_qkv(w)
    o, lse = _run(q, k, v, w.causal, w.scale)
    rows = np.array(W.sample_rows(w, 384))
    bits = [oracle_mod.bf16_bits(t) for t in (q, k, v)]
    o_ref, lse_ref = oracle_mod.attention_rows_bf16(*bits, w.causal, w.scale,
                                                    rows)
    _compare(o.reshape(-1, w.d)[rows], lse.reshape(-1)[rows], o_ref, lse_ref,
             name)
    # properties that hold at any size, checked on every row
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    vmax = np.abs(v.float().numpy()).max()
    assert np.abs(o).max() <= vmax * (1 + 2 ** -7)
    if w.causal:
        # row 0 of every head sees only key 0
        np.testing.assert_allclose(o[:, :, 0], v[:, :, 0].float().numpy(),
                                   atol=O_TOL)


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_gives_v(causal):
    w = W.shape_case(2, 3, 1, 128, causal, seed=3)
    q, k, v = W.make_qkv(w)
    o, lse = _run(q, k, v, causal, w.scale)
    vf = v.float().numpy()
    assert np.max(np.abs(o - vf)) <= 2 ** -8 * np.abs(vf).max()
    dots = w.scale * np.einsum("bhnd,bhnd->bhn", q.double().numpy(),
                               k.double().numpy())
    assert np.max(np.abs(lse - dots)) <= LSE_TOL


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_values(causal):
    B, H, N, d = 1, 2, 600, 64
    w = W.shape_case(B, H, N, d, causal, seed=4)
    _, k, v = W.make_qkv(w)
    q = torch.zeros_like(k)
    o, lse = _run(q, k, v, causal, w.scale)
    vd = v.double().numpy()
    if causal:
        ref = np.cumsum(vd, axis=2) / np.arange(1, N + 1).reshape(1, 1, N, 1)
        lref = np.log(np.arange(1, N + 1))
    else:
        ref = np.broadcast_to(vd.mean(axis=2, keepdims=True), vd.shape)
        lref = np.full(N, math.log(N))
    assert np.max(np.abs(o - ref)) <= O_TOL
    assert np.max(np.abs(lse - lref)) <= LSE_TOL


def test_row_shift_invariance():
    """With K[:, :, :, 0] = 1, adding c/scale to q[i, 0] adds c to every
    score of row i: O is unchanged and lse moves by c (all bf16-exact)."""
    B, H, N, d = 1, 1, 512, 64
    w = W.shape_case(B, H, N, d, False, seed=5)
    q, k, v = W.make_qkv(w)
    k[..., 0] = 1.0
    q[..., 0] = 0.0
    scale = 0.125
    o0, l0 = _run(q, k, v, False, scale)
    q2 = q.clone()
    rows = [0, 100, 511]
    q2[0, 0, rows, 0] = 64.0  # c = 64 * 0.125 = 8
    o1, l1 = _run(q2, k, v, False, scale)
    assert np.max(np.abs(o1 - o0)) <= O_TOL
    np.testing.assert_allclose(l1[0, 0, rows], l0[0, 0, rows] + 8.0,
                               atol=LSE_TOL)
    others = np.setdiff1d(np.arange(N), rows)
    assert np.array_equal(l1[0, 0, others], l0[0, 0, others])


def test_large_scores_stress_rescale(oracle_mod):
    """N(0, 2^2) queries and keys with a large scale: scores reach the
    hundreds and the running max moves many times along a row."""
    w = W.shape_case(1, 2, 2048, 128, False, seed=6, q_std=2.0, k_std=2.0)
    q, k, v = W.make_qkv(w)
    for scale in (w.scale, 1.0):
        o, lse = _run(q, k, v, False, scale)
        o_ref, lse_ref = _oracle_full(oracle_mod, q, k, v, False, scale)
        _compare(o, lse, o_ref, lse_ref, f"scale={scale}")


@pytest.mark.parametrize("H,d", [(1, 64), (80, 64), (40, 128)])
def test_increasing_scores_force_every_rescale(oracle_mod, H, d):
    """Scores that grow along the key axis make the running max rise on every
    key/value tile, exercising the output correction each iteration; with
    more heads than CTAs each CTA runs several units, so the correction also
    meets the unit boundaries (the next unit's first S and P.V against the
    previous unit's epilogue)."""
    B, N = 1, 1024
    q = torch.zeros(B, H, N, d)
    q[..., 0] = 1.0
    k = torch.zeros(B, H, N, d)
    k[..., 0] = torch.linspace(0, 400, N)
    g = torch.Generator().manual_seed(7)
    v = torch.randn(B, H, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    for causal in (False, True):
        o, lse = _run(q, k, v, causal, 1.0)
        o_ref, lse_ref = _oracle_full(oracle_mod, q, k, v, causal, 1.0)
        _compare(o, lse, o_ref, lse_ref, f"causal={causal}")


def test_deterministic_and_stream_safe():
    w = W.shape_case(2, 4, 777, 128, True, seed=8)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    o1, l1 = attn.attn_fwd(q, k, v, causal=True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = attn.attn_fwd(q, k, v, causal=True, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_outputs_do_not_leak_across_heads(oracle_mod):
    """Heads with very different value scales stay separate."""
    w = W.shape_case(2, 3, 300, 64, False, seed=9)
    q, k, v = W.make_qkv(w)
    scales = torch.tensor([1, 100, 0.01, 10, 1000, 0.1]).reshape(2, 3, 1, 1)
    v = (v.float() * scales).to(torch.bfloat16)
    o, lse = _run(q, k, v, False, w.scale)
    o_ref, lse_ref = _oracle_full(oracle_mod, q, k, v, False, w.scale)
    rel = np.abs(o - o_ref) / scales.numpy()
    assert rel.max() <= O_TOL
    assert np.max(np.abs(lse - lse_ref)) <= LSE_TOL


def test_host_buffer_entry_matches_device_entry():
    w = W.shape_case(1, 3, 1000, 128, True, seed=10)
    q, k, v = W.make_qkv(w)
    o_dev, l_dev = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    o_h = torch.empty_like(q).pin_memory()
    l_h = torch.empty(1, 3, 1000, dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.host_workspace_bytes(1, 3, 1000, 128),
                     dtype=torch.uint8, device="cuda")
    attn.attn_fwd_host(qp, kp, vp, o_h, l_h, True, w.scale, ws)
    torch.cuda.synchronize()
    assert attn.status() == 0
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(l_h, l_dev.cpu())


def test_host_buffer_entry_chunked_pipeline_matches_device_entry():
    """Large problems go through attn_fwd_host's copy / compute pipeline
    (heads in chunks on three streams); 13 heads make a ragged last chunk.
    Every head is computed by the same kernel either way, so the outputs
    match the device entry bit for bit, and work queued on the caller's
    stream afterwards sees them."""
    w = W.shape_case(1, 13, 16384, 128, False, seed=11)
    q, k, v = W.make_qkv(w)
    assert q.numel() * 2 >= 32 << 20
    o_dev, l_dev = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=False)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    o_h = torch.empty_like(q).pin_memory()
    l_h = torch.empty(1, 13, 16384, dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.host_workspace_bytes(1, 13, 16384, 128),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        attn.attn_fwd_host(qp, kp, vp, o_h, l_h, False, w.scale, ws,
                           stream=stream)
        done = torch.cuda.Event()
        done.record(stream)
    done.synchronize()
    assert attn.status() == 0
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(l_h, l_dev.cpu())


def test_device_errors_are_reported():
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    buf = torch.zeros(2 * 64 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(64, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    # misaligned output pointer
    rc = attn.attn_fwd_raw(q.data_ptr(), q.data_ptr(), q.data_ptr(),
                           buf.data_ptr() + 2, lse.data_ptr(), 1, 1, 64, 64, 0,
                           0.125, stream)
    assert rc == 4
    # host memory where device memory is required
    host = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    rc = attn.attn_fwd_raw(q.data_ptr(), q.data_ptr(), q.data_ptr(),
                           host.data_ptr(), lse.data_ptr(), 1, 1, 64, 64, 0,
                           0.125, stream)
    assert rc == 10
    assert attn.status() == 0
