"""GPU checks at sizes far beyond what the oracle computes: long sequences,
very many heads, tensors of more than 2^32 elements, and decode at the
largest key count the library accepts.

Inputs are "needles".  Every query is 64 e_0, every key is zero except a few
planted rows k_t = a_t e_0, and the scale is 1/8, so query i scores exactly
8 a_t against a planted key and 0 against the rest.  With the planted
scores 256, 384 and 512, every other key's weight exp(s - max) underflows
to exactly 0, so softmax is one-hot on the highest planted key a row sees:
O_i = V_t and lse_i = 8 a_t, closed forms at any size (the definition of
attention restated for one-hot weights; no oracle call).  Placing the
planted keys in the ragged last tile, on tile boundaries and just beyond a
causal row's horizon checks that every key tile is visited and the mask
holds at these sizes.

Tolerances: O is V_t divided by the row sum l = 2^r with |r| <= 2^-12 (the
score passes through an fma residual before the exponential), then rounded
to bf16, so |O - V_t| <= 2^-8 |V_t|; lse within 5e-3 as everywhere.  The
backward check is on dV alone: with one-hot weights dV_t is the sum of dO
over the rows whose weight sits on key t, and every other row of dV is
exactly 0.  (dQ and dK vanish in exact arithmetic here, but the kernel's
D = rowsum(dO o O) uses the bf16-rounded O, and that rounding adds up
coherently over a million rows, so they are not checked against 0.)
"""
import numpy as np
import pytest
import torch

from exact_io_aware_73_b200 import attn

pytestmark = pytest.mark.gpu

SCALE = 0.125   # 1/8 for every d here, so scores are exact multiples of 8
QV = 64.0       # every query is QV * e_0


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs a B200 (sm_100)")
    attn.lib()
    yield
    torch.cuda.empty_cache()
    assert attn.status() == 0


def _randn_bf16(shape, seed, chunk_rows=1 << 22):
    """Seeded N(0, 1) bf16 tensor on the device, made in row chunks so that
    the fp32 intermediate stays small."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    flat = out.view(-1, shape[-1])
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        flat[r0:r1] = torch.randn((r1 - r0, shape[-1]), generator=g, device="cuda",
                                  dtype=torch.float32).to(torch.bfloat16)
    return out


def _needle_inputs(BH, N, d, t2, seed):
    """q = QV e_0 for every row; k zero except k[h, 0] = 32 e_0 (score 256,
    seen by every row) and k[h, t2[h]] = 64 e_0 (score 512); v ~ N(0, 1)."""
    q = torch.zeros((BH, N, d), dtype=torch.bfloat16, device="cuda")
    q[:, :, 0] = QV
    k = torch.zeros_like(q)
    k[:, 0, 0] = 32.0
    k[torch.arange(BH, device="cuda"), t2, 0] = 64.0
    v = _randn_bf16((BH, N, d), seed)
    return q, k, v


def _check_needle_outputs(o, lse, v, t2, causal, rows_per_chunk=1 << 21):
    """O[h, i] = v[h, t(h, i)], lse = 512 where row i sees t2[h], else
    v[h, 0] and 256; checked on every row, a chunk of heads at a time."""
    BH, N, d = v.shape
    i = torch.arange(N, device="cuda")
    hc = max(1, rows_per_chunk // N)
    worst_o, worst_l = 0.0, 0.0
    for h0 in range(0, BH, hc):
        h1 = min(BH, h0 + hc)
        tt = t2[h0:h1]
        sees = (i[None, :] >= tt[:, None]) if causal else torch.ones(
            (h1 - h0, N), dtype=torch.bool, device="cuda")
        vt2 = v[torch.arange(h0, h1, device="cuda"), tt].float()      # [h, d]
        v0 = v[h0:h1, 0].float()
        want = torch.where(sees[:, :, None], vt2[:, None, :], v0[:, None, :])
        err = (o[h0:h1].float() - want).abs()
        bound = 2.0 ** -8 * want.abs() + 1e-6
        assert bool((err <= bound).all()), \
            f"heads {h0}..{h1}: max |O - V_t| {err.max().item():.3e}"
        worst_o = max(worst_o, float(err.max()))
        lwant = torch.where(sees, 512.0, 256.0)
        lerr = float((lse[h0:h1] - lwant).abs().max())
        assert lerr <= 5e-3, f"heads {h0}..{h1}: max |lse - 8 a_t| {lerr:.3e}"
        worst_l = max(worst_l, lerr)
    return worst_o, worst_l


# (B*H, N, d, causal, where the 512 needle sits)
LONG_CASES = [
    (1, (1 << 20) + 77, 64, False, "last"),       # ragged last tile
    (1, (1 << 21) + 77, 64, True, "boundary"),    # mid-sequence tile boundary
    (2, (1 << 19) + 77, 128, False, "last"),
    (2, (1 << 19) + 77, 128, True, "boundary"),
    # 8192 heads x 4173 rows x 128: 4.4e9 elements per tensor, > 2^32
    (8192, 4096 + 77, 128, False, "spread"),
    (8192, 4096 + 77, 128, True, "spread"),
]


def _t2(BH, N, where):
    if where == "last":
        t = [N - 1] * BH
    elif where == "boundary":
        t = [128 * (N // 256) + 128 * h for h in range(BH)]
    else:  # a different position per head, including both ends and boundaries
        rng = np.random.default_rng(BH + N)
        t = rng.integers(1, N, size=BH)
        t[:4] = [1, N - 1, 128, 256]
    return torch.as_tensor(np.asarray(t, dtype=np.int64), device="cuda")


@pytest.mark.parametrize("BH,N,d,causal,where", LONG_CASES)
def test_forward_needles_long_and_huge(BH, N, d, causal, where):
    t2 = _t2(BH, N, where)
    q, k, v = _needle_inputs(BH, N, d, t2, seed=BH + N + d)
    o, lse = attn.attn_fwd(q.view(1, BH, N, d), k.view(1, BH, N, d),
                           v.view(1, BH, N, d), causal=causal, scale=SCALE)
    assert attn.status() == 0
    e = _check_needle_outputs(o.view(BH, N, d), lse.view(BH, N), v, t2, causal)
    print(f"BH={BH} N={N} d={d} causal={causal}: max|O-V_t| {e[0]:.2e}, "
          f"max|dlse| {e[1]:.2e}")


def test_forward_at_maximum_head_count():
    """B*H = 2^24 heads (the library's limit) of one row each: O = V and
    lse = scale q.k exactly in exact arithmetic (one key), every head."""
    B, H, N, d = 4096, 4096, 1, 64
    BH = B * H
    q = _randn_bf16((BH, N, d), 11)
    k = _randn_bf16((BH, N, d), 12)
    v = _randn_bf16((BH, N, d), 13)
    o, lse = attn.attn_fwd(q.view(B, H, N, d), k.view(B, H, N, d),
                           v.view(B, H, N, d), causal=True, scale=SCALE)
    assert attn.status() == 0
    for h0 in range(0, BH, 1 << 22):
        sl = slice(h0, h0 + (1 << 22))
        err = (o.view(BH, N, d)[sl].float() - v[sl].float()).abs()
        assert bool((err <= 2.0 ** -8 * v[sl].float().abs() + 1e-6).all())
    # lse = scale * q.k, checked on the host in fp64 on spread heads
    idx = np.unique(np.r_[0, 1, BH - 1, np.random.default_rng(5).integers(0, BH, 4093)])
    it = torch.as_tensor(idx, device="cuda")
    qh, kh = (t[it, 0].double().cpu().numpy() for t in (q, k))
    want = SCALE * np.einsum("hd,hd->h", qh, kh)
    got = lse.view(BH)[it].cpu().numpy()
    assert np.abs(got - want).max() <= 5e-3


def _decode_with(kernel, *args, **kw):
    """attn_decode on the given kernel (1 CUDA cores, 2 tensor cores)."""
    attn.set_decode_kernel(kernel)
    try:
        return attn.attn_decode(*args, **kw)
    finally:
        attn.set_decode_kernel(0)


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("causal", [False, True])
def test_decode_needles_at_maximum_key_count(causal, kernel):
    """Nk = 2^26 keys (the library's limit), d = 64: K and V are 8.6 GB
    each.  Planted scores 256 (key 0), 384 (key 2^25, a tile boundary) and
    512 (the last key): with the causal mask only the last of the 4 queries
    sees the last key.  Both decode kernels."""
    B, H, Nq, Nk, d = 1, 1, 4, 1 << 26, 64
    q = torch.zeros((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    q[..., 0] = QV
    k = torch.zeros((B, H, Nk, d), dtype=torch.bfloat16, device="cuda")
    marks = {0: 32.0, 1 << 25: 48.0, Nk - 1: 64.0}
    for t, a in marks.items():
        k[0, 0, t, 0] = a
    v = _randn_bf16((B, H, Nk, d), 21)
    o, lse = _decode_with(kernel, q, k, v, causal=causal, scale=SCALE)
    assert attn.status() == 0
    o, lse = o.float().cpu().numpy()[0, 0], lse.cpu().numpy()[0, 0]
    for i in range(Nq):
        horizon = Nk - Nq + i if causal else Nk - 1
        t = max(tt for tt in marks if tt <= horizon)
        vt = v[0, 0, t].float().cpu().numpy()
        assert np.all(np.abs(o[i] - vt) <= 2.0 ** -8 * np.abs(vt) + 1e-6), (i, t)
        assert abs(lse[i] - 8.0 * marks[t]) <= 5e-3, (i, t, lse[i])
    del k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("causal", [False, True])
def test_backward_needles_long(causal):
    """N = 2^20 + 77, d = 64: dV_t = sum of dO over the rows whose weight
    sits on key t (fp64 sums on the host); every other row of dV is 0 up to
    the floor of the FMA-pipe exponential: it clamps its argument at -125,
    so a score far below its row's maximum still weighs 2^-125 instead of
    underflowing to 0, and such a row of dV sums at most N of those times
    |dO| (below 2^-100 here)."""
    BH, N, d = 1, (1 << 20) + 77, 64
    t2v = 128 * 4096
    t2 = torch.tensor([t2v], device="cuda")
    q, k, v = _needle_inputs(BH, N, d, t2, seed=31)
    shape = (1, BH, N, d)
    q, k, v = (x.view(shape) for x in (q, k, v))
    o, lse = attn.attn_fwd(q, k, v, causal=causal, scale=SCALE)
    do = _randn_bf16(shape, 32)
    dq, dk, dv = attn.attn_bwd(q, k, v, o, lse, do, causal=causal, scale=SCALE)
    assert attn.status() == 0
    dof = do[0, 0].double().cpu().numpy()
    if causal:
        want = {0: dof[:t2v].sum(axis=0), t2v: dof[t2v:].sum(axis=0)}
    else:
        want = {0: np.zeros(d), t2v: dof.sum(axis=0)}
    dvh = dv[0, 0].float().cpu().numpy()
    for t, w in want.items():
        count = t2v if (causal and t == 0) else N
        bound = 2.0 ** -8 * np.abs(w) + 1e-3 * np.sqrt(count)
        assert np.all(np.abs(dvh[t] - w) <= bound), (t, np.abs(dvh[t] - w).max())
    others = np.ones(N, dtype=bool)
    others[[0, t2v]] = False
    assert np.all(np.abs(dvh[others]) <= 2.0 ** -100)
    assert np.all(np.isfinite(dq.float().cpu().numpy()))
    assert np.all(np.isfinite(dk.float().cpu().numpy()))


def test_decode_query_groups_at_maximum_key_count():
    """13 queries on the CUDA-core kernel (four launches of up to 4, the last
    ragged) against 2^26 keys under the causal mask: query i sees keys up to
    Nk - 13 + i.  Planted
    scores 256 (key 0), 384 (key 2^25) and 512 (key Nk - 8, seen by queries
    5 and later only), so a group's key limit or its query offset being wrong
    shows in whole rows."""
    B, H, Nq, Nk, d = 1, 1, 13, 1 << 26, 64
    q = torch.zeros((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    q[..., 0] = QV
    k = torch.zeros((B, H, Nk, d), dtype=torch.bfloat16, device="cuda")
    marks = {0: 32.0, 1 << 25: 48.0, Nk - 8: 64.0}
    for t, a in marks.items():
        k[0, 0, t, 0] = a
    v = _randn_bf16((B, H, Nk, d), 22)
    o, lse = _decode_with(1, q, k, v, causal=True, scale=SCALE)
    assert attn.status() == 0
    o, lse = o.float().cpu().numpy()[0, 0], lse.cpu().numpy()[0, 0]
    for i in range(Nq):
        t = max(tt for tt in marks if tt <= Nk - Nq + i)
        assert (t == Nk - 8) == (i >= 5)
        vt = v[0, 0, t].float().cpu().numpy()
        assert np.all(np.abs(o[i] - vt) <= 2.0 ** -8 * np.abs(vt) + 1e-6), (i, t)
        assert abs(lse[i] - 8.0 * marks[t]) <= 5e-3, (i, t, lse[i])
    del k, v
    torch.cuda.empty_cache()


def test_decode_tensor_core_queries_at_maximum_key_count():
    """13 causal queries at d = 128 (one tensor-core launch) against 2^26
    keys: the same planted scores as the grouped test, so query i's output
    is the value of the highest planted key it sees, in closed form."""
    B, H, Nq, Nk, d = 1, 1, 13, 1 << 26, 128
    q = torch.zeros((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    q[..., 0] = QV
    k = torch.zeros((B, H, Nk, d), dtype=torch.bfloat16, device="cuda")
    marks = {0: 32.0, 1 << 25: 48.0, Nk - 8: 64.0}
    for t, a in marks.items():
        k[0, 0, t, 0] = a
    v = _randn_bf16((B, H, Nk, d), 23)
    o, lse = _decode_with(2, q, k, v, causal=True, scale=SCALE)
    assert attn.status() == 0
    o, lse = o.float().cpu().numpy()[0, 0], lse.cpu().numpy()[0, 0]
    for i in range(Nq):
        t = max(tt for tt in marks if tt <= Nk - Nq + i)
        assert (t == Nk - 8) == (i >= 5)
        vt = v[0, 0, t].float().cpu().numpy()
        assert np.all(np.abs(o[i] - vt) <= 2.0 ** -8 * np.abs(vt) + 1e-6), (i, t)
        assert abs(lse[i] - 8.0 * marks[t]) <= 5e-3, (i, t, lse[i])
    del k, v
    torch.cuda.empty_cache()
