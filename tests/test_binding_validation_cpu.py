"""The Python binding refuses tensors the C ABI would misread.

The C entry points receive bare pointers, so a wrong dtype, a non-contiguous
view or a mismatched shape cannot be seen below the binding.  Every wrapper
checks its tensors before it calls into the library; these checks run on the
CPU (host tensors stand in where a CUDA tensor is required, which the
wrapper refuses by device before anything else).
"""
import pytest
import torch

from exact_io_aware_73_b200 import attn


def _qkv(B=1, H=2, N=8, d=64, dtype=torch.bfloat16):
    return [torch.zeros(B, H, N, d, dtype=dtype) for _ in range(3)]


def test_device_entries_refuse_host_tensors():
    q, k, v = _qkv()
    with pytest.raises(TypeError, match="CUDA"):
        attn.attn_fwd(q, k, v)
    lse = torch.zeros(1, 2, 8)
    with pytest.raises(TypeError, match="CUDA"):
        attn.attn_bwd(q, k, v, q.clone(), lse, q.clone())
    with pytest.raises(TypeError, match="CUDA"):
        attn.attn_fwd_fp8(q, k, v)
    with pytest.raises(TypeError, match="CUDA"):
        attn.fp8_quantize(q, rotate=False)
    with pytest.raises(TypeError, match="CUDA"):
        attn.attn_decode(q[:, :, :1], k, v)
    with pytest.raises(TypeError, match="CUDA"):
        attn.attn_fwd_merge(q, k, v, torch.zeros(q.shape), lse, attn.MERGE_FIRST)
    with pytest.raises(TypeError, match="CUDA"):
        attn.merge_fold(torch.zeros(16, 64), torch.zeros(16),
                        torch.zeros(16, 64, dtype=torch.bfloat16), torch.zeros(16),
                        first=True)
    with pytest.raises(TypeError, match="CUDA"):
        attn.merge_finish(torch.zeros(16, 64), torch.zeros(16))
    with pytest.raises(TypeError, match="CUDA"):
        attn.attn_fwd_fp8_quantized(*(torch.zeros(1, 1, 8, 128, dtype=torch.uint8),
                                      torch.zeros(1, 1, 1)) * 2,
                                    torch.zeros(1, 1, 8, 128, dtype=torch.uint8),
                                    torch.zeros(1, 1), causal=False, scale=0.1)


def test_host_entries_check_dtype_layout_and_shape():
    q, k, v = _qkv()
    out = torch.zeros_like(q)
    lse = torch.zeros(1, 2, 8)
    ws = torch.zeros(16, dtype=torch.uint8)  # a host tensor: refused, needs CUDA
    # wrong dtype of an input
    with pytest.raises(TypeError, match="k must be"):
        attn.attn_fwd_host(q, k.float(), v, out, lse, False, 0.125, ws)
    # non-contiguous view of the right shape (every other column)
    k_strided = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)[..., ::2]
    assert k_strided.shape == k.shape and not k_strided.is_contiguous()
    with pytest.raises(ValueError, match="contiguous"):
        attn.attn_fwd_host(q, k_strided, v, out, lse, False, 0.125, ws)
    # shape mismatch
    with pytest.raises(ValueError, match="shape"):
        attn.attn_fwd_host(q, k[:, :, :4].contiguous(), v, out, lse, False, 0.125, ws)
    # lse of the wrong shape
    with pytest.raises(ValueError, match="lse"):
        attn.attn_fwd_host(q, k, v, out, torch.zeros(1, 2, 7), False, 0.125, ws)
    # output of the wrong dtype
    with pytest.raises(TypeError, match="out"):
        attn.attn_fwd_host(q, k, v, out.float(), lse, False, 0.125, ws)
    # the device workspace must be a CUDA tensor
    with pytest.raises(TypeError, match="workspace"):
        attn.attn_fwd_host(q, k, v, out, lse, False, 0.125, ws)
    # the allocation-free entry checks the same host tensors
    with pytest.raises(TypeError, match="v must be"):
        attn.attn_fwd_host_noalloc(q, k, v.half(), out, lse, False, 0.125)
    with pytest.raises(ValueError, match="q must be 4-D"):
        attn.attn_fwd_host_noalloc(q[0], k[0], v[0], out, lse, False, 0.125)


def test_expect_helper_contract():
    t = torch.zeros(2, 3, dtype=torch.float32)
    attn._expect("t", t, torch.float32, (2, 3), cuda=False)
    with pytest.raises(TypeError):
        attn._expect("t", t, torch.bfloat16, cuda=False)
    with pytest.raises(ValueError, match="shape"):
        attn._expect("t", t, torch.float32, (3, 2), cuda=False)
    with pytest.raises(ValueError, match="contiguous"):
        attn._expect("t", t.t(), torch.float32, cuda=False)
    with pytest.raises(TypeError):
        attn._expect("t", [1, 2], torch.float32, cuda=False)
