"""Sliding-window causal attention on the GPU (lt_linear_attn_fwd_window)
against the oracle's two-state form, element by element: windows shorter
than, equal to and longer than the 32-token chunk, up to beyond the
sequence; ragged tails, GQA, every width pair, packed sequences with empty
ones; fp32, bf16 and fp16 I/O.  Bars: 1e-4 (fp32), 2e-2 (16-bit), the row
metric of the forward tests."""
import pytest
import torch

import oracle
from parity import row_rel_err, TOL_BF16, TOL_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def L():
    import causal_linear_attention_chunked_b200 as lt
    return lt


WINDOWS = [1, 5, 31, 32, 33, 64, 100, 257, 5000]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16],
                         ids=["f32", "bf16", "f16"])
@pytest.mark.parametrize("window", WINDOWS)
def test_window_dense_vs_oracle(window, dtype):
    B, Hq, Hkv, N, d = 2, 4, 2, 700, 64
    scale = 1.0 if dtype == torch.float32 else d ** -0.5
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, d, dtype, scale, seed=window)
    out = L().linear_attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), window)
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    ref = oracle.fwd_window_recurrent(q, k, v, window)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert row_rel_err(out.float().cpu().numpy(), ref) <= tol


@pytest.mark.parametrize("shape", [(1, 2, 2, 300, 128, 128), (1, 4, 1, 129, 64, 128),
                                   (1, 2, 2, 1, 128, 64)])
def test_window_widths(shape):
    B, Hq, Hkv, N, d, dv = shape
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5, seed=N)
    for window in (7, 96):
        out = L().linear_attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), window)
        torch.cuda.synchronize()
        ref = oracle.fwd_window_quadratic(q, k, v, window)
        assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16


def test_window_packed_and_causal_limit():
    lens = [500, 0, 1, 77, 33]
    cu = inputs.cu_from_lengths(lens)
    T, Hq, Hkv, d = int(cu[-1]), 4, 2, 64
    g = inputs.generator(29)
    q, k, v = ((torch.randn(sh, generator=g) * 0.125).to(torch.bfloat16) for sh in
               ((T, Hq, d), (T, Hkv, d), (T, Hkv, d)))
    for window in (16, 40):
        out = L().linear_attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), window,
                                         cu_seqlens=cu.cuda())
        torch.cuda.synchronize()
        assert L().get_last_device_error() == 0
        ref = oracle.fwd_window_recurrent(q, k, v, window, cu_seqlens=cu.numpy())
        assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16
    # a window longer than every sequence is the causal form
    out = L().linear_attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), 10000, cu_seqlens=cu.cuda())
    ref = oracle.fwd_recurrent(q, k, v, causal=True, cu_seqlens=cu.numpy())
    torch.cuda.synchronize()
    assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16
