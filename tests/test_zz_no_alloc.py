"""lt_linear_attn_fwd_noalloc through the C ABI, against lt_linear_attn_fwd.

The no-allocation entry point serves callers that cannot let a library
allocate device memory (memory handed to their own allocator up front, no
stream-ordered allocation, a fixed footprint): it keeps the per-block partial
states in a fixed array inside the library instead of a stream-ordered
workspace.  Its results must match the allocating entry point within the bf16
tolerance, call after call, although every call reuses the same array.

The file name sorts last so that a run stopping at the first failure has run
every other test before these.
"""
import ctypes

import pytest
import torch

from parity import row_rel_err, TOL_BF16
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def _noalloc(q, k, v, out, causal, eps=1e-6):
    from causal_linear_attention_chunked_b200 import _binding as b
    B, N, Hq, d = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return b.lib.lt_linear_attn_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        B, Hq, Hkv, N, d, dv, int(causal), float(eps), None, stream)


def _case(B, Hq, Hkv, N, d, dv, seed):
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5, seed=seed)
    return q.cuda(), k.cuda(), v.cuda()


def test_noalloc_matches_allocating_entry_point_on_consecutive_calls(monkeypatch):
    import causal_linear_attention_chunked_b200 as L
    monkeypatch.delenv("LT_BLOCKS", raising=False)
    monkeypatch.delenv("LT_KERNEL", raising=False)
    cases = [
        # (B, Hq, Hkv, N, d, dv, causal): each cuts its sequences into
        # several blocks, so each call writes and reads the fixed array
        ((2, 8, 8, 4096, 64, 64), True),   # one cooperative launch
        ((2, 8, 8, 8192, 64, 64), True),   # two launches
        ((1, 8, 2, 3000, 128, 128), False),
        ((1, 4, 2, 2000, 128, 64), True),
    ]
    outs = []
    for i, (shape, causal) in enumerate(cases):
        B, Hq, Hkv, N, d, dv = shape
        nb, _, ws = L.linear_attn_fwd_plan(B, Hq, Hkv, N, d, dv, causal=causal)
        assert nb > 1 and ws > 0  # the case really uses the scratch array
        q, k, v = _case(B, Hq, Hkv, N, d, dv, seed=100 + i)
        out = torch.full((B, N, Hq, dv), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(q, k, v, out, causal) == 0
        outs.append((q, k, v, causal, out))
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    for q, k, v, causal, out in outs:
        ref = L.linear_attn_fwd(q, k, v, causal=causal, eps=1e-6)
        torch.cuda.synchronize()
        err = row_rel_err(out.float().cpu().numpy(), ref.float().cpu().numpy())
        assert err <= TOL_BF16, err


def test_noalloc_rejects_shapes_beyond_the_scratch_array(monkeypatch):
    """Forcing 64 blocks on 16 (sequence, KV head) lanes of d = dv = 128
    needs 16 * 64 * (128*128 + 128) * 4 bytes = 67.6 MB, more than the 16 MiB
    array: the call is refused before anything is enqueued and the output
    stays untouched; the next call that fits still runs."""
    from causal_linear_attention_chunked_b200 import _binding as b
    monkeypatch.setenv("LT_BLOCKS", "64")
    q, k, v = _case(1, 16, 16, 8192, 128, 128, seed=7)
    out = torch.full((1, 8192, 16, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(q, k, v, out, True) == b.LT_ERR_SCRATCH_TOO_SMALL
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    monkeypatch.setenv("LT_BLOCKS", "4")
    assert _noalloc(q, k, v, out, True) == 0
    import causal_linear_attention_chunked_b200 as L
    ref = L.linear_attn_fwd(q, k, v, causal=True, eps=1e-6)
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    assert row_rel_err(out.float().cpu().numpy(), ref.float().cpu().numpy()) <= TOL_BF16
