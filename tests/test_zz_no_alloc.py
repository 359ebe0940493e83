"""lt_linear_attn_fwd_noalloc through the C ABI.

The no-allocation entry point serves callers that cannot let a library
allocate device memory: a program that hands all device memory to its own
caching allocator at start-up, a set-up without stream-ordered allocation,
or code that must keep a fixed footprint with no allocator work in its launch
path.  It keeps the per-block partial states in a fixed array inside the
library instead of a stream-ordered workspace, and runs the very kernels of
lt_linear_attn_fwd in the same order: its outputs must equal that entry
point's bit for bit, call after call, although every call reuses (and
overwrites) the same array.  One case is also checked against the oracle.

The file name sorts last so that a run stopping at the first failure has run
every other test before these.
"""
import ctypes

import pytest
import torch

import oracle
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


CASES = [
    # (B, Hq, Hkv, N, d, dv), causal: each cuts its sequences into several
    # blocks, so each call writes and reads the fixed array
    ((2, 8, 8, 4096, 64, 64), True),   # one cooperative launch
    ((2, 8, 8, 8192, 64, 64), True),   # two launches
    ((1, 8, 2, 3000, 128, 128), False),
    ((1, 4, 2, 2000, 128, 64), True),
]


def test_noalloc_equals_allocating_entry_point_on_consecutive_calls(sched):
    import causal_linear_attention_chunked_b200 as L
    outs = []
    for i, (shape, causal) in enumerate(CASES):
        B, Hq, Hkv, N, d, dv = shape
        nb, _, ws = L.linear_attn_fwd_plan(B, Hq, Hkv, N, d, dv, causal=causal)
        assert nb > 1 and ws > 0  # the case really uses the scratch array
        q, k, v = _case(B, Hq, Hkv, N, d, dv, seed=100 + i)
        out = torch.full((B, N, Hq, dv), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(q, k, v, out, causal) == 0
        outs.append((q, k, v, causal, out))
    # a second round in reverse order: every call finds the array holding
    # another call's partial states
    again = []
    for q, k, v, causal, _ in reversed(outs):
        out = torch.full(q.shape[:3] + (v.shape[3],), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
        assert _noalloc(q, k, v, out, causal) == 0
        again.append(out)
    again.reverse()
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    for (q, k, v, causal, out), out2 in zip(outs, again):
        ref = L.linear_attn_fwd(q, k, v, causal=causal, eps=1e-6)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        assert torch.equal(out2, ref)


def test_noalloc_matches_the_oracle():
    B, Hq, Hkv, N, d, dv = 2, 8, 8, 4096, 64, 64
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, 0.125, seed=77)
    out = torch.empty((B, N, Hq, dv), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(q.cuda(), k.cuda(), v.cuda(), out, True) == 0
    torch.cuda.synchronize()
    ref = oracle.fwd_recurrent(q, k, v, causal=True, eps=1e-6)
    assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16


def test_noalloc_rejects_shapes_beyond_the_scratch_array(sched):
    """Forcing 64 blocks on 16 (sequence, KV head) lanes of d = dv = 128
    needs 16 * 64 * (128*128 + 128) * 4 bytes = 67.6 MB, more than the 16 MiB
    array: the call is refused before anything is enqueued and the output
    stays untouched; the next call that fits still runs."""
    from causal_linear_attention_chunked_b200 import _binding as b
    import causal_linear_attention_chunked_b200 as L
    sched(blocks=64)
    q, k, v = _case(1, 16, 16, 8192, 128, 128, seed=7)
    out = torch.full((1, 8192, 16, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(q, k, v, out, True) == b.LT_ERR_SCRATCH_TOO_SMALL
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    sched(blocks=4)
    assert _noalloc(q, k, v, out, True) == 0
    ref = L.linear_attn_fwd(q, k, v, causal=True, eps=1e-6)
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    assert torch.equal(out, ref)
