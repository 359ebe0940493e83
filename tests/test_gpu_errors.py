"""Error behaviour on the GPU: invalid pointers are rejected on the host
before anything is launched or written; an inconsistent cu_seqlens array is
skipped by the kernel (no fault) and reported through the error word."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_host_pointer_is_rejected_and_nothing_written():
    import causal_linear_attention_chunked_b200 as L
    from causal_linear_attention_chunked_b200 import _binding as b
    q = torch.randn(1, 64, 2, 64).bfloat16()  # host memory
    k, v = q.clone(), q.clone()
    out = torch.full((1, 64, 2, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    st = b.lib.lt_linear_attn_fwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                  ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                  1, 2, 2, 64, 64, 64, 1, 1e-6, None, None, 1)
    assert st == b.LT_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert (out == 7.0).all()


def test_misaligned_and_overlapping_buffers_are_rejected():
    from causal_linear_attention_chunked_b200 import _binding as b
    buf = torch.zeros(4 * 64 * 2 * 64 + 64, dtype=torch.bfloat16, device="cuda")
    base = buf.data_ptr()
    P = ctypes.c_void_p
    st = b.lib.lt_linear_attn_fwd(P(base + 2), P(base), P(base), P(base + 65536), 1, 2, 2, 64,
                                  64, 64, 1, 1e-6, None, None, 1)
    assert st == b.LT_ERR_INVALID_ARG
    q = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16, device="cuda")
    st = b.lib.lt_linear_attn_fwd(P(q.data_ptr()), P(q.data_ptr()), P(q.data_ptr()),
                                  P(q.data_ptr()), 1, 2, 2, 64, 64, 64, 1, 1e-6, None, None, 1)
    assert st == b.LT_ERR_INVALID_ARG


def test_bad_cu_seqlens_reported_not_faulted():
    import causal_linear_attention_chunked_b200 as L
    from causal_linear_attention_chunked_b200 import _binding as b
    q = torch.randn(100, 2, 64, device="cuda").bfloat16()
    out = torch.zeros_like(q)
    cu = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device="cuda")  # not monotone
    L.linear_attn_fwd(q, q, q, cu_seqlens=cu, out=out)
    assert L.get_last_device_error() == b.LT_ERR_DEVICE_BAD_SEQLENS
    assert L.get_last_device_error() == 0  # read-and-clear
    cu = torch.tensor([0, 60, 100, 140], dtype=torch.int32, device="cuda")  # beyond N
    L.linear_attn_fwd(q, q, q, cu_seqlens=cu, out=out)
    assert L.get_last_device_error() == b.LT_ERR_DEVICE_BAD_SEQLENS


def test_injected_workspace_allocation_failure(monkeypatch):
    """Host-side fault injection: the stream-ordered workspace allocation
    reports failure; the call returns LT_ERR_CUDA with nothing enqueued or
    written, and the next call (injection off) runs normally."""
    from causal_linear_attention_chunked_b200 import _binding as b, inputs
    L = b
    q, k, v = inputs.make_custom(2, 8, 8, 1024, 64, 64, torch.bfloat16, 0.125, seed=3)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    assert L.linear_attn_fwd_plan(2, 8, 8, 1024, 64, 64)[2] > 0  # this shape needs a workspace
    out = torch.full((2, 1024, 8, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    monkeypatch.setenv("LT_FAULT_WORKSPACE_ALLOC", "1")
    for call in (lambda: L.linear_attn_fwd(q, k, v, out=out),
                 lambda: L.linear_attn_fwd_state(q, k, v, out=out)):
        with pytest.raises(L.LtError) as ei:
            call()
        assert ei.value.status == b.LT_ERR_CUDA
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    monkeypatch.delenv("LT_FAULT_WORKSPACE_ALLOC")
    L.linear_attn_fwd(q, k, v, out=out)
    assert L.get_last_device_error() == 0
    assert bool(torch.isfinite(out.float()).all()) and not bool((out == 7.0).all())


def test_stalled_wait_times_out_and_device_stays_usable():
    """A bounded wait on a barrier nothing arrives on gives up after its
    limit and reports LT_ERR_DEVICE_TIMEOUT; the error word is then clear and
    the device runs a forward pass normally."""
    from causal_linear_attention_chunked_b200 import _binding as b, inputs
    assert b.lib.lt_selftest_wait_timeout(20000, None) == b.LT_OK  # 20 ms
    assert b.get_last_device_error() == b.LT_ERR_DEVICE_TIMEOUT
    assert b.get_last_device_error() == b.LT_OK
    q, k, v = inputs.make_custom(1, 2, 2, 300, 64, 64, torch.bfloat16, 0.125, seed=4)
    out = b.linear_attn_fwd(q.cuda(), k.cuda(), v.cuda())
    assert b.get_last_device_error() == b.LT_OK
    assert bool(torch.isfinite(out.float()).all())
