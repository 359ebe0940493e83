"""ctypes binding of liblt.so (the C ABI in include/lt_linear_attn.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch supplies device memory and the current stream.  Importing
this module loads the library; a missing library is an error (there is no
fallback path).
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblt.so")

LT_OK, LT_ERR_INVALID_ARG, LT_ERR_UNSUPPORTED, LT_ERR_CUDA = 0, 1, 2, 3
LT_ERR_DEVICE_TIMEOUT, LT_ERR_DEVICE_BAD_SEQLENS, LT_ERR_SCRATCH_TOO_SMALL = 4, 5, 6
LT_F32, LT_BF16, LT_F16 = 0, 1, 2
FEATURE_MAPS = {"elu1": 0, "relu": 1, "exp": 2}
LT_SCHED_AUTO, LT_SCHED_TWO_LAUNCH, LT_SCHED_GENERAL = 0, 1, 2
_SCHED = {"auto": LT_SCHED_AUTO, "two_launch": LT_SCHED_TWO_LAUNCH, "general": LT_SCHED_GENERAL}

# every entry point declared in include/lt_linear_attn.h
EXPORTED = ("lt_linear_attn_fwd", "lt_linear_attn_fwd_noalloc", "lt_linear_attn_fwd_plan",
            "lt_linear_attn_fwd_state", "lt_linear_attn_decode_step", "lt_status_string",
            "lt_get_last_device_error", "lt_abi_version", "lt_selftest_wait_timeout",
            "lt_debug_set_schedule", "lt_linear_attn_state", "lt_linear_attn_state_carry",
            "lt_linear_attn_bwd", "lt_linear_attn_fwd_ex", "lt_linear_attn_fwd_window")

if not os.path.exists(LIB_PATH):
    raise ImportError("liblt.so is not built (run `python -m "
                      "causal_linear_attention_chunked_b200.build`)")
lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
lib.lt_linear_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _vp,
                                   _i]
lib.lt_linear_attn_fwd.restype = _i
lib.lt_linear_attn_fwd_ex.argtypes = lib.lt_linear_attn_fwd.argtypes + [_i]
lib.lt_linear_attn_fwd_ex.restype = _i
lib.lt_linear_attn_fwd_window.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                                          _vp, _vp, _i]
lib.lt_linear_attn_fwd_window.restype = _i
lib.lt_linear_attn_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                                           _vp, _vp]
lib.lt_linear_attn_fwd_noalloc.restype = _i
lib.lt_linear_attn_fwd_plan.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                        ctypes.POINTER(_i), ctypes.POINTER(_i),
                                        ctypes.POINTER(ctypes.c_size_t)]
lib.lt_linear_attn_fwd_plan.restype = _i
lib.lt_linear_attn_fwd_state.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp,
                                         _vp, _vp, _vp, _vp, _vp, _i]
lib.lt_linear_attn_fwd_state.restype = _i
lib.lt_linear_attn_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f,
                                           _vp, _i]
lib.lt_linear_attn_decode_step.restype = _i
lib.lt_status_string.argtypes = [_i]
lib.lt_status_string.restype = ctypes.c_char_p
lib.lt_get_last_device_error.argtypes = [_vp]
lib.lt_get_last_device_error.restype = _i
lib.lt_abi_version.restype = _i
lib.lt_selftest_wait_timeout.argtypes = [ctypes.c_uint, _vp]
lib.lt_selftest_wait_timeout.restype = _i
lib.lt_linear_attn_state.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _i]
lib.lt_linear_attn_state.restype = _i
lib.lt_linear_attn_state_carry.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]
lib.lt_linear_attn_state_carry.restype = _i
lib.lt_linear_attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                   _f, _vp, _vp, _i]
lib.lt_linear_attn_bwd.restype = _i
lib.lt_debug_set_schedule.argtypes = [_i, _i]
lib.lt_debug_set_schedule.restype = _i


class LtError(RuntimeError):
    def __init__(self, status):
        self.status = status
        super().__init__(lib.lt_status_string(status).decode())


def _check(status):
    if status != LT_OK:
        raise LtError(status)


def _dtype_code(t):
    if t == torch.bfloat16:
        return LT_BF16
    if t == torch.float32:
        return LT_F32
    if t == torch.float16:
        return LT_F16
    raise TypeError("unsupported dtype %s (bfloat16, float16 or float32)" % t)


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def linear_attn_fwd(q, k, v, causal=True, eps=1e-6, cu_seqlens=None, out=None, stream=None,
                    feature_map="elu1"):
    """O = linear attention of (q, k, v); see include/lt_linear_attn.h.

    Dense: q [B, N, H_q, d], k [B, N, H_kv, d], v [B, N, H_kv, dv].
    Packed: q [N, H_q, d] ... with cu_seqlens (int32, device, B+1 entries).
    dtype bfloat16, float16 or float32.  feature_map: "elu1" (ELU + 1, the
    method's), "relu" or "exp" (lt_linear_attn_fwd_ex).
    Returns out with q's dtype, shape [..., H_q, dv].
    """
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv, dv = k.shape[2], v.shape[3]
        oshape = (B, N, Hq, dv)
    else:
        N, Hq, d = q.shape
        Hkv, dv = k.shape[1], v.shape[2]
        B = cu_seqlens.numel() - 1
        oshape = (N, Hq, dv)
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
            raise TypeError("cu_seqlens must be a contiguous int32 tensor")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    if out is None:
        out = torch.empty(oshape, dtype=q.dtype, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, Hq, Hkv, N, d, dv, int(bool(causal)),
            float(eps), _ptr(cu_seqlens), _stream_handle(stream, q.device), _dtype_code(q.dtype))
    if feature_map == "elu1":
        _check(lib.lt_linear_attn_fwd(*args))
    else:
        _check(lib.lt_linear_attn_fwd_ex(*args, FEATURE_MAPS[feature_map]))
    return out


def linear_attn_fwd_window(q, k, v, window, eps=1e-6, cu_seqlens=None, out=None, stream=None):
    """Sliding-window causal linear attention: row i attends to keys
    i - window < j <= i.  See lt_linear_attn_fwd_window."""
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv, dv = k.shape[2], v.shape[3]
        oshape = (B, N, Hq, dv)
    else:
        N, Hq, d = q.shape
        Hkv, dv = k.shape[1], v.shape[2]
        B = cu_seqlens.numel() - 1
        oshape = (N, Hq, dv)
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
            raise TypeError("cu_seqlens must be a contiguous int32 tensor")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    if out is None:
        out = torch.empty(oshape, dtype=q.dtype, device=q.device)
    _check(lib.lt_linear_attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, Hq, Hkv, N, d,
                                         dv, int(window), float(eps), _ptr(cu_seqlens),
                                         _stream_handle(stream, q.device), _dtype_code(q.dtype)))
    return out


def linear_attn_fwd_state(q, k, v, causal=True, eps=1e-6, cu_seqlens=None, S0=None, z0=None,
                          return_state=True, out=None, S_out=None, z_out=None, stream=None):
    """linear_attn_fwd continued from the state (S0, z0) (None: zero) and,
    with return_state, also returning the final state: (out, S, z), states
    fp32 [sequences, H_kv, d, dv] and [sequences, H_kv, d] (the layout of
    linear_attn_decode_step), written into S_out/z_out when given.  See
    lt_linear_attn_fwd_state in include/lt_linear_attn.h."""
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv, dv = k.shape[2], v.shape[3]
        oshape = (B, N, Hq, dv)
    else:
        N, Hq, d = q.shape
        Hkv, dv = k.shape[1], v.shape[2]
        B = cu_seqlens.numel() - 1
        oshape = (N, Hq, dv)
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
            raise TypeError("cu_seqlens must be a contiguous int32 tensor")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    for t in (S0, z0):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise TypeError("S0 and z0 must be contiguous float32 tensors")
    if out is None:
        out = torch.empty(oshape, dtype=q.dtype, device=q.device)
    S = z = None
    if return_state:
        S = S_out if S_out is not None else torch.empty((B, Hkv, d, dv), dtype=torch.float32,
                                                        device=q.device)
        z = z_out if z_out is not None else torch.empty((B, Hkv, d), dtype=torch.float32,
                                                        device=q.device)
    _check(lib.lt_linear_attn_fwd_state(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, Hq, Hkv, N, d,
                                        dv, int(bool(causal)), float(eps), _ptr(cu_seqlens),
                                        _ptr(S0), _ptr(z0), _ptr(S), _ptr(z),
                                        _stream_handle(stream, q.device), _dtype_code(q.dtype)))
    return (out, S, z) if return_state else out


def linear_attn_bwd(q, k, v, dout, causal=True, eps=1e-6, cu_seqlens=None, dq=None, dk=None,
                    dv=None, stream=None):
    """Gradients (dq, dk, dv) of linear attention for the upstream gradient
    dout (the output's shape and dtype).  See lt_linear_attn_bwd in
    include/lt_linear_attn.h."""
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv, dvw = k.shape[2], v.shape[3]
    else:
        N, Hq, d = q.shape
        Hkv, dvw = k.shape[1], v.shape[2]
        B = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
            raise TypeError("cu_seqlens must be a contiguous int32 tensor")
    for t in (q, k, v, dout):
        if not t.is_contiguous():
            raise ValueError("q, k, v, dout must be contiguous")
    if dout.dtype != q.dtype:
        raise TypeError("dout must have q's dtype")
    dq = dq if dq is not None else torch.empty_like(q)
    dk = dk if dk is not None else torch.empty_like(k)
    dv = dv if dv is not None else torch.empty_like(v)
    _check(lib.lt_linear_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                  _ptr(dv), B, Hq, Hkv, N, d, dvw, int(bool(causal)), float(eps),
                                  _ptr(cu_seqlens), _stream_handle(stream, q.device),
                                  _dtype_code(q.dtype)))
    return dq, dk, dv


def linear_attn_state(k, v, cu_seqlens=None, S0=None, z0=None, S_out=None, z_out=None,
                      stream=None):
    """The final state of every (sequence, KV head) without the outputs:
    (S, z) = (S0, z0) + sum over the sequence of phi(K_t)^T V_t and phi(K_t);
    fp32 [sequences, H_kv, d, dv] and [sequences, H_kv, d].  k, v as for
    linear_attn_fwd.  See lt_linear_attn_state in include/lt_linear_attn.h."""
    if cu_seqlens is None:
        B, N, Hkv, d = k.shape
        dv = v.shape[3]
    else:
        N, Hkv, d = k.shape
        dv = v.shape[2]
        B = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
            raise TypeError("cu_seqlens must be a contiguous int32 tensor")
    for t in (k, v):
        if not t.is_contiguous():
            raise ValueError("k, v must be contiguous")
    for t in (S0, z0):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise TypeError("S0 and z0 must be contiguous float32 tensors")
    S = S_out if S_out is not None else torch.empty((B, Hkv, d, dv), dtype=torch.float32,
                                                    device=k.device)
    z = z_out if z_out is not None else torch.empty((B, Hkv, d), dtype=torch.float32,
                                                    device=k.device)
    _check(lib.lt_linear_attn_state(_ptr(k), _ptr(v), B, Hkv, N, d, dv, _ptr(cu_seqlens), _ptr(S0),
                                    _ptr(z0), _ptr(S), _ptr(z), _stream_handle(stream, k.device),
                                    _dtype_code(k.dtype)))
    return S, z


def linear_attn_state_carry(S_all, z_all, rank, causal=True, S_out=None, z_out=None,
                            stream=None):
    """Segment `rank`'s starting state from every segment's state S_all
    [world, B, H_kv, d, dv], z_all [world, B, H_kv, d] (fp32): the sum over
    the earlier segments (causal) or the other segments (non-causal), in
    rank order.  See lt_linear_attn_state_carry."""
    world, B, Hkv, d, dv = S_all.shape
    for t in (S_all, z_all):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError("S_all and z_all must be contiguous float32 tensors")
    S = S_out if S_out is not None else torch.empty((B, Hkv, d, dv), dtype=torch.float32,
                                                    device=S_all.device)
    z = z_out if z_out is not None else torch.empty((B, Hkv, d), dtype=torch.float32,
                                                    device=S_all.device)
    _check(lib.lt_linear_attn_state_carry(_ptr(S_all), _ptr(z_all), world, int(rank),
                                          int(bool(causal)), B, Hkv, d, dv, _ptr(S), _ptr(z),
                                          _stream_handle(stream, S_all.device)))
    return S, z


def linear_attn_fwd_plan(B, H_q, H_kv, N, d, dv, causal=True, packed=False,
                         dtype=torch.bfloat16, num_sms=0):
    """(blocks per sequence, kernel launches, workspace bytes) of one
    linear_attn_fwd call on this shape; num_sms <= 0 asks the current
    device."""
    nb, nl, ws = _i(), _i(), ctypes.c_size_t()
    _check(lib.lt_linear_attn_fwd_plan(B, H_q, H_kv, N, d, dv, int(bool(causal)),
                                       int(bool(packed)), _dtype_code(dtype), int(num_sms),
                                       ctypes.byref(nb), ctypes.byref(nl), ctypes.byref(ws)))
    return nb.value, nl.value, ws.value


def linear_attn_decode_step(q, k, v, S, z, eps=1e-6, out=None, stream=None):
    """One recurrent step; S [B, H_kv, d, dv] and z [B, H_kv, d] (fp32) are
    updated in place.  q [B, H_q, d], k [B, H_kv, d], v [B, H_kv, dv]."""
    B, Hq, d = q.shape
    Hkv, dv = k.shape[1], v.shape[2]
    for t in (q, k, v, S, z):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    if S.dtype != torch.float32 or z.dtype != torch.float32:
        raise TypeError("S and z must be float32")
    if out is None:
        out = torch.empty((B, Hq, dv), dtype=q.dtype, device=q.device)
    _check(lib.lt_linear_attn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(z), _ptr(out),
                                          B, Hq, Hkv, d, dv, float(eps),
                                          _stream_handle(stream, q.device),
                                          _dtype_code(q.dtype)))
    return out


def set_schedule(kernel="auto", blocks=0):
    """Diagnostic override of the forward schedule, process-wide (tests and
    ablations): kernel "auto" | "two_launch" | "general", blocks 0 (the
    library's choice) or a block count per dense sequence."""
    _check(lib.lt_debug_set_schedule(_SCHED[kernel], int(blocks)))


def get_last_device_error(stream=None):
    """Synchronise the stream; return the device error status and clear it."""
    dev = torch.cuda.current_device()
    return lib.lt_get_last_device_error(_stream_handle(stream, dev))


def linear_attn_fwd_host(q, k, v, causal=True, eps=1e-6, cu_seqlens=None, device="cuda",
                         stream=None, out_host=None):
    """End-to-end call on HOST tensors: copy the inputs (pinned host memory
    recommended) to the device, run the forward pass, copy the result back.
    All copies and the kernel are enqueued on one stream; returns the host
    output once it has arrived."""
    dev = torch.device(device)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    with torch.cuda.stream(s):
        qd = q.to(dev, non_blocking=True)
        kd = k.to(dev, non_blocking=True)
        vd = v.to(dev, non_blocking=True)
        cud = cu_seqlens.to(dev, non_blocking=True) if cu_seqlens is not None else None
        od = linear_attn_fwd(qd, kd, vd, causal=causal, eps=eps, cu_seqlens=cud, stream=s)
        if out_host is None:
            out_host = torch.empty(od.shape, dtype=od.dtype, pin_memory=True)
        out_host.copy_(od, non_blocking=True)
    s.synchronize()
    return out_host
