"""fp64 CPU oracle for kernelised linear attention -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never touches it, and it shares no code with them.

Thin ctypes wrappers around ``lt_oracle.c``.  Every function takes CPU arrays
(numpy, or torch CPU tensors) holding the exact values given to the GPU
(float32, bfloat16 or float64), widens them to fp64 and returns fp64 numpy
arrays.  Layouts are token-major: dense ``[B][N][H][d]``, packed
``[N_total][H][d]`` with ``cu_seqlens``.  The mathematics and the page each
function follows are documented in ``lt_oracle.c``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_F32, _BF16, _F64, _F16 = 0, 1, 2, 3
PHI_KINDS = {"elu1": 0, "relu": 1, "exp": 2}
_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        vp, dp, ip = ctypes.c_void_p, ctypes.POINTER(ctypes.c_double), ctypes.c_int
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        fwd_args = [vp, vp, vp, ip, dp, ip, ip, ip, ip, ip, ip, ip, ctypes.c_double, i32p]
        lib.lt_oracle_fwd_quadratic.argtypes = fwd_args
        lib.lt_oracle_fwd_recurrent.argtypes = fwd_args
        lib.lt_oracle_fwd_rows.argtypes = [vp, vp, vp, ip, ip, ip, ip, ip, ip, ip, ip,
                                           ctypes.c_double, i32p, i64p, ip, dp]
        lib.lt_oracle_noncausal_numerator.argtypes = [vp, vp, vp, ip, dp, ip, ip, ip, ip, ip,
                                                      ip, i32p, ip]
        lib.lt_oracle_decode_step.argtypes = [vp, vp, vp, ip, dp, dp, dp, ip, ip, ip, ip, ip,
                                              ctypes.c_double]
        lib.lt_oracle_fwd_state.argtypes = fwd_args + [dp, dp, dp, dp]
        bwd_args = [vp, vp, vp, vp, ip, dp, dp, dp, ip, ip, ip, ip, ip, ip, ip,
                    ctypes.c_double, i32p]
        lib.lt_oracle_bwd_quadratic.argtypes = bwd_args
        lib.lt_oracle_bwd_recurrent.argtypes = bwd_args
        win_args = [vp, vp, vp, ip, dp, ip, ip, ip, ip, ip, ip, ip, ctypes.c_double, i32p]
        lib.lt_oracle_fwd_window_quadratic.argtypes = win_args
        lib.lt_oracle_fwd_window_recurrent.argtypes = win_args
        lib.lt_oracle_set_phi.argtypes = [ctypes.c_int]
        lib.lt_oracle_set_phi.restype = ctypes.c_int
        lib.lt_oracle_phi.argtypes = [ctypes.c_double]
        lib.lt_oracle_phi.restype = ctypes.c_double
        lib.lt_oracle_num_threads.restype = ctypes.c_int
        for name in ("lt_oracle_fwd_quadratic", "lt_oracle_fwd_recurrent", "lt_oracle_fwd_rows",
                     "lt_oracle_noncausal_numerator", "lt_oracle_decode_step",
                     "lt_oracle_fwd_state", "lt_oracle_bwd_quadratic",
                     "lt_oracle_bwd_recurrent", "lt_oracle_fwd_window_quadratic",
                     "lt_oracle_fwd_window_recurrent"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _raw(x):
    """Return (contiguous numpy array holding the raw bits, type code)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), _BF16
            if x.dtype == torch.float16:
                return x.view(torch.int16).numpy().view(np.uint16), _F16
            if x.dtype == torch.float32:
                return x.numpy(), _F32
            if x.dtype == torch.float64:
                return x.numpy(), _F64
            raise TypeError("unsupported dtype %s" % x.dtype)
    except ImportError:
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16), _F16
    if x.dtype == np.float32:
        return x, _F32
    if x.dtype == np.float64:
        return x, _F64
    raise TypeError("unsupported dtype %s" % x.dtype)


def _same_type(*arrs):
    raws = [_raw(a) for a in arrs]
    types = {t for _, t in raws}
    if len(types) != 1:
        raise TypeError("q, k, v must share one dtype")
    return [r for r, _ in raws], types.pop()


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _cu(cu_seqlens):
    if cu_seqlens is None:
        return None, None
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    return cu, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _geometry(q, k, v, cu_seqlens):
    """(B, Hq, Hkv, N, d, dv, out_shape) from token-major shapes."""
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv, dv = k.shape[2], v.shape[3]
        return B, Hq, Hkv, N, d, dv, (B, N, Hq, dv)
    N, Hq, d = q.shape
    Hkv, dv = k.shape[1], v.shape[2]
    B = len(cu_seqlens) - 1
    return B, Hq, Hkv, N, d, dv, (N, Hq, dv)


class feature_map:
    """Context manager: the oracle's feature map within the block ("elu1",
    the method's ELU + 1 and the default; "relu"; "exp")."""

    def __init__(self, kind):
        self.kind = PHI_KINDS[kind]

    def __enter__(self):
        if _load().lt_oracle_set_phi(self.kind) != 0:
            raise ValueError("unknown feature map")
        return self

    def __exit__(self, *exc):
        _load().lt_oracle_set_phi(0)
        return False


def phi(x: float, kind="elu1") -> float:
    """The feature map in fp64 (default: phi(x) = ELU(x) + 1, alpha = 1)."""
    with feature_map(kind):
        return _load().lt_oracle_phi(float(x))


def num_threads() -> int:
    return _load().lt_oracle_num_threads()


def _fwd(fn, q, k, v, causal, eps, cu_seqlens):
    (rq, rk, rv), t = _same_type(q, k, v)
    B, Hq, Hkv, N, d, dv, oshape = _geometry(rq, rk, rv, cu_seqlens)
    out = np.zeros(oshape, dtype=np.float64)
    cu, cup = _cu(cu_seqlens)
    rc = fn(_ptr(rq), _ptr(rk), _ptr(rv), t, _dptr(out), B, Hq, Hkv, N, d, dv,
            int(bool(causal)), float(eps), cup)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def fwd_quadratic(q, k, v, causal=True, eps=1e-6, cu_seqlens=None, phi="elu1"):
    """Masked quadratic form: O_i = sum_j a_ij V_j / (sum_j a_ij + eps)."""
    with feature_map(phi):
        return _fwd(_load().lt_oracle_fwd_quadratic, q, k, v, causal, eps, cu_seqlens)


def fwd_recurrent(q, k, v, causal=True, eps=1e-6, cu_seqlens=None, phi="elu1"):
    """Recurrent (RNN) form over the fixed-size state (S, z)."""
    with feature_map(phi):
        return _fwd(_load().lt_oracle_fwd_recurrent, q, k, v, causal, eps, cu_seqlens)


def fwd_state(q, k, v, causal=True, eps=1e-6, cu_seqlens=None, S0=None, z0=None):
    """Recurrent form continued from the state (S0, z0) (zero if None);
    returns (out, S, z) with the state after each sequence's last token.
    States are per (sequence, KV head): S [B][Hkv][d][dv], z [B][Hkv][d]."""
    (rq, rk, rv), t = _same_type(q, k, v)
    B, Hq, Hkv, N, d, dv, oshape = _geometry(rq, rk, rv, cu_seqlens)
    out = np.zeros(oshape, dtype=np.float64)
    S = np.zeros((B, Hkv, d, dv), dtype=np.float64)
    z = np.zeros((B, Hkv, d), dtype=np.float64)
    s0 = None if S0 is None else np.ascontiguousarray(np.asarray(S0, dtype=np.float64).reshape(S.shape))
    z0_ = None if z0 is None else np.ascontiguousarray(np.asarray(z0, dtype=np.float64).reshape(z.shape))
    cu, cup = _cu(cu_seqlens)
    rc = _load().lt_oracle_fwd_state(
        _ptr(rq), _ptr(rk), _ptr(rv), t, _dptr(out), B, Hq, Hkv, N, d, dv, int(bool(causal)),
        float(eps), cup, None if s0 is None else _dptr(s0), None if z0_ is None else _dptr(z0_),
        _dptr(S), _dptr(z))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out, S, z


def fwd_rows(q, k, v, rows, causal=True, eps=1e-6, cu_seqlens=None, phi="elu1"):
    """Selected output rows by the quadratic definition.

    ``rows``: integer array of shape [R, 3] holding (sequence, position
    within the sequence, query head).  Returns fp64 [R, dv].
    """
    (rq, rk, rv), t = _same_type(q, k, v)
    B, Hq, Hkv, N, d, dv, _ = _geometry(rq, rk, rv, cu_seqlens)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    out = np.zeros((rows.shape[0], dv), dtype=np.float64)
    cu, cup = _cu(cu_seqlens)
    with feature_map(phi):
        rc = _load().lt_oracle_fwd_rows(_ptr(rq), _ptr(rk), _ptr(rv), t, B, Hq, Hkv, N, d, dv,
                                        int(bool(causal)), float(eps), cup,
                                        rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                        rows.shape[0], _dptr(out))
    if rc != 0:
        raise ValueError("oracle rejected a row index")
    return out


def noncausal_numerator(q, k, v, order, cu_seqlens=None):
    """Unnormalised phi(Q)(phi(K)^T V); order 0 = scores first, 1 = KV first."""
    (rq, rk, rv), t = _same_type(q, k, v)
    B, Hq, Hkv, N, d, dv, oshape = _geometry(rq, rk, rv, cu_seqlens)
    out = np.zeros(oshape, dtype=np.float64)
    cu, cup = _cu(cu_seqlens)
    rc = _load().lt_oracle_noncausal_numerator(_ptr(rq), _ptr(rk), _ptr(rv), t, _dptr(out),
                                               B, Hq, Hkv, N, d, dv, cup, int(order))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def decode_step(q, k, v, S, z, eps=1e-6):
    """One recurrent decode step.

    q [B][Hq][d], k [B][Hkv][d], v [B][Hkv][dv]; S [B][Hkv][d][dv] and
    z [B][Hkv][d] are fp64 numpy arrays updated in place.  Returns
    out [B][Hq][dv] in fp64.
    """
    (rq, rk, rv), t = _same_type(q, k, v)
    B, Hq, d = rq.shape
    Hkv, dv = rk.shape[1], rv.shape[2]
    if S.dtype != np.float64 or z.dtype != np.float64 or not S.flags.c_contiguous \
            or not z.flags.c_contiguous:
        raise TypeError("S and z must be C-contiguous float64 arrays")
    out = np.zeros((B, Hq, dv), dtype=np.float64)
    rc = _load().lt_oracle_decode_step(_ptr(rq), _ptr(rk), _ptr(rv), t, _dptr(S), _dptr(z),
                                       _dptr(out), B, Hq, Hkv, d, dv, float(eps))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def _bwd(fn, q, k, v, dout, causal, eps, cu_seqlens):
    (rq, rk, rv, rdo), t = _same_type(q, k, v, dout)
    B, Hq, Hkv, N, d, dv, oshape = _geometry(rq, rk, rv, cu_seqlens)
    if tuple(rdo.shape) != tuple(oshape):
        raise ValueError("dout must have the output's shape %s" % (oshape,))
    dq = np.zeros(rq.shape, dtype=np.float64)
    dk = np.zeros(rk.shape, dtype=np.float64)
    dvv = np.zeros(rv.shape, dtype=np.float64)
    cu, cup = _cu(cu_seqlens)
    rc = fn(_ptr(rq), _ptr(rk), _ptr(rv), _ptr(rdo), t, _dptr(dq), _dptr(dk), _dptr(dvv), B, Hq,
            Hkv, N, d, dv, int(bool(causal)), float(eps), cup)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return dq, dk, dvv


def bwd_quadratic(q, k, v, dout, causal=True, eps=1e-6, cu_seqlens=None):
    """Gradients (dQ, dK, dV) of sum(O * dout) by the quadratic definition."""
    return _bwd(_load().lt_oracle_bwd_quadratic, q, k, v, dout, causal, eps, cu_seqlens)


def bwd_recurrent(q, k, v, dout, causal=True, eps=1e-6, cu_seqlens=None):
    """Gradients (dQ, dK, dV) by the forward and reverse state recurrences."""
    return _bwd(_load().lt_oracle_bwd_recurrent, q, k, v, dout, causal, eps, cu_seqlens)


def _fwd_window(fn, q, k, v, window, eps, cu_seqlens):
    (rq, rk, rv), t = _same_type(q, k, v)
    B, Hq, Hkv, N, d, dv, oshape = _geometry(rq, rk, rv, cu_seqlens)
    out = np.zeros(oshape, dtype=np.float64)
    cu, cup = _cu(cu_seqlens)
    rc = fn(_ptr(rq), _ptr(rk), _ptr(rv), t, _dptr(out), B, Hq, Hkv, N, d, dv, int(window),
            float(eps), cup)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def fwd_window_quadratic(q, k, v, window, eps=1e-6, cu_seqlens=None):
    """Sliding-window causal attention: keys i - window < j <= i, by the
    masked quadratic definition."""
    return _fwd_window(_load().lt_oracle_fwd_window_quadratic, q, k, v, window, eps, cu_seqlens)


def fwd_window_recurrent(q, k, v, window, eps=1e-6, cu_seqlens=None):
    """Sliding-window causal attention as the difference of the prefix state
    and a prefix state `window` tokens behind."""
    return _fwd_window(_load().lt_oracle_fwd_window_recurrent, q, k, v, window, eps, cu_seqlens)
