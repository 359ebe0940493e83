"""Kernelised (linear) attention for NVIDIA B200 (sm_100a).

    O_i = phi(Q_i) S_i / (phi(Q_i) . z_i + eps),  phi(x) = ELU(x) + 1,

causal or non-causal, with grouped-query heads, packed variable-length
sequences, a forward pass that starts from and returns the recurrent state,
and a recurrent decode step.  The computation runs in the CUDA
library ``liblt.so`` behind the C ABI of ``include/lt_linear_attn.h``; this
package is a thin ctypes binding over it (PyTorch supplies device memory and
streams).  ``inputs`` holds the seeded synthetic workloads.

The binding (and with it the library) is loaded on first use of one of the
API names below; a missing library raises ImportError.
"""
_API = ("linear_attn_fwd", "linear_attn_fwd_state", "linear_attn_fwd_plan",
        "linear_attn_decode_step", "linear_attn_state", "linear_attn_state_carry",
        "linear_attn_bwd", "linear_attn_fwd_window",
        "set_schedule",
        "get_last_device_error",
        "linear_attn_fwd_host", "LtError")


def __getattr__(name):
    if name in _API:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)
