"""Parity metric shared by the GPU tests.

Row metric (the tolerance reading used throughout): for every output row
(token, head) take ||O_gpu - O_ref||_inf / ||O_ref||_inf and report the
maximum over rows.  Elementwise relative error is meaningless for outputs
near zero (V has mean 0), so each row is measured against its own largest
entry.  Bars: 1e-4 for fp32 I/O, 2e-2 for bf16 I/O with fp32 accumulation.
"""
import numpy as np

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def row_rel_err(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    g2 = gpu.reshape(-1, gpu.shape[-1])
    r2 = ref.reshape(-1, ref.shape[-1])
    assert np.all(np.isfinite(g2)), "non-finite GPU output"
    den = np.abs(r2).max(axis=1)
    den = np.maximum(den, 1e-30)
    return float((np.abs(g2 - r2).max(axis=1) / den).max())


def tol_for(dtype):
    import torch
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def state_rel_err(got, ref):
    """Largest error of a state, relative to the largest magnitude of the
    same (sequence, KV head) state."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got))
    g2 = got.reshape(got.shape[0] * got.shape[1], -1)
    r2 = ref.reshape(ref.shape[0] * ref.shape[1], -1)
    den = np.maximum(np.abs(r2).max(axis=1), 1e-30)
    return float((np.abs(g2 - r2).max(axis=1) / den).max())


# fp32 state accumulated from bf16-rounded phi(K): relative error of a state
# well inside the bf16 rounding of its terms (2^-8)
TOL_STATE_BF16 = 8e-3
TOL_STATE_F32 = 1e-4


def grad_rel_err(got, ref, cu=None):
    """Gradient metric: per (sequence, head) slice, the largest error
    relative to the slice's largest entry; the maximum over slices.

    A row of dQ (or dK) can be a near-exact cancellation whose true value is
    proportional to eps -- the first token of a causal sequence attends only
    to itself, so its output moves with Q_0 and K_0 only through eps -- and a
    per-row relative error is then meaningless; the slice holds the terms'
    scale.  Dense arrays [B][N][H][w]; packed [T][H][w] with cu_seqlens."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got))
    if cu is None:
        slices = [(got[b, :, h], ref[b, :, h]) for b in range(got.shape[0])
                  for h in range(got.shape[2])]
    else:
        c = [int(x) for x in cu]
        slices = [(got[c[s]:c[s + 1], h], ref[c[s]:c[s + 1], h]) for s in range(len(c) - 1)
                  for h in range(got.shape[1]) if c[s + 1] > c[s]]
    worst = 0.0
    for g, r in slices:
        worst = max(worst, float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30)))
    return worst
