"""Context parallelism: one sequence cut into contiguous segments across the
ranks of a torch.distributed process group, rank r holding segment r.

The only exchange is the recurrent state (S, z) per (sequence, KV head),
d*dv + d fp32 values, which is what makes linear attention split this way
(lineartile 1.0.0, "Reference": the recurrent view; "Features": multi-GPU
sharding; the inter-segment carry is the second level of the chunked scan of
"Why Stream Wins at Ultra-Long Context", section 5.3).  Per rank, every step
in the CUDA library on one stream:

  1. the segment's own state from a zero state, without outputs
     (lt_linear_attn_state);
  2. an all-gather of every segment's state (NCCL over NVLink on GPUs);
  3. the carry: the states of the earlier segments (causal) or of every
     other segment (non-causal), summed in rank order in fp32, so every run
     gives the same bits (lt_linear_attn_state_carry);
  4. the segment's outputs from that carry (lt_linear_attn_fwd_state).

A rank whose segment is empty contributes a zero state and returns an empty
output, after taking part in the same collective as every other rank.
"""
import contextlib

import torch


class LibraryOps:
    """The three steps as the CUDA library runs them (the default)."""

    def state(self, k, v, stream=None):
        from ._binding import linear_attn_state
        return linear_attn_state(k, v, stream=stream)

    def carry(self, S_all, z_all, rank, causal, stream=None):
        from ._binding import linear_attn_state_carry
        return linear_attn_state_carry(S_all, z_all, rank, causal=causal, stream=stream)

    def fwd_state(self, q, k, v, causal, eps, S0, z0, stream=None):
        from ._binding import linear_attn_fwd_state
        return linear_attn_fwd_state(q, k, v, causal=causal, eps=eps, S0=S0, z0=z0,
                                     return_state=False, stream=stream)


def linear_attn_fwd_cp(q, k, v, causal=True, eps=1e-6, group=None, stream=None, ops=None):
    """This rank's outputs of linear attention over the whole sequence.

    q [B, n_r, H_q, d], k [B, n_r, H_kv, d], v [B, n_r, H_kv, dv]: this
    rank's segment of every batch row (segments contiguous, in rank order;
    lengths may differ between ranks, and may be zero).  group: the process
    group (default: the world).  stream: the CUDA stream for every step
    (default: the current stream); the collective is ordered on it.  ops:
    the three steps (default: the CUDA library, ``LibraryOps``).
    Returns out [B, n_r, H_q, dv].
    """
    import torch.distributed as dist
    ops = ops if ops is not None else LibraryOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, n_r, Hq, d = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    cuda = q.is_cuda
    if cuda and stream is None:
        stream = torch.cuda.current_stream(q.device)
    ctx = torch.cuda.stream(stream) if cuda else contextlib.nullcontext()
    with ctx:
        kw = {"stream": stream} if cuda else {}
        if n_r > 0:
            S, z = ops.state(k, v, **kw)
        else:
            S = torch.zeros((B, Hkv, d, dv), dtype=torch.float32, device=q.device)
            z = torch.zeros((B, Hkv, d), dtype=torch.float32, device=q.device)
        S_all = torch.empty((world,) + tuple(S.shape), dtype=torch.float32, device=q.device)
        z_all = torch.empty((world,) + tuple(z.shape), dtype=torch.float32, device=q.device)
        dist.all_gather(list(S_all.unbind(0)), S, group=group)
        dist.all_gather(list(z_all.unbind(0)), z, group=group)
        S0, z0 = ops.carry(S_all, z_all, rank, causal, **kw)
        if n_r == 0:
            return torch.empty((B, 0, Hq, dv), dtype=q.dtype, device=q.device)
        return ops.fwd_state(q, k, v, causal, eps, S0, z0, **kw)
