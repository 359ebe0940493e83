"""Context parallelism: one sequence cut into contiguous segments across the
ranks of a torch.distributed process group, rank r holding segment r.

The only exchange is the recurrent state (S, z) per (sequence, KV head),
d*dv + d fp32 values, which is what makes linear attention split this way
(lineartile 1.0.0, "Reference": the recurrent view; the inter-segment carry
is the second level of the chunked scan of "Why Stream Wins at Ultra-Long
Context", section 5.3).  Per rank:

  1. the segment's own final state, from a zero state (lt_linear_attn_fwd_state);
  2. an all-gather of every segment's state (NCCL over NVLink on GPUs);
  3. the carry: the states of the earlier segments (causal) or of every
     other segment (non-causal), summed in rank order in fp32, so every run
     gives the same bits;
  4. the segment's outputs from that carry (lt_linear_attn_fwd_state).

Step 1 also computes the segment's outputs from a zero state, which step 4
recomputes: the price of reusing the forward entry point for the state.
"""
import torch


def linear_attn_fwd_cp(q, k, v, causal=True, eps=1e-6, group=None, stream=None,
                       fwd_state=None):
    """This rank's outputs of linear attention over the whole sequence.

    q [B, n_r, H_q, d], k [B, n_r, H_kv, d], v [B, n_r, H_kv, dv]: this
    rank's segment of every batch row (segments contiguous, in rank order;
    lengths may differ between ranks).  group: the process group (default:
    the world).  fwd_state: the stateful forward (default: the CUDA library's
    linear_attn_fwd_state); its signature is that of linear_attn_fwd_state.
    Returns out [B, n_r, H_q, dv].
    """
    import torch.distributed as dist
    if fwd_state is None:
        from ._binding import linear_attn_fwd_state as fwd_state
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    kw = {} if stream is None else {"stream": stream}
    _, S, z = fwd_state(q, k, v, causal=True, eps=eps, **kw)
    Ss = [torch.empty_like(S) for _ in range(world)]
    zs = [torch.empty_like(z) for _ in range(world)]
    dist.all_gather(Ss, S, group=group)
    dist.all_gather(zs, z, group=group)
    S0 = torch.zeros_like(S)
    z0 = torch.zeros_like(z)
    for r in range(world):
        if r < rank or (not causal and r != rank):
            S0 += Ss[r]
            z0 += zs[r]
    return fwd_state(q, k, v, causal=causal, eps=eps, S0=S0, z0=z0, return_state=False, **kw)
