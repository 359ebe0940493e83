"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method: it only draws random numbers
and casts them.  Recipe (the same for every caller):

* ``torch.Generator`` on the CPU, seeded with the workload's seed;
* for packed workloads the sequence lengths are drawn first
  (``torch.randint`` inclusive of both bounds), then Q, K, V in that order
  with ``torch.randn`` in fp32;
* Q, K, V are multiplied by ``scale`` (1/sqrt(d) for the bf16 workloads,
  1 for the fp32 one) and cast to the run dtype with round-to-nearest-even.

The workloads follow the sizes and value distributions of the pages' usage
example (d_model 512 split over 8 heads of 64, sequences of 1k-64k tokens)
and the GQA / packed-sequence / decode features the lineartile page lists.
"""
from dataclasses import dataclass, field
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int            # batch rows, or number of packed sequences
    Hq: int
    Hkv: int
    N: int            # tokens per row (dense); 0 for packed (drawn lengths)
    d: int
    dv: int
    dtype: torch.dtype
    scale: float
    causal: bool
    seed: int
    packed_len: tuple = field(default=None)   # (lo, hi) for packed workloads
    eps: float = 1e-6


def _w(name, B, Hq, Hkv, N, d, dtype, causal, seed, packed_len=None, unit_scale=False):
    return Workload(name, B, Hq, Hkv, N, d, d, dtype, 1.0 if unit_scale else 1.0 / math.sqrt(d),
                    causal, seed, packed_len)


WORKLOADS = {
    # fp32 I/O, unit-variance inputs, single head
    "fp32_b1h1n256d64": _w("fp32_b1h1n256d64", 1, 1, 1, 256, 64, torch.float32, True, 1,
                           unit_scale=True),
    # the usage example of the lineartile page: d_model 512 = 8 heads x 64, B=2, N=4096
    "bf16_b2h8n4096d64": _w("bf16_b2h8n4096d64", 2, 8, 8, 4096, 64, torch.bfloat16, True, 2),
    # one long sequence, causal and non-causal
    "bf16_b1h8n65536d64": _w("bf16_b1h8n65536d64", 1, 8, 8, 65536, 64, torch.bfloat16, True, 3),
    "bf16_b1h8n65536d64_noncausal": _w("bf16_b1h8n65536d64_noncausal", 1, 8, 8, 65536, 64,
                                       torch.bfloat16, False, 3),
    # grouped-query attention: 32 query heads over 8 KV heads, d = 128
    "bf16_gqa_b2hq32hkv8n16384d128": _w("bf16_gqa_b2hq32hkv8n16384d128", 2, 32, 8, 16384, 128,
                                        torch.bfloat16, True, 4),
    # 64 packed sequences with lengths uniform in [128, 8192]
    "bf16_varlen64_h8d64": _w("bf16_varlen64_h8d64", 64, 8, 8, 0, 64, torch.bfloat16, True, 5,
                              packed_len=(128, 8192)),
}

# recurrent decode: batch 64, 8 heads of 64, 1000 steps from a zero state
DECODE = dict(name="decode_b64h8d64_1000steps", B=64, Hq=8, Hkv=8, d=64, dv=64, steps=1000,
              dtype=torch.bfloat16, scale=1.0 / 8.0, seed=6, eps=1e-6)


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def draw_lengths(n: int, lo: int, hi: int, g: torch.Generator) -> torch.Tensor:
    """n sequence lengths uniform on the integers lo..hi (inclusive)."""
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64)


def cu_from_lengths(lengths) -> torch.Tensor:
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    return cu.to(torch.int32)


def draw_qkv(shape_q, shape_k, shape_v, scale, dtype, g):
    q = (torch.randn(shape_q, generator=g, dtype=torch.float32) * scale).to(dtype)
    k = (torch.randn(shape_k, generator=g, dtype=torch.float32) * scale).to(dtype)
    v = (torch.randn(shape_v, generator=g, dtype=torch.float32) * scale).to(dtype)
    return q, k, v


def make(w: Workload, seed=None, n_override=None, lengths=None):
    """Draw (q, k, v, cu_seqlens) on the CPU for workload ``w``.

    ``n_override`` replaces N for dense workloads (smaller parity cases of the
    same kind); ``lengths`` fixes the packed sequence lengths instead of
    drawing them.  cu_seqlens is None for dense workloads.
    """
    g = generator(w.seed if seed is None else seed)
    if w.packed_len is not None or lengths is not None:
        if lengths is None:
            lengths = draw_lengths(w.B, w.packed_len[0], w.packed_len[1], g)
        cu = cu_from_lengths(lengths)
        total = int(cu[-1])
        q, k, v = draw_qkv((total, w.Hq, w.d), (total, w.Hkv, w.d), (total, w.Hkv, w.dv),
                           w.scale, w.dtype, g)
        return q, k, v, cu
    N = w.N if n_override is None else n_override
    q, k, v = draw_qkv((w.B, N, w.Hq, w.d), (w.B, N, w.Hkv, w.d), (w.B, N, w.Hkv, w.dv),
                       w.scale, w.dtype, g)
    return q, k, v, None


def make_custom(B, Hq, Hkv, N, d, dv, dtype, scale, seed):
    """Dense token-major q, k, v of arbitrary shape (for edge cases)."""
    g = generator(seed)
    return draw_qkv((B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, dv), scale, dtype, g)


def make_decode_step(B, Hq, Hkv, d, dv, dtype, scale, g):
    """q [B][Hq][d], k [B][Hkv][d], v [B][Hkv][dv] for one decode step."""
    return draw_qkv((B, Hq, d), (B, Hkv, d), (B, Hkv, dv), scale, dtype, g)


def tokens(w: Workload, cu=None) -> int:
    """B*Hq*N (dense) or Hq*sum(lengths) (packed): the metric's unit count."""
    if cu is not None:
        return int(cu[-1]) * w.Hq
    return w.B * w.Hq * w.N
