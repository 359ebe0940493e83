"""Small, self-checking invocations of the library's kernels for ncu captures.

    python -m causal_linear_attention_chunked_b200.profile_cases CASE

CASE is one of:
  fused    the forward pass at bf16, B=2, H=8, N=4096, d=dv=64, causal:
           six calls over eight seeded input sets, so a capture can skip the
           first launches and still see a launch with cold inputs
  decode   eight decode steps of the decode workload (B=64, H=8, d=dv=64) from
           a zero state
  bwd      one backward call at that shape with a random upstream gradient
  gqa      four forward passes of the GQA workload cut to one sequence
           (B=1, Hq=32, Hkv=8, N=16384, d=dv=128)

Each case checks the library's device error word after synchronising and
prints "ok"; inputs come from the seeded generators of ``inputs``.
"""
import sys

import torch

from . import inputs


def _lib():
    import causal_linear_attention_chunked_b200 as lt
    return lt


def fused():
    L = _lib()
    w = inputs.WORKLOADS["bf16_b2h8n4096d64"]
    sets = []
    for r in range(8):
        q, k, v, _ = inputs.make(w, seed=w.seed + r)
        sets.append((q.cuda(), k.cuda(), v.cuda()))
    for i in range(6):
        q, k, v = sets[i % 8]
        L.linear_attn_fwd(q, k, v, causal=True, eps=w.eps)
    torch.cuda.synchronize()


def decode():
    L = _lib()
    c = inputs.DECODE
    B, Hq, Hkv, d, dv = c["B"], c["Hq"], c["Hkv"], c["d"], c["dv"]
    g = inputs.generator(c["seed"])
    S = torch.zeros(B, Hkv, d, dv, device="cuda")
    z = torch.zeros(B, Hkv, d, device="cuda")
    for _ in range(8):
        q, k, v = (x.cuda() for x in
                   inputs.make_decode_step(B, Hq, Hkv, d, dv, c["dtype"], c["scale"], g))
        L.linear_attn_decode_step(q, k, v, S, z)
    torch.cuda.synchronize()


def bwd():
    L = _lib()
    w = inputs.WORKLOADS["bf16_b2h8n4096d64"]
    q, k, v, _ = inputs.make(w, seed=w.seed + 700)
    g = inputs.generator(w.seed + 701)
    dout = torch.randn(q.shape[:-1] + (w.dv,), generator=g).to(w.dtype)
    L.linear_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), causal=True, eps=w.eps)
    torch.cuda.synchronize()


def gqa():
    import dataclasses
    L = _lib()
    w = dataclasses.replace(inputs.WORKLOADS["bf16_gqa_b2hq32hkv8n16384d128"], B=1)
    q, k, v, _ = inputs.make(w, seed=7)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty(q.shape[:-1] + (w.dv,), dtype=w.dtype, device="cuda")
    for _ in range(4):
        L.linear_attn_fwd(q, k, v, causal=True, eps=w.eps, out=o)
    torch.cuda.synchronize()


CASES = {"fused": fused, "decode": decode, "bwd": bwd, "gqa": gqa}


def main(argv):
    if len(argv) != 1 or argv[0] not in CASES:
        raise SystemExit("usage: python -m causal_linear_attention_chunked_b200.profile_cases "
                         "{%s}" % ",".join(CASES))
    CASES[argv[0]]()
    if _lib().get_last_device_error() != 0:
        raise SystemExit("device error word set")
    print("ok")


if __name__ == "__main__":
    main(sys.argv[1:])
