"""Backward pass on the GPU (lt_linear_attn_bwd through the C ABI) against
the oracle's recurrent backward form, element by element on seeded inputs:
several 32-token chunks and a ragged tail, every width pair, GQA, causal
and non-causal, packed sequences with empty ones, fp32 and bf16 I/O.

Metric (tests/parity.py grad_rel_err): per (sequence, head) slice of each
gradient, the largest error relative to the slice's largest entry, with the
forward's bars: 1e-4 for fp32 I/O, 2e-2 for bf16 I/O (every product in fp32,
each gradient rounded once to bf16; the inputs are bf16 values the oracle
reads exactly).  Per-row relative errors do not apply to gradients: the
first token of a causal sequence moves with Q_0 and K_0 only through eps, so
its dQ row is a cancellation below fp32 resolution of its terms."""
import numpy as np
import pytest
import torch

import oracle
from parity import grad_rel_err, TOL_BF16, TOL_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def L():
    import causal_linear_attention_chunked_b200 as lt
    return lt


CASES = [
    # (B, Hq, Hkv, N, d, dv, causal)
    (1, 2, 2, 31, 64, 64, True),
    (2, 2, 2, 33, 64, 64, True),
    (1, 4, 2, 100, 64, 64, True),
    (2, 8, 2, 300, 64, 64, True),
    (1, 2, 2, 257, 128, 128, True),
    (1, 4, 1, 130, 64, 128, True),
    (1, 2, 2, 90, 128, 64, True),
    (2, 4, 2, 200, 64, 64, False),
    (1, 2, 1, 150, 128, 128, False),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dN%dd%ddv%d%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "nc"))
def test_bwd_dense_vs_oracle(case, dtype):
    B, Hq, Hkv, N, d, dv, causal = case
    scale = 1.0 if dtype == torch.float32 else d ** -0.5
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, dtype, scale, seed=N + 3 * d + dv)
    g = inputs.generator(N + 7)
    dout = torch.randn((B, N, Hq, dv), generator=g).to(dtype)
    dq, dk, dvv = L().linear_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    ref = oracle.bwd_recurrent(q, k, v, dout, causal=causal, eps=1e-6)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    for got, r, name in zip((dq, dk, dvv), ref, ("dq", "dk", "dv")):
        err = grad_rel_err(got.float().cpu().numpy(), r)
        assert err <= tol, (name, err)


def test_bwd_packed_with_empty_sequences():
    lens = [70, 0, 2, 33, 0, 128]  # one-token sequences: test_bwd_one_token
    cu = inputs.cu_from_lengths(lens)
    T, Hq, Hkv, d, dv = int(cu[-1]), 4, 2, 64, 64
    g = inputs.generator(41)
    q, k, v, dout = ((torch.randn(sh, generator=g) * 0.125).to(torch.bfloat16) for sh in
                     ((T, Hq, d), (T, Hkv, d), (T, Hkv, dv), (T, Hq, dv)))
    for causal in (True, False):
        dq, dk, dvv = L().linear_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dout.cuda(),
                                          causal=causal, cu_seqlens=cu.cuda())
        torch.cuda.synchronize()
        assert L().get_last_device_error() == 0
        ref = oracle.bwd_recurrent(q, k, v, dout, causal=causal, cu_seqlens=cu.numpy())
        for got, r in zip((dq, dk, dvv), ref):
            assert grad_rel_err(got.float().cpu().numpy(), r, cu=cu.numpy()) <= TOL_BF16


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_bwd_one_token(dtype):
    """One token: O_0 = V_0 a / (a + eps), so dV_0 = dO_0 a / (a + eps) and
    dQ_0, dK_0 are proportional to eps (here 1e-6): dV against the oracle,
    dQ and dK at most 1e-5 of the scale |dO| |V| of their terms."""
    q, k, v = inputs.make_custom(2, 4, 2, 1, 64, 64, dtype, 0.125, seed=3)
    g = inputs.generator(4)
    dout = torch.randn((2, 1, 4, 64), generator=g).to(dtype)
    dq, dk, dvv = L().linear_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dout.cuda())
    torch.cuda.synchronize()
    ref = oracle.bwd_recurrent(q, k, v, dout, causal=True, eps=1e-6)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert grad_rel_err(dvv.float().cpu().numpy(), ref[2]) <= tol
    term = float(dout.float().abs().max() * v.float().abs().max())
    assert float(dq.float().abs().max()) <= 1e-5 * term
    assert float(dk.float().abs().max()) <= 1e-5 * term


def test_bwd_hand_example_on_gpu():
    """The hand-worked 2x2 gradients (embedded in 64 feature dims whose
    padding underflows phi) through the fp32 path."""
    import json, os
    gld = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                      "hand_2x2_backward.json")))
    d = dv = 64
    q = torch.full((1, 2, 1, d), -200.0)
    k = torch.full((1, 2, 1, d), -200.0)
    q[0, :, 0, :2] = torch.tensor(gld["q"])
    k[0, :, 0, :2] = torch.tensor(gld["k"])
    v = torch.zeros((1, 2, 1, dv))
    v[0, :, 0, :2] = torch.tensor(gld["v"])
    dout = torch.zeros((1, 2, 1, dv))
    dout[0, :, 0, :2] = torch.tensor(gld["dout"])
    for causal, key in ((True, "causal"), (False, "noncausal")):
        dq, dk, dvv = L().linear_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dout.cuda(),
                                          causal=causal, eps=0.0)
        torch.cuda.synchronize()
        for got, name in ((dq, "dq"), (dk, "dk"), (dvv, "dv")):
            g2 = got[0, :, 0, :2].cpu().double().numpy()
            assert np.allclose(g2, gld[key][name], rtol=1e-5, atol=1e-6), (key, name, g2)


def test_bwd_deterministic():
    q, k, v = (t.cuda() for t in inputs.make_custom(2, 8, 2, 700, 64, 64, torch.bfloat16, 0.125,
                                                     seed=5))
    dout = torch.randn((2, 700, 8, 64), device="cuda").to(torch.bfloat16)
    a = L().linear_attn_bwd(q, k, v, dout)
    b = L().linear_attn_bwd(q, k, v, dout)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


FULL = ["bf16_b2h8n4096d64", "bf16_b1h8n65536d64", "bf16_b1h8n65536d64_noncausal",
        "bf16_gqa_b2hq32hkv8n16384d128", "bf16_varlen64_h8d64"]


@pytest.mark.parametrize("name", FULL)
def test_bwd_full_size_every_element(name):
    """Every gradient element of the bf16 workloads at full size (the block
    count the library picks for them: many blocks per sequence, carried
    block sums) against the oracle's recurrent backward form."""
    w = inputs.WORKLOADS[name]
    q, k, v, cu = inputs.make(w, seed=w.seed + 700)
    g = inputs.generator(w.seed + 701)
    dout = torch.randn(q.shape[:-1] + (w.dv,), generator=g).to(w.dtype)
    cuc = cu.cuda() if cu is not None else None
    dq, dk, dvv = L().linear_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dout.cuda(),
                                      causal=w.causal, eps=w.eps, cu_seqlens=cuc)
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    ref = oracle.bwd_recurrent(q, k, v, dout, causal=w.causal, eps=w.eps,
                               cu_seqlens=cu.numpy() if cu is not None else None)
    for got, r, nm in zip((dq, dk, dvv), ref, ("dq", "dk", "dv")):
        err = grad_rel_err(got.float().cpu().numpy(), r,
                           cu=cu.numpy() if cu is not None else None)
        assert err <= TOL_BF16, (nm, err)
