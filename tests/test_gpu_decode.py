"""The recurrent decode step on the GPU against the oracle's decode step,
and chained steps against the causal forward pass (C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from parity import row_rel_err, TOL_BF16, TOL_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(64, 8, 8, 64, 64), (3, 8, 2, 128, 128), (5, 4, 1, 64, 128),
                                   (2, 6, 3, 128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_steps_vs_oracle(shape, dtype):
    import causal_linear_attention_chunked_b200 as L
    B, Hq, Hkv, d, dv = shape
    g = inputs.generator(11)
    S = torch.zeros(B, Hkv, d, dv, device="cuda")
    z = torch.zeros(B, Hkv, d, device="cuda")
    Sr = np.zeros((B, Hkv, d, dv))
    zr = np.zeros((B, Hkv, d))
    tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_F32
    for step in range(40):
        q, k, v = inputs.make_decode_step(B, Hq, Hkv, d, dv, dtype, d ** -0.5, g)
        out = L.linear_attn_decode_step(q.cuda(), k.cuda(), v.cuda(), S, z)
        ref = oracle.decode_step(q, k, v, Sr, zr)
        assert row_rel_err(out.float().cpu().numpy(), ref) <= tol, step
    # the state itself is fp32 on both sides up to accumulation order
    assert np.abs(S.cpu().numpy() - Sr).max() <= 1e-5 * np.abs(Sr).max()
    assert np.abs(z.cpu().numpy() - zr).max() <= 1e-5 * np.abs(zr).max()


def test_decode_workload_1000_steps():
    """Batch 64, 8 heads of 64, 1000 steps from a zero state."""
    import causal_linear_attention_chunked_b200 as L
    c = inputs.DECODE
    B, Hq, Hkv, d, dv = c["B"], c["Hq"], c["Hkv"], c["d"], c["dv"]
    g = inputs.generator(c["seed"])
    S = torch.zeros(B, Hkv, d, dv, device="cuda")
    z = torch.zeros(B, Hkv, d, device="cuda")
    Sr = np.zeros((B, Hkv, d, dv))
    zr = np.zeros((B, Hkv, d))
    worst = 0.0
    for step in range(c["steps"]):
        q, k, v = inputs.make_decode_step(B, Hq, Hkv, d, dv, c["dtype"], c["scale"], g)
        out = L.linear_attn_decode_step(q.cuda(), k.cuda(), v.cuda(), S, z, eps=c["eps"])
        ref = oracle.decode_step(q, k, v, Sr, zr, eps=c["eps"])
        if step % 50 == 0 or step == c["steps"] - 1:
            worst = max(worst, row_rel_err(out.float().cpu().numpy(), ref))
    assert worst <= TOL_BF16, worst
    assert np.abs(S.cpu().numpy() - Sr).max() <= 1e-4 * np.abs(Sr).max()


def test_decode_chain_matches_forward():
    """N decode steps reproduce the causal forward pass of the same tokens."""
    import causal_linear_attention_chunked_b200 as L
    B, N, Hq, Hkv, d, dv = 2, 300, 4, 2, 64, 64
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, 0.125, seed=3)
    fwd = L.linear_attn_fwd(q.cuda(), k.cuda(), v.cuda()).float().cpu().numpy()
    S = torch.zeros(B, Hkv, d, dv, device="cuda")
    z = torch.zeros(B, Hkv, d, device="cuda")
    outs = []
    for t in range(N):
        outs.append(L.linear_attn_decode_step(q[:, t].contiguous().cuda(),
                                              k[:, t].contiguous().cuda(),
                                              v[:, t].contiguous().cuda(), S, z).float().cpu())
    dec = torch.stack(outs, dim=1).numpy()
    ref = oracle.fwd_recurrent(q, k, v, causal=True, eps=1e-6)
    assert row_rel_err(dec, ref) <= TOL_BF16
    assert row_rel_err(fwd, ref) <= TOL_BF16
