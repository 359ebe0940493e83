"""The forward pass continued from a given state and returning the final
state (lt_linear_attn_fwd_state), against the fp64 oracle's stateful
recurrent form, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from parity import row_rel_err, state_rel_err, TOL_BF16, TOL_F32, TOL_STATE_BF16, TOL_STATE_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def lt():
    import causal_linear_attention_chunked_b200 as L
    return L




def prefix_state(B, Hkv, d, dv, n, dtype, seed):
    """A plausible (S0, z0): the fp32-rounded final state of a random prefix
    (the oracle's), with the fp64 copy the oracle is given."""
    q, k, v = inputs.make_custom(B, Hkv, Hkv, n, d, dv, dtype, d ** -0.5, seed=seed)
    _, S, z = oracle.fwd_state(q, k, v, causal=True, eps=1e-6)
    S32 = torch.from_numpy(S).float()
    z32 = torch.from_numpy(z).float()
    return S32, z32, S32.double().numpy(), z32.double().numpy()


DENSE = [
    # (B, Hq, Hkv, N, d, dv, causal)
    (2, 4, 2, 300, 64, 64, True),      # three one-chunk blocks
    (1, 2, 2, 3000, 64, 64, True),     # long blocks
    (2, 4, 2, 300, 64, 64, False),
    (1, 8, 2, 517, 128, 128, True),    # GQA, general kernel
    (1, 4, 2, 300, 128, 128, False),
    (1, 2, 2, 260, 64, 128, True),
    (1, 4, 2, 260, 128, 64, True),
]


@pytest.mark.parametrize("case", DENSE, ids=lambda c: "B%dHq%dHkv%dN%dd%ddv%d%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "nc"))
def test_zero_state_matches_forward_bitwise(case):
    """From a zero state the carries are the very sums the forward pass
    forms, in the same order: identical outputs."""
    B, Hq, Hkv, N, d, dv, causal = case
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5, seed=N + d)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    L = lt()
    ref = L.linear_attn_fwd(q, k, v, causal=causal)
    got = L.linear_attn_fwd_state(q, k, v, causal=causal, return_state=False)
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    assert torch.equal(got, ref)


@pytest.mark.parametrize("case", DENSE, ids=lambda c: "B%dHq%dHkv%dN%dd%ddv%d%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "nc"))
def test_from_state_vs_oracle(case):
    B, Hq, Hkv, N, d, dv, causal = case
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5, seed=N + 7)
    S0, z0, S0d, z0d = prefix_state(B, Hkv, d, dv, 200, torch.bfloat16, seed=N + 8)
    ref, S_ref, z_ref = oracle.fwd_state(q, k, v, causal=causal, eps=1e-6, S0=S0d, z0=z0d)
    L = lt()
    out, S, z = L.linear_attn_fwd_state(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                                        S0=S0.cuda(), z0=z0.cuda())
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16
    assert state_rel_err(S.cpu().numpy(), S_ref) <= TOL_STATE_BF16
    assert state_rel_err(z.cpu().numpy()[..., None], z_ref[..., None]) <= TOL_STATE_BF16


@pytest.mark.parametrize("d,dv", [(64, 64), (128, 128)])
@pytest.mark.parametrize("n1", [1, 128, 700])
def test_split_continuation(d, dv, n1):
    """Cut a sequence, continue the second part from the first part's final
    state: the outputs are those of the uncut sequence (oracle)."""
    B, Hq, Hkv, N = 2, 4, 2, 1000
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5, seed=n1)
    ref = oracle.fwd_recurrent(q, k, v, causal=True, eps=1e-6)
    L = lt()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1, S1, z1 = L.linear_attn_fwd_state(qc[:, :n1].contiguous(), kc[:, :n1].contiguous(),
                                         vc[:, :n1].contiguous())
    o2, S2, z2 = L.linear_attn_fwd_state(qc[:, n1:].contiguous(), kc[:, n1:].contiguous(),
                                         vc[:, n1:].contiguous(), S0=S1, z0=z1)
    _, S_all, z_all = L.linear_attn_fwd_state(qc, kc, vc)
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    got = torch.cat([o1, o2], dim=1).float().cpu().numpy()
    assert row_rel_err(got, ref) <= TOL_BF16
    _, S_ref, _ = oracle.fwd_state(q, k, v, causal=True, eps=1e-6)
    assert state_rel_err(S2.cpu().numpy(), S_ref) <= TOL_STATE_BF16
    assert state_rel_err(S_all.cpu().numpy(), S_ref) <= TOL_STATE_BF16


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prefill_then_decode(dtype):
    """The final state of a prefill seeds the decode step: the decoded rows
    equal the causal forward pass over prefill + decoded tokens (oracle)."""
    B, Hq, Hkv, N, T, d, dv = 3, 8, 2, 333, 4, 64, 64
    scale = d ** -0.5 if dtype == torch.bfloat16 else 1.0
    q, k, v = inputs.make_custom(B, Hq, Hkv, N + T, d, dv, dtype, scale, seed=91)
    ref = oracle.fwd_recurrent(q, k, v, causal=True, eps=1e-6)
    L = lt()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    _, S, z = L.linear_attn_fwd_state(qc[:, :N].contiguous(), kc[:, :N].contiguous(),
                                      vc[:, :N].contiguous())
    tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_F32
    for t in range(T):
        o = L.linear_attn_decode_step(qc[:, N + t].contiguous(), kc[:, N + t].contiguous(),
                                      vc[:, N + t].contiguous(), S, z)
        torch.cuda.synchronize()
        assert row_rel_err(o.float().cpu().numpy(), ref[:, N + t]) <= tol
    assert L.get_last_device_error() == 0


@pytest.mark.parametrize("d,dv,causal", [(64, 64, True), (64, 64, False), (128, 128, True),
                                         (128, 128, False)])
def test_packed_with_empty_sequence(d, dv, causal):
    """Packed sequences, one of them empty: per-sequence states; the empty
    sequence returns its initial state unchanged."""
    lens = [130, 0, 257, 5]
    Hq, Hkv = 4, 2
    w = inputs.Workload("t", len(lens), Hq, Hkv, 0, d, dv, torch.bfloat16, d ** -0.5, causal,
                        sum(lens))
    q, k, v, cu = inputs.make(w, lengths=lens)
    S0, z0, S0d, z0d = prefix_state(len(lens), Hkv, d, dv, 150, torch.bfloat16, seed=5)
    ref, S_ref, z_ref = oracle.fwd_state(q, k, v, causal=causal, eps=1e-6, cu_seqlens=cu.numpy(),
                                         S0=S0d, z0=z0d)
    L = lt()
    out, S, z = L.linear_attn_fwd_state(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                                        cu_seqlens=cu.cuda(), S0=S0.cuda(), z0=z0.cuda())
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16
    assert state_rel_err(S.cpu().numpy(), S_ref) <= TOL_STATE_BF16
    assert torch.equal(S[1].cpu(), S0[1]) and torch.equal(z[1].cpu(), z0[1])


@pytest.mark.parametrize("causal", [True, False])
def test_f32_from_state_vs_oracle(causal):
    B, Hq, Hkv, N, d, dv = 2, 4, 2, 100, 64, 64
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.float32, 1.0, seed=17)
    S0, z0, S0d, z0d = prefix_state(B, Hkv, d, dv, 50, torch.float32, seed=18)
    ref, S_ref, z_ref = oracle.fwd_state(q, k, v, causal=causal, eps=1e-6, S0=S0d, z0=z0d)
    L = lt()
    out, S, z = L.linear_attn_fwd_state(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                                        S0=S0.cuda(), z0=z0.cuda())
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    assert row_rel_err(out.cpu().numpy(), ref) <= TOL_F32
    assert state_rel_err(S.cpu().numpy(), S_ref) <= TOL_STATE_F32
    assert state_rel_err(z.cpu().numpy()[..., None], z_ref[..., None]) <= TOL_STATE_F32
