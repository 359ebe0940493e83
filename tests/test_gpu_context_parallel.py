"""Context parallelism through the CUDA library on one GPU.

* The state without outputs (lt_linear_attn_state) and the rank-ordered
  carry (lt_linear_attn_state_carry) against the oracle.
* Segments of one sequence run one after another on this GPU, as the ranks
  would run them: each segment's state, the carry of every rank from the
  gathered states, each segment's outputs from its carry -- together they
  must equal attention over the whole sequence (oracle), causal and not,
  with GQA and an empty segment.
* linear_attn_fwd_cp itself in a one-rank NCCL process group, on the
  current stream and on a side stream.
The multi-rank host logic (gloo, several processes) is in
test_context_parallel.py; this box has one GPU per call."""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle
from parity import row_rel_err, state_rel_err, TOL_BF16, TOL_F32, TOL_STATE_BF16, TOL_STATE_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def L():
    import causal_linear_attention_chunked_b200 as lt
    return lt


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(2, 4, 2, 1000, 64, 64), (1, 2, 2, 3000, 128, 128),
                                   (1, 2, 1, 700, 64, 128)])
def test_state_only_matches_oracle(dtype, shape):
    B, Hq, Hkv, N, d, dv = shape
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, dtype, d ** -0.5, seed=N + d)
    g = inputs.generator(5)
    S0 = torch.rand((B, Hkv, d, dv), generator=g)
    z0 = torch.rand((B, Hkv, d), generator=g)
    S, z = L().linear_attn_state(k.cuda(), v.cuda(), S0=S0.cuda(), z0=z0.cuda())
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    _, Sr, zr = oracle.fwd_state(q, k, v, causal=True, S0=S0.double().numpy(),
                                 z0=z0.double().numpy())
    tol = TOL_STATE_F32 if dtype == torch.float32 else TOL_STATE_BF16
    assert state_rel_err(S.cpu().numpy(), Sr) <= tol
    assert state_rel_err(z.cpu().numpy()[..., None], zr[..., None]) <= tol


def test_state_only_packed_with_empty_sequence():
    lens = [300, 0, 129, 1]
    cu = inputs.cu_from_lengths(lens)
    T, Hkv, d = int(cu[-1]), 2, 64
    g = inputs.generator(11)
    k = (torch.randn((T, Hkv, d), generator=g) * 0.125).to(torch.bfloat16)
    v = (torch.randn((T, Hkv, d), generator=g) * 0.125).to(torch.bfloat16)
    S, z = L().linear_attn_state(k.cuda(), v.cuda(), cu_seqlens=cu.cuda())
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    _, Sr, zr = oracle.fwd_state(k, k, v, causal=True, cu_seqlens=cu.numpy())
    nz = [0, 2, 3]  # the non-empty sequences; the empty one has a zero state
    assert state_rel_err(S.cpu().numpy()[nz], Sr[nz]) <= TOL_STATE_BF16
    assert state_rel_err(z.cpu().numpy()[nz][..., None], zr[nz][..., None]) <= TOL_STATE_BF16
    assert float(S[1].abs().max()) == 0.0 and float(z[1].abs().max()) == 0.0


@pytest.mark.parametrize("causal", [True, False])
def test_carry_sums_in_rank_order(causal):
    world, B, Hkv, d, dv = 5, 2, 3, 64, 128
    g = inputs.generator(21)
    S_all = torch.randn((world, B, Hkv, d, dv), generator=g)
    z_all = torch.randn((world, B, Hkv, d), generator=g)
    for rank in range(world):
        S0, z0 = L().linear_attn_state_carry(S_all.cuda(), z_all.cuda(), rank, causal=causal)
        sel = [r for r in range(world) if (r < rank if causal else r != rank)]
        Sr = sum((S_all[r].double() for r in sel), torch.zeros_like(S_all[0], dtype=torch.float64))
        zr = sum((z_all[r].double() for r in sel), torch.zeros_like(z_all[0], dtype=torch.float64))
        assert torch.allclose(S0.cpu().double(), Sr, rtol=0, atol=1e-5)
        assert torch.allclose(z0.cpu().double(), zr, rtol=0, atol=1e-5)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("cuts", [(0, 1500, 4000), (0, 999, 999, 2500, 4000)],
                         ids=["2seg", "4seg_empty"])
def test_segments_reproduce_the_whole_sequence(causal, dtype, cuts):
    B, Hq, Hkv, N, d, dv = 2, 8, 2, 4000, 64, 64
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, dtype, d ** -0.5, seed=77)
    world = len(cuts) - 1
    segs = [tuple(x[:, cuts[r]:cuts[r + 1]].contiguous().cuda() for x in (q, k, v))
            for r in range(world)]
    states = []
    for (qs, ks, vs) in segs:
        if ks.shape[1] == 0:
            states.append((torch.zeros((B, Hkv, d, dv), device="cuda"),
                           torch.zeros((B, Hkv, d), device="cuda")))
        else:
            states.append(L().linear_attn_state(ks, vs))
    S_all = torch.stack([s for s, _ in states])
    z_all = torch.stack([z for _, z in states])
    outs = []
    for r, (qs, ks, vs) in enumerate(segs):
        S0, z0 = L().linear_attn_state_carry(S_all, z_all, r, causal=causal)
        if qs.shape[1] == 0:
            continue
        outs.append(L().linear_attn_fwd_state(qs, ks, vs, causal=causal, S0=S0, z0=z0,
                                              return_state=False))
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    got = torch.cat(outs, dim=1).float().cpu().numpy()
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert row_rel_err(got, ref) <= tol


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture
def one_rank_group():
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        yield
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("side_stream", [False, True])
def test_fwd_cp_one_rank_nccl(one_rank_group, side_stream):
    from causal_linear_attention_chunked_b200.context_parallel import linear_attn_fwd_cp
    B, Hq, Hkv, N, d, dv = 2, 8, 8, 3000, 64, 64
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, 0.125, seed=31)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    s = torch.cuda.Stream() if side_stream else None
    if s is not None:
        s.wait_stream(torch.cuda.current_stream())
    out = linear_attn_fwd_cp(qd, kd, vd, causal=True, stream=s)
    if s is not None:
        torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    ref = oracle.fwd_recurrent(q, k, v, causal=True, eps=1e-6)
    assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16
