"""Context parallelism host logic on the CPU: two gloo ranks each hold one
segment of every sequence; the exchange of segment states, the rank-ordered
carry and the second pass must reproduce attention over the whole sequence.
The oracle's stateful form stands in for the GPU kernel here (test only)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, N, HQ, HKV, D, DV = 2, 61, 4, 2, 8, 6
CUT = 25  # rank 0 holds tokens [0, CUT), rank 1 the rest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = np.random.default_rng(123)
    return (g.standard_normal((B, N, HQ, D)), g.standard_normal((B, N, HKV, D)),
            g.standard_normal((B, N, HKV, DV)))


def _oracle_fwd_state(q, k, v, causal=True, eps=1e-6, S0=None, z0=None, return_state=True):
    """The stateful forward on the CPU, states rounded to fp32 as the GPU's."""
    import torch
    import oracle
    out, S, z = oracle.fwd_state(q.numpy(), k.numpy(), v.numpy(), causal=causal, eps=eps,
                                 S0=None if S0 is None else S0.double().numpy(),
                                 z0=None if z0 is None else z0.double().numpy())
    out = torch.from_numpy(out)
    if not return_state:
        return out
    return out, torch.from_numpy(S).float(), torch.from_numpy(z).float()


def _rank_main(rank, world, port, out_dir, causal):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    from causal_linear_attention_chunked_b200.context_parallel import linear_attn_fwd_cp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x[:, :CUT] if rank == 0 else x[:, CUT:]))
               for x in _inputs())
    out = linear_attn_fwd_cp(q, k, v, causal=causal, eps=1e-6, fwd_state=_oracle_fwd_state)
    np.save(os.path.join(out_dir, "rank%d.npy" % rank), out.numpy())
    dist.destroy_process_group()


@pytest.mark.parametrize("causal", [True, False])
def test_two_rank_context_parallel(tmp_path, causal):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), causal))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    got = np.concatenate([np.load(tmp_path / ("rank%d.npy" % r)) for r in range(world)], axis=1)
    ref = oracle.fwd_quadratic(*_inputs(), causal=causal, eps=1e-6)
    # the exchanged states are fp32: relative error of the order of 1e-7
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
