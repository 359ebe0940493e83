"""Context parallelism host logic on the CPU: gloo ranks each hold one
segment of every sequence; the exchange of segment states, the rank-ordered
carry and the second pass must reproduce attention over the whole sequence.
The oracle stands in for the CUDA library's three steps here (test only);
the GPU run of the same function through the library is in
test_gpu_context_parallel.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, N, HQ, HKV, D, DV = 2, 61, 4, 2, 8, 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = np.random.default_rng(123)
    return (g.standard_normal((B, N, HQ, D)), g.standard_normal((B, N, HKV, D)),
            g.standard_normal((B, N, HKV, DV)))


class OracleOps:
    """The library's three steps restated with the oracle (CPU, fp64 math,
    states rounded to fp32 as the library returns them)."""

    def state(self, k, v):
        import torch
        import oracle
        _, S, z = oracle.fwd_state(k.numpy(), k.numpy(), v.numpy(), causal=True, eps=1e-6)
        return torch.from_numpy(S).float(), torch.from_numpy(z).float()

    def carry(self, S_all, z_all, rank, causal):
        sel = [r for r in range(S_all.shape[0]) if (r < rank if causal else r != rank)]
        S0, z0 = S_all[0] * 0, z_all[0] * 0
        for r in sel:
            S0 = S0 + S_all[r]
            z0 = z0 + z_all[r]
        return S0, z0

    def fwd_state(self, q, k, v, causal, eps, S0, z0):
        import torch
        import oracle
        out, _, _ = oracle.fwd_state(q.numpy(), k.numpy(), v.numpy(), causal=causal, eps=eps,
                                     S0=S0.double().numpy(), z0=z0.double().numpy())
        return torch.from_numpy(out)


def _rank_main(rank, world, port, out_dir, causal, cuts):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    from causal_linear_attention_chunked_b200.context_parallel import linear_attn_fwd_cp
    from test_context_parallel import OracleOps
    dist.init_process_group("gloo", rank=rank, world_size=world)
    lo, hi = cuts[rank], cuts[rank + 1]
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x[:, lo:hi])) for x in _inputs())
    out = linear_attn_fwd_cp(q, k, v, causal=causal, eps=1e-6, ops=OracleOps())
    assert out.shape == (B, hi - lo, HQ, DV)
    np.save(os.path.join(out_dir, "rank%d.npy" % rank), out.numpy())
    dist.destroy_process_group()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("cuts", [(0, 25, N), (0, 20, 20, N)], ids=["2ranks", "3ranks_empty"])
def test_context_parallel_ranks(tmp_path, causal, cuts):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    world, port = len(cuts) - 1, _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), causal, cuts))
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
