"""The benchmark workloads at full size, in the launch configuration the
benchmark times: outputs checked against the oracle on sampled rows (first
and last rows, chunk boundaries, random rows), and on every row against
properties that hold at any size (finite; inside the hull of the values
seen so far)."""
import numpy as np
import pytest
import torch

import oracle
from parity import row_rel_err, TOL_BF16, TOL_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def sample_rows(n_seq_lens, Hq, rng, per_seq=12):
    rows = []
    for s, n in enumerate(n_seq_lens):
        if n == 0:
            continue
        cand = {0, n - 1, min(127, n - 1), min(128, n - 1), min(129, n - 1), n // 2}
        cand |= set(int(x) for x in rng.integers(0, n, per_seq))
        for i in sorted(cand):
            rows.append((s, i, int(rng.integers(0, Hq))))
    return np.array(rows, dtype=np.int64)


def check_hull(out, v, Hq, Hkv, causal, cu=None):
    """Every output lies (up to the bf16 output rounding and eps) inside the
    per-column [min, max] of the values it averages."""
    G = Hq // Hkv
    if cu is None:
        vv = v.float()
        if causal:
            hi = torch.cummax(vv, dim=1).values
            lo = torch.cummin(vv, dim=1).values
        else:
            hi = vv.max(dim=1, keepdim=True).values.expand_as(vv)
            lo = vv.min(dim=1, keepdim=True).values.expand_as(vv)
        hi = hi.repeat_interleave(G, dim=2)
        lo = lo.repeat_interleave(G, dim=2)
        o = out.float()
        slack = 1e-2 * (hi.abs().amax(dim=-1, keepdim=True) + 1e-6)
        assert torch.isfinite(o).all()
        assert (o <= hi + slack).all() and (o >= lo - slack).all()


@pytest.mark.parametrize("name", ["bf16_b2h8n4096d64", "bf16_b1h8n65536d64",
                                  "bf16_b1h8n65536d64_noncausal", "bf16_gqa_b2hq32hkv8n16384d128",
                                  "bf16_varlen64_h8d64"])
def test_workload_full_size(name):
    import causal_linear_attention_chunked_b200 as L
    w = inputs.WORKLOADS[name]
    q, k, v, cu = inputs.make(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cud = cu.cuda() if cu is not None else None
    out = L.linear_attn_fwd(qd, kd, vd, causal=w.causal, eps=w.eps, cu_seqlens=cud)
    assert L.get_last_device_error() == 0
    rng = np.random.default_rng(w.seed)
    if cu is None:
        lens = [w.N] * w.B
    else:
        lens = (cu[1:] - cu[:-1]).tolist()
    rows = sample_rows(lens, w.Hq, rng)
    ref = oracle.fwd_rows(q, k, v, rows, causal=w.causal, eps=w.eps,
                          cu_seqlens=None if cu is None else cu.numpy())
    o = out.float().cpu()
    if cu is None:
        got = np.stack([o[s, i, h].numpy() for s, i, h in rows])
    else:
        got = np.stack([o[int(cu[s]) + i, h].numpy() for s, i, h in rows])
    err = row_rel_err(got, ref)
    assert err <= TOL_BF16, err
    if cu is None:
        check_hull(out, vd, w.Hq, w.Hkv, w.causal)
    else:
        assert torch.isfinite(out).all()


def test_fp32_workload_full_size():
    import causal_linear_attention_chunked_b200 as L
    w = inputs.WORKLOADS["fp32_b1h1n256d64"]
    q, k, v, _ = inputs.make(w)
    out = L.linear_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, eps=w.eps)
    ref = oracle.fwd_quadratic(q, k, v, causal=True, eps=w.eps)
    assert row_rel_err(out.cpu().numpy(), ref) <= TOL_F32
