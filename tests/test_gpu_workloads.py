"""The benchmark workloads at full size, in the launch configuration the
benchmark times.

Every output row is compared with the oracle's recurrent form (fp64, the
form pinned against the quadratic definition on small inputs).  Two further
witnesses: sampled rows (first and last rows, chunk boundaries, random rows)
against the quadratic definition itself, and the convex-hull bound on every
row (each output is a weighted average of the values seen so far, so it lies
inside their per-column range), per sequence for packed inputs."""
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


def _hull_bounds(vv, causal):
    """Per-column [min, max] of the values each row averages; vv [N, H, dv]."""
    if causal:
        return torch.cummin(vv, dim=0).values, torch.cummax(vv, dim=0).values
    lo = vv.min(dim=0, keepdim=True).values.expand_as(vv)
    hi = vv.max(dim=0, keepdim=True).values.expand_as(vv)
    return lo, hi


def check_hull(out, v, Hq, Hkv, causal, cu=None):
    """Every output lies (up to the bf16 output rounding and eps) inside the
    per-column [min, max] of the values it averages."""
    G = Hq // Hkv
    o_all = out.float()
    assert torch.isfinite(o_all).all()
    if cu is None:
        segs = [(o_all[b], v[b].float()) for b in range(out.shape[0])]
    else:
        c = cu.tolist()
        segs = [(o_all[c[s]:c[s + 1]], v[c[s]:c[s + 1]].float())
                for s in range(len(c) - 1) if c[s + 1] > c[s]]
    for o, vv in segs:
        lo, hi = _hull_bounds(vv, causal)
        hi = hi.repeat_interleave(G, dim=1)
        lo = lo.repeat_interleave(G, dim=1)
        slack = 1e-2 * (hi.abs().amax(dim=-1, keepdim=True) + 1e-6)
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
    cu_np = None if cu is None else cu.numpy()
    o = out.float().cpu()

    # every row against the recurrent form
    ref = oracle.fwd_recurrent(q, k, v, causal=w.causal, eps=w.eps, cu_seqlens=cu_np)
    err_all = row_rel_err(o.numpy(), ref)
    assert err_all <= TOL_BF16, err_all
    del ref

    # sampled rows against the quadratic definition
    rng = np.random.default_rng(w.seed)
    lens = [w.N] * w.B if cu is None else (cu[1:] - cu[:-1]).tolist()
    rows = sample_rows(lens, w.Hq, rng)
    ref_rows = oracle.fwd_rows(q, k, v, rows, causal=w.causal, eps=w.eps, cu_seqlens=cu_np)
    if cu is None:
        got = np.stack([o[s, i, h].numpy() for s, i, h in rows])
    else:
        got = np.stack([o[int(cu[s]) + i, h].numpy() for s, i, h in rows])
    err = row_rel_err(got, ref_rows)
    assert err <= TOL_BF16, err

    check_hull(out, vd, w.Hq, w.Hkv, w.causal, cu=cu)


def test_fp32_workload_full_size():
    import causal_linear_attention_chunked_b200 as L
    w = inputs.WORKLOADS["fp32_b1h1n256d64"]
    q, k, v, _ = inputs.make(w)
    out = L.linear_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, eps=w.eps)
    ref = oracle.fwd_quadratic(q, k, v, causal=True, eps=w.eps)
    assert row_rel_err(out.cpu().numpy(), ref) <= TOL_F32
    ref = oracle.fwd_recurrent(q, k, v, causal=True, eps=w.eps)
    assert row_rel_err(out.cpu().numpy(), ref) <= TOL_F32
