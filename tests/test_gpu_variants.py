"""The forward pass's variants on the GPU against the oracle, element by
element: fp16 inputs and outputs (tensor cores on bf16 operands), and the
ReLU and exp feature maps (lt_linear_attn_fwd_ex) in every dtype; causal and
non-causal, GQA, d = dv = 64 and 128, ragged tails, several blocks, packed
sequences with empty ones.  Bars: 2e-2 for the 16-bit dtypes, 1e-4 for fp32
(the row metric of the forward tests)."""
import pytest
import torch

import oracle
from parity import row_rel_err, TOL_BF16, TOL_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def L():
    import causal_linear_attention_chunked_b200 as lt
    return lt


CASES = [
    # (B, Hq, Hkv, N, d, causal)
    (1, 2, 2, 200, 64, True),
    (2, 8, 2, 1000, 64, True),      # GQA, several blocks, ragged tail
    (1, 4, 4, 3000, 64, False),
    (1, 4, 2, 700, 128, True),
    (2, 2, 2, 300, 128, False),
]


def _run(q, k, v, causal, phi, cu=None):
    out = L().linear_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, feature_map=phi,
                              cu_seqlens=None if cu is None else cu.cuda())
    torch.cuda.synchronize()
    assert L().get_last_device_error() == 0
    return out


@pytest.mark.parametrize("phi", ["elu1", "relu", "exp"])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32],
                         ids=["f16", "bf16", "f32"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dN%dd%d%s" % (
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "nc"))
def test_variant_dense_vs_oracle(case, dtype, phi):
    B, Hq, Hkv, N, d, causal = case
    scale = 1.0 if dtype == torch.float32 else d ** -0.5
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, d, dtype, scale, seed=N + d)
    out = _run(q, k, v, causal, phi)
    assert out.dtype == dtype
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6, phi=phi)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert row_rel_err(out.float().cpu().numpy(), ref) <= tol


@pytest.mark.parametrize("phi", ["elu1", "relu"])
def test_variant_packed_fp16(phi):
    lens = [300, 0, 1, 129, 1000]
    cu = inputs.cu_from_lengths(lens)
    T, Hq, Hkv, d = int(cu[-1]), 4, 2, 64
    g = inputs.generator(17)
    q, k, v = ((torch.randn(sh, generator=g) * 0.125).half() for sh in
               ((T, Hq, d), (T, Hkv, d), (T, Hkv, d)))
    for causal in (True, False):
        out = _run(q, k, v, causal, phi, cu=cu)
        ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6, cu_seqlens=cu.numpy(),
                                   phi=phi)
        assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16


def test_fp16_keeps_its_range_on_long_sequences():
    """At 65536 tokens the normaliser z grows past fp16's largest value
    (65504); the tensor-core operands are bf16, so the fp16 path still
    returns finite outputs that match the oracle (sampled rows)."""
    import numpy as np
    B, Hq, Hkv, N, d = 1, 2, 2, 65536, 64
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, d, torch.float16, 0.125, seed=23)
    out = _run(q, k, v, True, "elu1")
    assert torch.isfinite(out).all()
    rows = np.array([(0, i, h) for i in (0, 127, 128, 30000, 65535) for h in range(Hq)])
    ref = oracle.fwd_rows(q, k, v, rows, causal=True, eps=1e-6)
    got = out.float().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert row_rel_err(got, ref) <= TOL_BF16
