"""GPU forward pass against the fp64 oracle, element by element, on seeded
inputs that span several 128-token chunks and a ragged tail (bf16) or
several 32-token chunks (fp32).  Every call goes through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import pins
from parity import row_rel_err, tol_for, TOL_BF16, TOL_F32
from causal_linear_attention_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def lt():
    import causal_linear_attention_chunked_b200 as L
    return L


def run_dense(q, k, v, causal, eps=1e-6):
    L = lt()
    out = L.linear_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, eps=eps)
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    return out.float().cpu().numpy()


DENSE_CASES = [
    # (B, Hq, Hkv, N, d, dv, causal)
    (1, 1, 1, 1, 64, 64, True),
    (1, 2, 2, 127, 64, 64, True),
    (2, 2, 2, 128, 64, 64, True),
    (1, 1, 1, 129, 64, 64, True),
    (2, 3, 3, 3 * 128 + 5, 64, 64, True),
    (1, 8, 2, 600, 64, 64, True),
    (1, 4, 1, 1000, 64, 64, False),
    (2, 2, 2, 257, 64, 64, False),
    (1, 4, 4, 300, 128, 128, True),
    (1, 8, 2, 517, 128, 128, True),
    (1, 4, 2, 300, 128, 128, False),
    (1, 2, 2, 300, 64, 128, True),
    (1, 4, 2, 260, 128, 64, True),
    (1, 2, 1, 200, 64, 128, False),
]


@pytest.mark.parametrize("case", DENSE_CASES, ids=lambda c: "B%dHq%dHkv%dN%dd%ddv%d%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "nc"))
def test_bf16_dense_vs_oracle(case):
    B, Hq, Hkv, N, d, dv, causal = case
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5, seed=hash(case) % 1000)
    got = run_dense(q, k, v, causal)
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
    err = row_rel_err(got, ref)
    assert err <= TOL_BF16, err


@pytest.mark.parametrize("scale", [1.0, 3.0])
def test_bf16_large_magnitude_inputs(scale):
    """sigma = 1 and 3: phi underflows for very negative inputs, scores spread."""
    q, k, v = inputs.make_custom(1, 4, 4, 700, 64, 64, torch.bfloat16, scale, seed=77)
    for causal in (True, False):
        got = run_dense(q, k, v, causal)
        ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
        assert row_rel_err(got, ref) <= TOL_BF16


@pytest.mark.parametrize("case", [
    (1, 1, 1, 256, 64, 64, True),   # the fp32 workload's shape
    (2, 4, 2, 100, 64, 64, True),
    (1, 2, 2, 77, 128, 128, False),
    (1, 2, 1, 65, 64, 128, True),
])
def test_f32_vs_oracle(case):
    B, Hq, Hkv, N, d, dv, causal = case
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.float32, 1.0, seed=N)
    got = run_dense(q, k, v, causal)
    ref = oracle.fwd_quadratic(q, k, v, causal=causal, eps=1e-6)
    assert row_rel_err(got, ref) <= TOL_F32


def test_f32_workload_full():
    w = inputs.WORKLOADS["fp32_b1h1n256d64"]
    q, k, v, _ = inputs.make(w)
    got = run_dense(q, k, v, True, w.eps)
    ref = oracle.fwd_quadratic(q, k, v, causal=True, eps=w.eps)
    assert row_rel_err(got, ref) <= TOL_F32


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dd", [(64, 64), (128, 128)])
def test_hand_example_on_gpu(dtype, dd):
    """The exact 3-token example of tests/golden/hand_3tok_exact.json."""
    q, k, v, g = pins.hand_3tok_inputs(d=dd[0], dv=dd[1], dtype=dtype)
    for causal, key in ((True, "causal_eps0_first3cols"), (False, "noncausal_eps0_first3cols")):
        got = run_dense(q, k, v, causal, eps=0.0)[0, :, 0]
        tol = 1e-6 if dtype == torch.float32 else 4e-3
        assert np.abs(got[:, :3] - np.array(g[key])).max() <= tol
        assert np.all(got[:, 3:] == 0.0)


VARLEN_CASES = [
    ([1, 127, 128, 129, 300], 2, 2, 64, 64, True),
    ([0, 5, 0, 260, 1], 4, 2, 64, 64, True),
    ([200, 0, 131], 4, 4, 64, 64, False),
    ([130, 7, 257], 8, 2, 128, 128, True),
    ([64, 300], 2, 1, 128, 128, False),
]


@pytest.mark.parametrize("case", VARLEN_CASES, ids=lambda c: "L%s_Hq%dHkv%d_d%d_%s" % (
    "-".join(map(str, c[0])), c[1], c[2], c[3], "c" if c[5] else "nc"))
def test_bf16_packed_vs_oracle(case):
    lens, Hq, Hkv, d, dv, causal = case
    w = inputs.Workload("t", len(lens), Hq, Hkv, 0, d, dv, torch.bfloat16, d ** -0.5, causal,
                        sum(lens))
    q, k, v, cu = inputs.make(w, lengths=lens)
    L = lt()
    out = L.linear_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, eps=1e-6,
                            cu_seqlens=cu.cuda())
    assert L.get_last_device_error() == 0
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6, cu_seqlens=cu.numpy())
    assert row_rel_err(out.float().cpu().numpy(), ref) <= TOL_BF16


def test_bf16_deterministic():
    q, k, v = inputs.make_custom(2, 4, 2, 1111, 64, 64, torch.bfloat16, 0.125, seed=5)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    L = lt()
    a = L.linear_attn_fwd(q, k, v)
    b = L.linear_attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("case", DENSE_CASES[:8], ids=lambda c: "B%dHq%dHkv%dN%d%s" % (
    c[0], c[1], c[2], c[3], "c" if c[6] else "nc"))
def test_sequential_kernel_forced(sched, case):
    """The general kernel run fully sequentially (one CTA per (sequence,
    KV head)) on the d = dv = 64 shapes the specialised kernel normally
    takes."""
    sched(kernel="general")
    sched(blocks=1)
    B, Hq, Hkv, N, d, dv, causal = case
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5, seed=N)
    got = run_dense(q, k, v, causal)
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
    assert row_rel_err(got, ref) <= TOL_BF16


def test_block_and_general_kernels_agree_closely(sched):
    """The two kernels differ only in rounding order (state operand, bf16
    output rounding of each); two independent bf16 roundings of the same
    value can differ by 2 ulp (0.78% of an entry), so their outputs must
    agree to 1e-2 in the row metric, well inside the 2e-2 bar."""
    q, k, v = inputs.make_custom(2, 8, 8, 4096, 64, 64, torch.bfloat16, 0.125, seed=9)
    a = run_dense(q, k, v, True)
    sched(kernel="general")
    b = run_dense(q, k, v, True)
    assert row_rel_err(a, b) <= 1e-2


BLOCK_CASES = [
    # (B, Hq, Hkv, N, causal)
    (1, 2, 2, 1000, True),      # 8 chunks, ragged tail
    (2, 4, 2, 777, True),       # GQA
    (1, 1, 1, 2049, False),     # 17 chunks, non-causal
    (1, 2, 1, 130, True),       # 2 chunks: more blocks requested than chunks
    (1, 3, 3, 3 * 128 * 5 + 7, True),  # uneven blocks and a ragged last chunk
    (2, 2, 2, 1500, False),
]


@pytest.mark.parametrize("mode", ["auto", "pair"])
@pytest.mark.parametrize("nb", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("case", BLOCK_CASES, ids=lambda c: "B%dHq%dHkv%dN%d%s" % (
    c[0], c[1], c[2], c[3], "c" if c[4] else "nc"))
def test_block_kernel_block_counts(sched, nb, case, mode):
    """d = dv = 64, the sequence cut into nb blocks (schedule override).
    "pair": the block aggregates in a first launch, then one CTA per block
    from the carried prefix.  "auto": blocks of at most four chunks run as
    one cooperative launch whose blocks exchange their aggregates through the
    workspace; other shapes as "pair"."""
    sched(blocks=nb)
    if mode == "pair":
        sched(kernel="two_launch")
    else:
        sched(kernel="auto")
    B, Hq, Hkv, N, causal = case
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, 64, 64, torch.bfloat16, 0.125, seed=N + 7 * nb)
    got = run_dense(q, k, v, causal)
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
    assert row_rel_err(got, ref) <= TOL_BF16


FUSED_CASES = [
    # (B, Hq, Hkv, N, causal, forced block count or 0): one cooperative launch
    # in which the blocks publish and gather the aggregates themselves
    (2, 8, 8, 4096, True, 0),        # B2 H8 N4096: 8 blocks of 4 chunks
    (4, 8, 8, 2000, True, 0),        # 4 blocks of 4 chunks, ragged last chunk
    (1, 4, 4, 7 * 128 + 117, True, 0),  # 8 blocks of 1 chunk
    (2, 4, 1, 1000, True, 0),        # 4 query heads per KV head: 8 blocks of 1 chunk
    (1, 8, 4, 3000, True, 12),       # GQA, 12 blocks of 2 chunks x 2 query heads
    (1, 8, 2, 3000, True, 0),        # GQA, 24 blocks of 1 chunk x 4 query heads
    (1, 2, 2, 1024, False, 0),
    (3, 2, 2, 900, False, 0),
    (1, 4, 2, 1500, False, 6),       # 6 blocks of 2 chunks x 2 query heads
    (1, 4, 1, 1000, False, 0),       # 8 blocks of 1 chunk x 4 query heads
]


@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: "B%dHq%dHkv%dN%d%s%s" % (
    c[0], c[1], c[2], c[3], "c" if c[4] else "nc", "-nb%d" % c[5] if c[5] else ""))
def test_fused_launch_agrees_with_two_launches(sched, case):
    """The one-launch path splits each chunk's starting state into the carry
    of the earlier blocks and the block's own earlier chunks and rounds each
    part to the bf16 operand separately; the two-launch path rounds their sum
    once.  Both match the oracle, and they agree with each other to within
    two bf16 roundings (1e-2 in the row metric)."""
    import causal_linear_attention_chunked_b200 as L
    B, Hq, Hkv, N, causal, nb_forced = case
    sched(kernel="auto")
    if nb_forced:
        sched(blocks=nb_forced)
    else:
        sched(blocks=0)
    nb, launches, ws = L.linear_attn_fwd_plan(B, Hq, Hkv, N, 64, 64, causal=causal)
    assert nb >= 2 and launches == 1 and ws > 0
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, 64, 64, torch.bfloat16, 0.125, seed=N + B)
    one = run_dense(q, k, v, causal)
    sched(kernel="two_launch")
    assert L.linear_attn_fwd_plan(B, Hq, Hkv, N, 64, 64, causal=causal)[1] == 2
    two = run_dense(q, k, v, causal)
    assert row_rel_err(one, two) <= 1e-2
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
    assert row_rel_err(one, ref) <= TOL_BF16
    assert row_rel_err(two, ref) <= TOL_BF16


def test_fused_launch_in_cuda_graph_replays_with_new_inputs(sched):
    """A captured one-launch call replayed with new input contents: each
    replay publishes its own aggregates and meets at its own grid barrier,
    so no replay takes another replay's aggregates for its own."""
    import causal_linear_attention_chunked_b200 as L
    B, Hq, Hkv, N = 2, 8, 8, 4096
    assert L.linear_attn_fwd_plan(B, Hq, Hkv, N, 64, 64, causal=True)[1] == 1
    q, k, v = (t.cuda() for t in inputs.make_custom(B, Hq, Hkv, N, 64, 64, torch.bfloat16,
                                                     0.125, seed=900))
    out = torch.empty((B, N, Hq, 64), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        L.linear_attn_fwd(q, k, v, causal=True, out=out, stream=s)  # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        L.linear_attn_fwd(q, k, v, causal=True, out=out, stream=s)
    for seed in (901, 902, 903):
        q2, k2, v2 = inputs.make_custom(B, Hq, Hkv, N, 64, 64, torch.bfloat16, 0.125, seed=seed)
        q.copy_(q2)
        k.copy_(k2)
        v.copy_(v2)
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert L.get_last_device_error() == 0
        sel = np.array([(b, n, h) for b in range(B) for n in (0, 1, 511, 512, 2047, 2048, 3000, 4095)
                        for h in range(Hq)])
        ref = oracle.fwd_rows(q2, k2, v2, sel, causal=True, eps=1e-6)
        o = out.float().cpu().numpy()
        got = o[sel[:, 0], sel[:, 1], sel[:, 2]]
        assert row_rel_err(got, ref) <= TOL_BF16


def test_fused_launch_many_back_to_back(sched):
    """Forty one-launch calls in a row on one stream, alternating two input
    sets without synchronising: each meets the grid barrier of its own
    launch, so every output equals the first output of its input set."""
    import causal_linear_attention_chunked_b200 as L
    B, Hq, Hkv, N = 2, 8, 8, 4096
    assert L.linear_attn_fwd_plan(B, Hq, Hkv, N, 64, 64, causal=True)[1] == 1
    sets = [tuple(t.cuda() for t in inputs.make_custom(B, Hq, Hkv, N, 64, 64, torch.bfloat16,
                                                      0.125, seed=sd)) for sd in (31, 32)]
    outs = [L.linear_attn_fwd(*sets[i % 2], causal=True) for i in range(40)]
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    for i, o in enumerate(outs):
        assert torch.equal(o, outs[i % 2]), i
    assert not torch.equal(outs[0], outs[1])


def test_block_kernel_deterministic_across_block_counts(sched):
    """Every block count computes the same function; results agree to a few
    bf16 ulps (only the summation order of the carried state differs)."""
    q, k, v = inputs.make_custom(1, 4, 4, 3000, 64, 64, torch.bfloat16, 0.125, seed=4)
    outs = []
    for nb in (1, 4, 12):
        sched(blocks=nb)
        outs.append(run_dense(q, k, v, True))
    for o in outs[1:]:
        assert row_rel_err(o, outs[0]) <= 1e-2


GENERAL_BLOCK_CASES = [
    # (B, Hq, Hkv, N, d, dv, causal)
    (1, 4, 2, 1000, 128, 128, True),   # GQA, ragged tail
    (2, 2, 2, 777, 128, 128, False),
    (1, 2, 2, 1300, 64, 128, True),
    (1, 4, 2, 900, 128, 64, True),
    (1, 2, 1, 1100, 64, 128, False),
    (1, 4, 4, 1200, 64, 64, True),     # the general kernel on d = dv = 64
]


@pytest.mark.parametrize("nb", [1, 2, 3, 5])
@pytest.mark.parametrize("case", GENERAL_BLOCK_CASES, ids=lambda c: "B%dHq%dHkv%dN%dd%ddv%d%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "nc"))
def test_general_kernel_block_counts(sched, nb, case):
    """The general kernel (every width pair) with the sequence cut into nb
    blocks: the state launch's block aggregates are summed into the carry
    each block starts from (written into its TMEM state accumulator when
    causal, used as the whole state when not)."""
    sched(kernel="general")
    sched(blocks=nb)
    B, Hq, Hkv, N, d, dv, causal = case
    q, k, v = inputs.make_custom(B, Hq, Hkv, N, d, dv, torch.bfloat16, d ** -0.5,
                                 seed=N + 11 * nb)
    got = run_dense(q, k, v, causal)
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
    assert row_rel_err(got, ref) <= TOL_BF16


# A ragged last chunk loads the next packed sequence's (or the next batch
# row's) first rows into its tiles, and the kernels zero those rows before any
# product.  Here that neighbour holds NaN and Inf: every other sequence must
# still match the oracle on clean data, with no non-finite output.  Covers the
# one-launch kernel (dense d = dv = 64, three one-chunk blocks), the block
# kernel (packed d = dv = 64), the general kernel (d = dv = 128, packed and
# blocked) and the state launch (dense d = 128, non-causal aggregates).
ISOLATION_CASES = [
    # (layout, lengths, Hq, Hkv, d, dv, causal); dense layout: B = 2, N = lengths
    ("packed", [130, 200, 77], 4, 2, 64, 64, True),
    ("packed", [130, 200, 77], 4, 2, 64, 64, False),
    ("packed", [130, 200, 77], 4, 2, 128, 128, True),
    ("packed", [130, 200, 77], 4, 2, 128, 128, False),
    ("dense", 300, 4, 2, 64, 64, True),
    ("dense", 300, 4, 2, 64, 64, False),
    ("dense", 300, 4, 2, 128, 128, True),
    ("dense", 300, 4, 2, 128, 128, False),
]


def _poison(t, rows):
    """q -> NaN, k -> +Inf, v -> NaN on the given token rows (first axis after
    flattening the batch)."""
    t = t.clone()
    t.view(-1, *t.shape[-2:])[rows] = float("nan")
    return t


@pytest.mark.parametrize("case", ISOLATION_CASES, ids=lambda c: "%s_d%d_%s" % (
    c[0], c[4], "c" if c[6] else "nc"))
def test_nonfinite_neighbour_is_isolated(case):
    layout, lens, Hq, Hkv, d, dv, causal = case
    L = lt()
    if layout == "packed":
        w = inputs.Workload("t", len(lens), Hq, Hkv, 0, d, dv, torch.bfloat16, d ** -0.5, causal,
                            sum(lens))
        q, k, v, cu = inputs.make(w, lengths=lens)
        bad = torch.arange(lens[0], lens[0] + lens[1])  # the middle sequence
        keep = torch.cat([torch.arange(0, lens[0]), torch.arange(lens[0] + lens[1], sum(lens))])
        cu_dev = cu.cuda()
    else:
        q, k, v = inputs.make_custom(2, Hq, Hkv, lens, d, dv, torch.bfloat16, d ** -0.5, seed=31)
        bad = torch.arange(lens, 2 * lens)  # batch row 1, flattened tokens
        keep = torch.arange(0, lens)
        cu, cu_dev = None, None
    ref = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6,
                               cu_seqlens=None if cu is None else cu.numpy())
    qp = _poison(q, bad)
    kp = k.clone()
    kp.view(-1, *k.shape[-2:])[bad] = float("inf")
    vp = _poison(v, bad)
    out = L.linear_attn_fwd(qp.cuda(), kp.cuda(), vp.cuda(), causal=causal, eps=1e-6,
                            cu_seqlens=cu_dev)
    torch.cuda.synchronize()
    assert L.get_last_device_error() == 0
    got = out.float().cpu().numpy().reshape(-1, Hq, dv)[keep.numpy()]
    ref = np.asarray(ref).reshape(-1, Hq, dv)[keep.numpy()]
    assert row_rel_err(got, ref) <= TOL_BF16
