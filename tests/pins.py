"""Pins for the fp64 oracle: checks against facts the pages and the
mathematics fix, independent of the oracle's own code.

Each ``pin_*`` function raises AssertionError when the oracle (as currently
loaded in the ``oracle`` package) violates the fact.  They are run directly
by ``test_oracle_pins.py`` and against deliberately broken copies of the
oracle by ``test_oracle_mutants.py`` (every planted mistake must trip at
least one pin).
"""
import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def pin_phi_is_elu_plus_one():
    """phi(x) = ELU(x) + 1 (alpha = 1), checked against torch's ELU."""
    xs = np.concatenate([np.linspace(-30, 30, 601), [-1e-12, 0.0, 1e-12, -800.0]])
    ref = torch.nn.functional.elu(torch.tensor(xs, dtype=torch.float64), alpha=1.0) + 1.0
    got = np.array([oracle.phi(x) for x in xs])
    # torch forms ELU+1 as expm1(x) + 1, whose absolute rounding is ~1e-16
    assert np.allclose(got, ref.numpy(), rtol=1e-14, atol=2e-16), "phi != ELU+1"
    assert oracle.phi(0.0) == 1.0 and oracle.phi(1.0) == 2.0
    assert abs(oracle.phi(-math.log(2.0)) - 0.5) < 1e-16


def pin_feature_maps():
    """The other feature maps against torch: ReLU = max(x, 0), exp; and a
    forward pass under each map equals the quadratic form written with that
    map's features (the ELU + 1 pins above hold the forms together)."""
    xs = np.concatenate([np.linspace(-30, 30, 601), [-1e-12, 0.0, 1e-12]])
    t = torch.tensor(xs, dtype=torch.float64)
    for kind, ref in (("relu", torch.relu(t)), ("exp", torch.exp(t))):
        got = np.array([oracle.phi(x, kind) for x in xs])
        assert np.allclose(got, ref.numpy(), rtol=1e-15, atol=0), kind
    assert oracle.phi(-1.0) == math.exp(-1.0)  # the default is back after each call
    # under map m, phi(Q) phi(K)^T has the same entries as the ELU + 1 form
    # applied to inputs whose ELU + 1 features are m's features: for ReLU,
    # x -> x - 1 maps x > 1 onto ELU + 1's linear branch, and zero features
    # come from very negative inputs (exp underflows to 0)
    q = np.abs(_rand((1, 9, 2, 4), 150)) + 1.1
    k = np.abs(_rand((1, 9, 2, 4), 151)) + 1.1
    k[0, ::3, 0, 1] = -1.0  # relu features 0 here
    v = _rand((1, 9, 2, 3), 152)
    kk = np.where(k > 0, k - 1.0, -800.0)
    for causal in (True, False):
        a = oracle.fwd_quadratic(q, k, v, causal=causal, eps=1e-6, phi="relu")
        b = oracle.fwd_quadratic(q - 1.0, kk, v, causal=causal, eps=1e-6)
        assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()
        a = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6, phi="relu")
        assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()
    # exp: phi(x) = e^x for every x equals ELU + 1 on inputs <= 0; shift by a
    # constant c (e^(x - c) = e^x e^-c cancels between numerator and
    # denominator when eps = 0)
    q2, k2 = _rand((1, 7, 2, 3), 153), _rand((1, 7, 2, 3), 154)
    c = max(q2.max(), k2.max()) + 0.5
    for causal in (True, False):
        a = oracle.fwd_recurrent(q2, k2, v[:, :7], causal=causal, eps=0.0, phi="exp")
        b = oracle.fwd_quadratic(q2 - c, k2 - c, v[:, :7], causal=causal, eps=0.0)
        assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()


def pin_fp16_inputs_widened_exactly():
    """fp16 inputs are read as the exact values they hold: the oracle on
    fp16 tensors equals the oracle on the same values in fp64, subnormals,
    the largest finite value and signed zero included."""
    h = torch.tensor([0.0, -0.0, 1.0, -2.5, 65504.0, 6.1e-5, 5.96e-8, -3.0e-6, 0.333],
                     dtype=torch.float16)
    assert h.double().tolist() == [float(x) for x in h.double().numpy()]
    q = (torch.randn(1, 11, 2, 4, generator=torch.Generator().manual_seed(9)) * 0.7).half()
    k = (torch.randn(1, 11, 2, 4, generator=torch.Generator().manual_seed(10)) * 0.7).half()
    v = (torch.randn(1, 11, 2, 3, generator=torch.Generator().manual_seed(11))).half()
    v[0, 3, 0] = h[:3]
    k[0, 5, 1, :] = h[5:9]
    for causal in (True, False):
        a = oracle.fwd_quadratic(q, k, v, causal=causal)
        b = oracle.fwd_quadratic(q.double(), k.double(), v.double(), causal=causal)
        assert np.array_equal(a, b)
    vv = torch.tensor([[[[1.0, 65504.0, 5.96e-8]]]], dtype=torch.float16)
    o = oracle.fwd_recurrent(torch.zeros(1, 1, 1, 2).half(), torch.zeros(1, 1, 1, 2).half(), vv,
                             eps=0.0)
    assert o.tolist() == [[[[1.0, 65504.0, float(torch.tensor(5.96e-8).half().double())]]]]


def pin_sliding_window():
    """Sliding window (keys i - w < j <= i): the windowed quadratic form and
    the difference of two prefix states agree; w >= n is the causal form;
    w = 1 gives each row its own value (scaled by a/(a+eps)); constant keys
    give the moving average of the last w values (eps = 0); packed sequences
    equal independent calls; GQA equals replication."""
    B, N, Hq, Hkv, d, dv = 2, 29, 4, 2, 5, 3
    q = _rand((B, N, Hq, d), 160)
    k = _rand((B, N, Hkv, d), 161)
    v = _rand((B, N, Hkv, dv), 162)
    for w in (1, 2, 7, 28, 29, 100):
        a = oracle.fwd_window_quadratic(q, k, v, w)
        b = oracle.fwd_window_recurrent(q, k, v, w)
        assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max(), w
    full = oracle.fwd_quadratic(q, k, v, causal=True)
    for w in (29, 100):
        assert np.abs(oracle.fwd_window_recurrent(q, k, v, w) - full).max() <= 1e-12 * np.abs(full).max()
    o1 = oracle.fwd_window_quadratic(q, k, v, 1, eps=0.0)
    assert np.abs(o1 - np.repeat(v, Hq // Hkv, axis=2)).max() <= 1e-14
    kc = np.broadcast_to(_rand((1, 1, Hkv, d), 163), k.shape).copy()
    for w in (3, 8):
        o = oracle.fwd_window_recurrent(q, kc, v, w, eps=0.0)
        csum = np.concatenate([np.zeros((B, 1, Hkv, dv)), np.cumsum(v, axis=1)], axis=1)
        idx = np.arange(N)
        lo = np.maximum(idx - w + 1, 0)
        mean = (csum[:, idx + 1] - csum[:, lo]) / (idx - lo + 1).reshape(1, N, 1, 1)
        assert np.abs(o - np.repeat(mean, Hq // Hkv, axis=2)).max() <= 1e-13, w
    G = Hq // Hkv
    a = oracle.fwd_window_recurrent(q, k, v, 6)
    b = oracle.fwd_window_quadratic(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), 6)
    assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()
    lens = [9, 0, 1, 14]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    qp, kp, vp = _rand((T, Hq, d), 164), _rand((T, Hkv, d), 165), _rand((T, Hkv, dv), 166)
    packed = oracle.fwd_window_recurrent(qp, kp, vp, 4, cu_seqlens=cu)
    for s_, n in enumerate(lens):
        if n:
            x, y = cu[s_], cu[s_ + 1]
            dense = oracle.fwd_window_quadratic(qp[None, x:y], kp[None, x:y], vp[None, x:y], 4)[0]
            assert np.abs(packed[x:y] - dense).max() <= 1e-12 * max(1.0, np.abs(dense).max())


def _hand_2x2_inputs(g):
    q = np.array(g["q"], dtype=np.float64).reshape(1, 2, 1, 2)
    k = np.array([[1.0, 0.0], [0.0, -math.log(2.0)]]).reshape(1, 2, 1, 2)
    v = np.array(g["v"], dtype=np.float64).reshape(1, 2, 1, 2)
    return q, k, v


def pin_hand_2x2():
    """Hand-worked 2x2 example (tests/golden/hand_2x2.json)."""
    g = _load("hand_2x2.json")
    q, k, v = _hand_2x2_inputs(g)
    for fn in (oracle.fwd_quadratic, oracle.fwd_recurrent):
        got = fn(q, k, v, causal=True, eps=0.0)[0, :, 0]
        assert np.allclose(got, g["causal_eps0"], rtol=0, atol=1e-15), (fn.__name__, got)
        got = fn(q, k, v, causal=False, eps=0.0)[0, :, 0]
        assert np.allclose(got, g["noncausal_eps0"], rtol=0, atol=1e-15), (fn.__name__, got)
        got = fn(q, k, v, causal=True, eps=1e-6)[0, :, 0]
        assert np.allclose(got, g["causal_eps1e-6"], rtol=0, atol=1e-15), (fn.__name__, got)
    for order in (0, 1):
        got = oracle.noncausal_numerator(q, k, v, order)[0, :, 0]
        assert np.allclose(got, g["noncausal_numerator"], rtol=0, atol=1e-15), (order, got)
    rows = np.array([[0, 0, 0], [0, 1, 0]])
    got = oracle.fwd_rows(q, k, v, rows, causal=True, eps=0.0)
    assert np.allclose(got, g["causal_eps0"], rtol=0, atol=1e-15)
    got = oracle.fwd_rows(q, k, v, rows, causal=False, eps=0.0)
    assert np.allclose(got, g["noncausal_eps0"], rtol=0, atol=1e-15), got
    got = oracle.fwd_rows(q, k, v, rows, causal=True, eps=1e-6)
    assert np.allclose(got, g["causal_eps1e-6"], rtol=0, atol=1e-15), got


def hand_3tok_inputs(d=64, dv=64, dtype=torch.float32):
    """The exact 3-token example embedded in d feature dims (padding -9984)."""
    g = _load("hand_3tok_exact.json")
    q = torch.full((1, 3, 1, d), g["pad_value"], dtype=torch.float64)
    k = torch.full((1, 3, 1, d), g["pad_value"], dtype=torch.float64)
    q[0, :, 0, :2] = torch.tensor(g["q_active"], dtype=torch.float64)
    k[0, :, 0, :2] = torch.tensor(g["k_active"], dtype=torch.float64)
    v = torch.zeros((1, 3, 1, dv), dtype=torch.float64)
    for j in range(3):
        v[0, j, 0, j] = 1.0
    return q.to(dtype), k.to(dtype), v.to(dtype), g


def pin_hand_3tok():
    """Exact 3-token example with underflowing padding dims, fp32 and bf16 inputs."""
    for dt in (torch.float32, torch.bfloat16):
        q, k, v, g = hand_3tok_inputs(dtype=dt)
        for fn in (oracle.fwd_quadratic, oracle.fwd_recurrent):
            got = fn(q, k, v, causal=True, eps=0.0)[0, :, 0]
            assert np.allclose(got[:, :3], g["causal_eps0_first3cols"], rtol=0, atol=1e-15)
            assert np.all(got[:, 3:] == 0.0)
            got = fn(q, k, v, causal=False, eps=0.0)[0, :, 0]
            assert np.allclose(got[:, :3], g["noncausal_eps0_first3cols"], rtol=0, atol=1e-15)


TWO_FORM_CASES = [
    # (B, Hq, Hkv, N, d, dv, causal)
    (1, 1, 1, 1, 1, 1, True),
    (1, 1, 1, 7, 2, 3, True),
    (2, 2, 1, 33, 3, 8, True),
    (1, 4, 2, 65, 8, 2, False),
    (2, 8, 2, 40, 64, 64, True),
    (1, 2, 2, 19, 64, 128, False),
]


def pin_two_forms_agree():
    """Quadratic and recurrent forms agree to 1e-12 relative (tiny inputs)."""
    for i, (B, Hq, Hkv, N, d, dv, causal) in enumerate(TWO_FORM_CASES):
        q = _rand((B, N, Hq, d), 10 + i)
        k = _rand((B, N, Hkv, d), 20 + i)
        v = _rand((B, N, Hkv, dv), 30 + i)
        a = oracle.fwd_quadratic(q, k, v, causal=causal, eps=1e-6)
        b = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
        scale = max(1e-300, np.abs(a).max())
        assert np.abs(a - b).max() <= 1e-12 * scale, (i, np.abs(a - b).max(), scale)


def pin_associativity():
    """(phi(Q) phi(K)^T) V == phi(Q) (phi(K)^T V); and the normalised
    non-causal output equals numerator / numerator-with-V-all-ones."""
    q = _rand((2, 23, 4, 5), 1)
    k = _rand((2, 23, 2, 5), 2)
    v = _rand((2, 23, 2, 6), 3)
    n0 = oracle.noncausal_numerator(q, k, v, 0)
    n1 = oracle.noncausal_numerator(q, k, v, 1)
    assert np.abs(n0 - n1).max() <= 1e-12 * np.abs(n0).max()
    den = oracle.noncausal_numerator(q, k, np.ones_like(v), 1)
    o = oracle.fwd_recurrent(q, k, v, causal=False, eps=0.0)
    assert np.abs(o - n0 / den).max() <= 1e-12 * np.abs(o).max()


def pin_constant_keys_give_prefix_mean():
    """All keys equal => every score in a row is equal => with eps = 0 the
    causal output is the running mean of V and the non-causal one the mean."""
    B, N, H, d, dv = 1, 17, 2, 4, 3
    q = _rand((B, N, H, d), 4)
    k = np.broadcast_to(_rand((1, 1, H, d), 5), (B, N, H, d)).copy()
    v = _rand((B, N, H, dv), 6)
    prefix_mean = np.cumsum(v, axis=1) / np.arange(1, N + 1).reshape(1, N, 1, 1)
    for fn in (oracle.fwd_quadratic, oracle.fwd_recurrent):
        o = fn(q, k, v, causal=True, eps=0.0)
        assert np.abs(o - prefix_mean).max() <= 1e-13
        o = fn(q, k, v, causal=False, eps=0.0)
        assert np.abs(o - v.mean(axis=1, keepdims=True)).max() <= 1e-13


def pin_first_row_is_v0():
    """Causal row 0 sees only token 0: O_0 = V_0 * a/(a + eps)."""
    q = _rand((2, 9, 3, 4), 7)
    k = _rand((2, 9, 3, 4), 8)
    v = _rand((2, 9, 3, 5), 9)
    for fn in (oracle.fwd_quadratic, oracle.fwd_recurrent):
        o = fn(q, k, v, causal=True, eps=0.0)
        assert np.abs(o[:, 0] - v[:, 0]).max() <= 1e-14


def pin_weights_sum_to_one_minus_eps_over_den():
    """With V = 1 every output equals sum(a)/(sum(a)+eps): exactly 1 at eps=0,
    in (0, 1) for eps > 0 and decreasing in eps; den > 0 always."""
    q = _rand((1, 31, 2, 6), 11, 3.0)
    k = _rand((1, 31, 2, 6), 12, 3.0)
    ones = np.ones((1, 31, 2, 4))
    for causal in (True, False):
        for fn in (oracle.fwd_quadratic, oracle.fwd_recurrent):
            o0 = fn(q, k, ones, causal=causal, eps=0.0)
            assert np.abs(o0 - 1.0).max() <= 1e-14
            o1 = fn(q, k, ones, causal=causal, eps=1e-3)
            o2 = fn(q, k, ones, causal=causal, eps=1e-1)
            assert np.all(o1 < 1.0) and np.all(o2 > 0.0) and np.all(o2 < o1)
    # den from the V=1 output: 1 - O = eps/den  => den = eps/(1-O) > 0
    o = oracle.fwd_recurrent(q, k, ones, causal=True, eps=1e-2)
    assert np.all(1e-2 / (1.0 - o) > 0)


def pin_convex_hull():
    """At eps = 0 each causal output is a convex combination of V_0..V_i."""
    q = _rand((1, 40, 2, 8), 13)
    k = _rand((1, 40, 2, 8), 14)
    v = _rand((1, 40, 2, 5), 15)
    o = oracle.fwd_quadratic(q, k, v, causal=True, eps=0.0)
    lo = np.minimum.accumulate(v, axis=1)
    hi = np.maximum.accumulate(v, axis=1)
    assert np.all(o >= lo - 1e-13) and np.all(o <= hi + 1e-13)


def pin_gqa_equals_replication():
    """H_kv < H_q equals explicit replication of each KV head over its group
    of G = H_q/H_kv consecutive query heads."""
    B, N, Hq, Hkv, d, dv = 2, 21, 8, 2, 4, 3
    q = _rand((B, N, Hq, d), 16)
    k = _rand((B, N, Hkv, d), 17)
    v = _rand((B, N, Hkv, dv), 18)
    G = Hq // Hkv
    kr = np.repeat(k, G, axis=2)
    vr = np.repeat(v, G, axis=2)
    for causal in (True, False):
        a = oracle.fwd_recurrent(q, k, v, causal=causal, eps=1e-6)
        b = oracle.fwd_quadratic(q, kr, vr, causal=causal, eps=1e-6)
        assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()


def pin_packed_equals_independent():
    """Packed sequences (cu_seqlens) equal independent dense calls."""
    lens = [5, 1, 0, 12, 7]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv, d, dv = int(cu[-1]), 4, 2, 3, 5
    q = _rand((T, Hq, d), 19)
    k = _rand((T, Hkv, d), 20)
    v = _rand((T, Hkv, dv), 21)
    for causal in (True, False):
        for fn in (oracle.fwd_quadratic, oracle.fwd_recurrent):
            packed = fn(q, k, v, causal=causal, eps=1e-6, cu_seqlens=cu)
            for s, n in enumerate(lens):
                if n == 0:
                    continue
                a, b = cu[s], cu[s + 1]
                dense = oracle.fwd_quadratic(q[None, a:b], k[None, a:b], v[None, a:b],
                                             causal=causal, eps=1e-6)[0]
                assert np.abs(packed[a:b] - dense).max() <= 1e-12 * max(1.0, np.abs(dense).max())


def pin_rows_equal_quadratic_packed_gqa():
    """Selected rows (the full-size checker) equal the same rows of the
    quadratic form, itself pinned above, on packed GQA sequences (an empty
    one among them) and on a dense batch, causal and non-causal: every
    sequence, the first and last position of each, and random heads."""
    lens = [9, 0, 1, 17, 6]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv, d, dv = int(cu[-1]), 6, 2, 5, 4
    q = _rand((T, Hq, d), 70)
    k = _rand((T, Hkv, d), 71)
    v = _rand((T, Hkv, dv), 72)
    g = np.random.default_rng(73)
    rows = []
    for s, n in enumerate(lens):
        for i in sorted({0, n - 1, n // 2} if n else ()):
            for h in (0, Hq - 1, int(g.integers(0, Hq))):
                rows.append((s, i, h))
    rows = np.array(rows, dtype=np.int64)
    for causal in (True, False):
        full = oracle.fwd_quadratic(q, k, v, causal=causal, eps=1e-6, cu_seqlens=cu)
        want = np.stack([full[cu[s] + i, h] for s, i, h in rows])
        got = oracle.fwd_rows(q, k, v, rows, causal=causal, eps=1e-6, cu_seqlens=cu)
        assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max(), causal
    B, N = 2, 13
    qd = _rand((B, N, Hq, d), 74)
    kd = _rand((B, N, Hkv, d), 75)
    vd = _rand((B, N, Hkv, dv), 76)
    rows = np.array([(b, i, h) for b in range(B) for i in (0, 6, N - 1) for h in (1, Hq - 2)],
                    dtype=np.int64)
    for causal in (True, False):
        full = oracle.fwd_quadratic(qd, kd, vd, causal=causal, eps=1e-6)
        want = np.stack([full[b, i, h] for b, i, h in rows])
        got = oracle.fwd_rows(qd, kd, vd, rows, causal=causal, eps=1e-6)
        assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max(), causal


def pin_decode_chain_equals_causal():
    """N decode steps from a zero state reproduce the causal forward row by row."""
    B, N, Hq, Hkv, d, dv = 3, 11, 4, 2, 5, 6
    q = _rand((B, N, Hq, d), 22)
    k = _rand((B, N, Hkv, d), 23)
    v = _rand((B, N, Hkv, dv), 24)
    ref = oracle.fwd_quadratic(q, k, v, causal=True, eps=1e-6)
    S = np.zeros((B, Hkv, d, dv))
    z = np.zeros((B, Hkv, d))
    for t in range(N):
        o = oracle.decode_step(np.ascontiguousarray(q[:, t]), np.ascontiguousarray(k[:, t]),
                               np.ascontiguousarray(v[:, t]), S, z, eps=1e-6)
        assert np.abs(o - ref[:, t]).max() <= 1e-12 * max(1.0, np.abs(ref[:, t]).max())


def pin_value_scaling_and_key_permutation():
    """O(Q, K, cV) = c O(Q, K, V); non-causal output is invariant to a joint
    permutation of the key/value tokens (queries held fixed)."""
    q = _rand((1, 15, 2, 4), 25)
    k = _rand((1, 15, 2, 4), 26)
    v = _rand((1, 15, 2, 3), 27)
    a = oracle.fwd_recurrent(q, k, v, causal=True, eps=1e-6)
    b = oracle.fwd_recurrent(q, k, -2.5 * v, causal=True, eps=1e-6)
    assert np.abs(b + 2.5 * a).max() <= 1e-12 * np.abs(b).max()
    perm = np.random.default_rng(0).permutation(15)
    o = oracle.noncausal_numerator(q, k, v, 0)
    op = oracle.noncausal_numerator(q, k[:, perm], v[:, perm], 0)
    assert np.abs(o - op).max() <= 1e-12 * np.abs(o).max()


def pin_state_split_continuation():
    """Cutting causal sequences at any point and continuing the second part
    from the first part's final state reproduces the unsplit output (the
    quadratic form) row by row, dense and packed, with GQA; the continued
    run ends in the unsplit run's final state."""
    B, N, Hq, Hkv, d, dv = 2, 23, 4, 2, 5, 6
    q = _rand((B, N, Hq, d), 41)
    k = _rand((B, N, Hkv, d), 42)
    v = _rand((B, N, Hkv, dv), 43)
    ref = oracle.fwd_quadratic(q, k, v, causal=True, eps=1e-6)
    _, S_all, z_all = oracle.fwd_state(q, k, v, causal=True, eps=1e-6)
    for n1 in (1, 9, 22):
        o1, S1, z1 = oracle.fwd_state(q[:, :n1], k[:, :n1], v[:, :n1], causal=True, eps=1e-6)
        o2, S2, z2 = oracle.fwd_state(q[:, n1:], k[:, n1:], v[:, n1:], causal=True, eps=1e-6,
                                      S0=S1, z0=z1)
        got = np.concatenate([o1, o2], axis=1)
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
        assert np.abs(S2 - S_all).max() <= 1e-12 * np.abs(S_all).max()
        assert np.abs(z2 - z_all).max() <= 1e-12 * np.abs(z_all).max()
    # packed: sequence b of the second call continues sequence b of the first
    lens1, lens2 = [4, 0, 7], [5, 3, 0]
    g = np.random.default_rng(44)
    n_all = [a + b for a, b in zip(lens1, lens2)]
    qs = [g.standard_normal((n, Hq, d)) for n in n_all]
    ks = [g.standard_normal((n, Hkv, d)) for n in n_all]
    vs = [g.standard_normal((n, Hkv, dv)) for n in n_all]
    cu1 = np.cumsum([0] + lens1).astype(np.int32)
    cu2 = np.cumsum([0] + lens2).astype(np.int32)
    part = lambda xs, lo, hi: np.concatenate([x[l:h] for x, l, h in zip(xs, lo, hi)])
    hi1 = lens1
    o1, S1, z1 = oracle.fwd_state(part(qs, [0] * 3, hi1), part(ks, [0] * 3, hi1),
                                  part(vs, [0] * 3, hi1), causal=True, eps=1e-6, cu_seqlens=cu1)
    o2, _, _ = oracle.fwd_state(part(qs, hi1, n_all), part(ks, hi1, n_all), part(vs, hi1, n_all),
                                causal=True, eps=1e-6, cu_seqlens=cu2, S0=S1, z0=z1)
    for b in range(3):
        r = oracle.fwd_quadratic(qs[b][None], ks[b][None], vs[b][None], causal=True, eps=1e-6)[0]
        got = np.concatenate([o1[cu1[b]:cu1[b + 1]], o2[cu2[b]:cu2[b + 1]]])
        assert np.abs(got - r).max() <= 1e-12 * max(1.0, np.abs(r).max())


def pin_state_final_equals_decode_chain():
    """The final state of a forward pass from a given state equals the state
    that as many decode steps from that state reach (prefill -> decode)."""
    B, N, Hq, Hkv, d, dv = 2, 9, 4, 2, 5, 3
    q = _rand((B, N, Hq, d), 45)
    k = _rand((B, N, Hkv, d), 46)
    v = _rand((B, N, Hkv, dv), 47)
    S0 = np.abs(_rand((B, Hkv, d, dv), 48))
    z0 = np.abs(_rand((B, Hkv, d), 49))
    _, S_f, z_f = oracle.fwd_state(q, k, v, causal=True, eps=1e-6, S0=S0, z0=z0)
    S, z = S0.copy(), z0.copy()
    for t in range(N):
        oracle.decode_step(np.ascontiguousarray(q[:, t]), np.ascontiguousarray(k[:, t]),
                           np.ascontiguousarray(v[:, t]), S, z, eps=1e-6)
    assert np.abs(S_f - S).max() <= 1e-12 * np.abs(S).max()
    assert np.abs(z_f - z).max() <= 1e-12 * np.abs(z).max()


def pin_state_noncausal_prefix():
    """Non-causal from the state of a prefix p equals non-causal attention of
    the rows of x over the keys of p and x together (quadratic form)."""
    B, Hq, Hkv, d, dv = 1, 4, 2, 4, 5
    p = [_rand((B, 6, H, w), 50 + i) for i, (H, w) in enumerate(((Hq, d), (Hkv, d), (Hkv, dv)))]
    x = [_rand((B, 8, H, w), 60 + i) for i, (H, w) in enumerate(((Hq, d), (Hkv, d), (Hkv, dv)))]
    _, Sp, zp = oracle.fwd_state(*p, causal=True, eps=1e-6)
    got, _, _ = oracle.fwd_state(*x, causal=False, eps=1e-6, S0=Sp, z0=zp)
    cat = [np.concatenate([a, b], axis=1) for a, b in zip(p, x)]
    ref = oracle.fwd_quadratic(*cat, causal=False, eps=1e-6)[:, 6:]
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


def pin_bwd_hand_2x2():
    """Hand-worked gradients of the 2x2 example (tests/golden/hand_2x2_backward.json)."""
    g = _load("hand_2x2_backward.json")
    q, k, v, do = (np.array(g[x], dtype=np.float64).reshape(1, 2, 1, 2)
                   for x in ("q", "k", "v", "dout"))
    for causal, key in ((True, "causal"), (False, "noncausal")):
        for fn in (oracle.bwd_quadratic, oracle.bwd_recurrent):
            dq, dk, dv = fn(q, k, v, do, causal=causal, eps=0.0)
            for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
                assert np.allclose(got[0, :, 0], g[key][name], rtol=0, atol=1e-15), \
                    (fn.__name__, key, name, got[0, :, 0])


def _loss(q, k, v, do, causal, eps, cu=None):
    return float((oracle.fwd_quadratic(q, k, v, causal=causal, eps=eps, cu_seqlens=cu) * do).sum())


def pin_bwd_finite_differences():
    """Both backward forms equal central finite differences of
    L = sum(O * dO) through the (pinned) quadratic forward form: every entry
    of Q, K and V, with negative inputs (phi' = e^x), GQA, eps > 0, causal and
    non-causal, dense and packed."""
    cases = [
        # (B, N, Hq, Hkv, d, dv, causal, eps, packed lengths or None)
        (1, 5, 2, 1, 3, 2, True, 1e-3, None),
        (2, 4, 2, 2, 2, 3, False, 0.0, None),
        (1, 0, 2, 1, 2, 2, True, 1e-2, [3, 0, 2]),
    ]
    h = 1e-5
    for i, (B, N, Hq, Hkv, d, dv, causal, eps, lens) in enumerate(cases):
        cu = None
        if lens is not None:
            cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
            T = int(cu[-1])
            shapes = ((T, Hq, d), (T, Hkv, d), (T, Hkv, dv), (T, Hq, dv))
        else:
            shapes = ((B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, dv), (B, N, Hq, dv))
        q, k, v, do = (_rand(sh, 80 + 4 * i + j, 1.5) for j, sh in enumerate(shapes))
        grads = [fn(q, k, v, do, causal=causal, eps=eps, cu_seqlens=cu)
                 for fn in (oracle.bwd_quadratic, oracle.bwd_recurrent)]
        for which, x in enumerate((q, k, v)):
            fd = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = [q, k, v]
                args_m = [q, k, v]
                args_p[which], args_m[which] = xp, xm
                fd[idx] = (_loss(*args_p, do, causal, eps, cu) -
                           _loss(*args_m, do, causal, eps, cu)) / (2 * h)
            scale = max(1e-12, np.abs(fd).max())
            for gr in grads:
                err = np.abs(gr[which] - fd).max() / scale
                assert err <= 1e-6, (i, which, err)


def pin_bwd_two_forms_agree():
    """The differentiated quadratic form and the two recurrences agree to
    1e-12 relative on random inputs (GQA, widths 64 and 128, non-causal)."""
    cases = [(2, 30, 4, 2, 8, 5, True), (1, 40, 2, 2, 64, 64, True), (1, 25, 4, 1, 6, 128, False),
             (2, 17, 2, 2, 64, 64, False)]
    for i, (B, N, Hq, Hkv, d, dv, causal) in enumerate(cases):
        q = _rand((B, N, Hq, d), 90 + i, 0.5)
        k = _rand((B, N, Hkv, d), 100 + i, 0.5)
        v = _rand((B, N, Hkv, dv), 110 + i)
        do = _rand((B, N, Hq, dv), 120 + i)
        a = oracle.bwd_quadratic(q, k, v, do, causal=causal, eps=1e-6)
        b = oracle.bwd_recurrent(q, k, v, do, causal=causal, eps=1e-6)
        for x, y in zip(a, b):
            assert np.abs(x - y).max() <= 1e-12 * max(1e-300, np.abs(x).max()), i


def pin_bwd_packed_and_gqa():
    """Packed sequences give the gradients of independent dense calls; with
    GQA, dK and dV of a KV head are the sums over its query heads of the
    gradients with each KV head explicitly replicated."""
    lens = [6, 0, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv, d, dv = int(cu[-1]), 4, 2, 3, 4
    q, k, v, do = (_rand(sh, 130 + j) for j, sh in
                   enumerate(((T, Hq, d), (T, Hkv, d), (T, Hkv, dv), (T, Hq, dv))))
    for causal in (True, False):
        pk = oracle.bwd_recurrent(q, k, v, do, causal=causal, eps=1e-6, cu_seqlens=cu)
        for s, n in enumerate(lens):
            if n == 0:
                continue
            a, b = cu[s], cu[s + 1]
            dense = oracle.bwd_quadratic(q[None, a:b], k[None, a:b], v[None, a:b],
                                         do[None, a:b], causal=causal, eps=1e-6)
            for x, y in zip(pk, dense):
                assert np.abs(x[a:b] - y[0]).max() <= 1e-12 * max(1.0, np.abs(y).max())
    B, N = 2, 11
    q, k, v, do = (_rand(sh, 140 + j) for j, sh in
                   enumerate(((B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, dv), (B, N, Hq, dv))))
    G = Hq // Hkv
    for causal in (True, False):
        dq, dk, dv_ = oracle.bwd_recurrent(q, k, v, do, causal=causal, eps=1e-6)
        rq, rk, rv = oracle.bwd_quadratic(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2),
                                          do, causal=causal, eps=1e-6)
        assert np.abs(dq - rq).max() <= 1e-12 * np.abs(rq).max()
        assert np.abs(dk - rk.reshape(B, N, Hkv, G, d).sum(3)).max() <= 1e-12 * np.abs(dk).max()
        assert np.abs(dv_ - rv.reshape(B, N, Hkv, G, dv).sum(3)).max() <= 1e-12 * np.abs(dv_).max()


ALL_PINS = [
    pin_phi_is_elu_plus_one,
    pin_feature_maps,
    pin_fp16_inputs_widened_exactly,
    pin_sliding_window,
    pin_hand_2x2,
    pin_hand_3tok,
    pin_two_forms_agree,
    pin_associativity,
    pin_constant_keys_give_prefix_mean,
    pin_first_row_is_v0,
    pin_weights_sum_to_one_minus_eps_over_den,
    pin_convex_hull,
    pin_gqa_equals_replication,
    pin_packed_equals_independent,
    pin_rows_equal_quadratic_packed_gqa,
    pin_decode_chain_equals_causal,
    pin_value_scaling_and_key_permutation,
    pin_state_split_continuation,
    pin_state_final_equals_decode_chain,
    pin_state_noncausal_prefix,
    pin_bwd_hand_2x2,
    pin_bwd_finite_differences,
    pin_bwd_two_forms_agree,
    pin_bwd_packed_and_gqa,
]
