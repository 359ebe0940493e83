"""The C ABI: the library loads, exports every entry point the header
declares, and rejects invalid arguments on the host (CPU only: none of these
calls reaches a CUDA API)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"LT_API\s+[\w\s\*]+?\b(lt_\w+)\s*\(", src)
    return names


def test_header_declares_entry_points():
    names = declared_functions()
    assert "lt_linear_attn_fwd" in names and "lt_linear_attn_decode_step" in names


def test_library_exports_every_declared_symbol():
    from causal_linear_attention_chunked_b200 import _binding as b
    for name in declared_functions():
        assert hasattr(b.lib, name), name
    assert set(declared_functions()) == set(b.EXPORTED)


def test_abi_version_and_status_strings():
    from causal_linear_attention_chunked_b200 import _binding as b
    assert b.lib.lt_abi_version() == 1
    for code in range(7):
        assert b.lib.lt_status_string(code).startswith(b"LT_")
    assert b.lib.lt_status_string(99) == b"unknown lt_status_t"


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every case fails before that


@pytest.mark.parametrize("case,expect", [
    (dict(q=None), 1),
    (dict(B=0), 1),
    (dict(Hq=0), 1),
    (dict(Hkv=3, Hq=8), 1),
    (dict(N=0), 1),
    (dict(causal=2), 1),
    (dict(eps=-1.0), 1),
    (dict(eps=float("nan")), 1),
    (dict(eps=float("inf")), 1),
    (dict(d=32), 2),
    (dict(dv=96), 2),
    (dict(dtype=7), 2),
    (dict(B=70000), 1),
    (dict(B=1 << 16, N=1 << 16), 1),
    (dict(Hkv=70000, Hq=70000), 1),
])
def test_fwd_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, Hq=8, Hkv=8, N=16, d=64, dv=64, causal=1,
             eps=1e-6, cu=None, stream=None, dtype=1)
    a.update(case)
    st = b.lib.lt_linear_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"], a["Hkv"],
                                  a["N"], a["d"], a["dv"], a["causal"], a["eps"], a["cu"],
                                  a["stream"], a["dtype"])
    assert st == expect


@pytest.mark.parametrize("case", [
    dict(q=None), dict(q=None, d=32), dict(B=0), dict(Hkv=3, Hq=8), dict(N=0), dict(causal=2),
    dict(eps=-1.0), dict(eps=float("nan")), dict(d=32), dict(dv=96), dict(d=32, eps=-1.0),
    dict(B=70000), dict(B=1 << 16, N=1 << 16), dict(Hkv=70000, Hq=70000),
])
def test_noalloc_returns_the_same_status_as_fwd(case):
    """The no-allocation entry point makes lt_linear_attn_fwd's checks in the
    same order, so the same bad arguments give the same status code."""
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, Hq=8, Hkv=8, N=16, d=64, dv=64, causal=1,
             eps=1e-6)
    a.update(case)
    args = (a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
            a["dv"], a["causal"], a["eps"], None, None)
    st_fwd = b.lib.lt_linear_attn_fwd(*args, 1)
    st_na = b.lib.lt_linear_attn_fwd_noalloc(*args)
    assert st_fwd != 0 and st_na == st_fwd, (st_fwd, st_na)


def test_schedule_override_validates_and_resets():
    from causal_linear_attention_chunked_b200 import _binding as b
    assert b.lib.lt_debug_set_schedule(3, 0) == 1
    assert b.lib.lt_debug_set_schedule(0, -1) == 1
    nb, nl, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    try:
        assert b.lib.lt_debug_set_schedule(b.LT_SCHED_TWO_LAUNCH, 3) == 0
        assert b.lib.lt_linear_attn_fwd_plan(2, 8, 8, 4096, 64, 64, 1, 0, 1, 148, ctypes.byref(nb),
                                             ctypes.byref(nl), ctypes.byref(ws)) == 0
        assert (nb.value, nl.value) == (3, 2)
    finally:
        assert b.lib.lt_debug_set_schedule(b.LT_SCHED_AUTO, 0) == 0
    assert b.lib.lt_linear_attn_fwd_plan(2, 8, 8, 4096, 64, 64, 1, 0, 1, 148, ctypes.byref(nb),
                                         ctypes.byref(nl), ctypes.byref(ws)) == 0
    assert (nb.value, nl.value) == (8, 1)


@pytest.mark.parametrize("case,expect", [
    (dict(S=None), 1),
    (dict(B=0), 1),
    (dict(Hkv=3, Hq=8), 1),
    (dict(eps=-1e-3), 1),
    (dict(d=48), 2),
    (dict(dtype=5), 2),
])
def test_decode_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(q=FAKE, k=FAKE, v=FAKE, S=FAKE, z=FAKE, out=FAKE, B=4, Hq=8, Hkv=8, d=64, dv=64,
             eps=1e-6, stream=None, dtype=1)
    a.update(case)
    st = b.lib.lt_linear_attn_decode_step(a["q"], a["k"], a["v"], a["S"], a["z"], a["out"],
                                          a["B"], a["Hq"], a["Hkv"], a["d"], a["dv"], a["eps"],
                                          a["stream"], a["dtype"])
    assert st == expect


@pytest.mark.parametrize("case,expect", [
    (dict(S0=FAKE), 1),             # S0 without z0
    (dict(z0=FAKE), 1),             # z0 without S0
    (dict(S_out=FAKE), 1),          # S_out without z_out
    (dict(z_out=FAKE), 1),
    (dict(q=None), 1),
    (dict(B=0), 1),
    (dict(Hkv=3, Hq=8), 1),
    (dict(causal=2), 1),
    (dict(eps=float("nan")), 1),
    (dict(d=32), 2),
    (dict(dtype=7), 2),
])
def test_fwd_state_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, Hq=8, Hkv=8, N=16, d=64, dv=64, causal=1,
             eps=1e-6, cu=None, S0=None, z0=None, S_out=None, z_out=None, stream=None, dtype=1)
    a.update(case)
    st = b.lib.lt_linear_attn_fwd_state(a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"],
                                        a["Hkv"], a["N"], a["d"], a["dv"], a["causal"], a["eps"],
                                        a["cu"], a["S0"], a["z0"], a["S_out"], a["z_out"],
                                        a["stream"], a["dtype"])
    assert st == expect


@pytest.mark.parametrize("case,expect", [
    (dict(k=None), 1), (dict(S_out=None), 1), (dict(S0=FAKE), 1), (dict(z0=FAKE), 1),
    (dict(B=0), 1), (dict(N=0), 1), (dict(Hkv=0), 1), (dict(d=32), 2), (dict(dv=96), 2),
    (dict(dtype=4), 2), (dict(B=70000), 1),
])
def test_state_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(k=FAKE, v=FAKE, B=1, Hkv=8, N=16, d=64, dv=64, cu=None, S0=None, z0=None,
             S_out=FAKE, z_out=FAKE, stream=None, dtype=1)
    a.update(case)
    st = b.lib.lt_linear_attn_state(a["k"], a["v"], a["B"], a["Hkv"], a["N"], a["d"], a["dv"],
                                    a["cu"], a["S0"], a["z0"], a["S_out"], a["z_out"],
                                    a["stream"], a["dtype"])
    assert st == expect


@pytest.mark.parametrize("case,expect", [
    (dict(S_all=None), 1), (dict(z_out=None), 1), (dict(world=0), 1), (dict(rank=-1), 1),
    (dict(rank=4), 1), (dict(causal=3), 1), (dict(B=0), 1), (dict(d=48), 2),
])
def test_state_carry_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(S_all=FAKE, z_all=FAKE, world=4, rank=1, causal=1, B=1, Hkv=2, d=64, dv=64,
             S_out=FAKE, z_out=FAKE)
    a.update(case)
    st = b.lib.lt_linear_attn_state_carry(a["S_all"], a["z_all"], a["world"], a["rank"],
                                          a["causal"], a["B"], a["Hkv"], a["d"], a["dv"],
                                          a["S_out"], a["z_out"], None)
    assert st == expect


@pytest.mark.parametrize("case,expect", [
    (dict(q=None), 1), (dict(dout=None), 1), (dict(dq=None), 1), (dict(dv=None), 1),
    (dict(B=0), 1), (dict(Hkv=3, Hq=8), 1), (dict(causal=2), 1), (dict(eps=-1.0), 1),
    (dict(d=32), 2), (dict(dtype=9), 2),
])
def test_bwd_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(q=FAKE, k=FAKE, v=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, Hq=8, Hkv=8,
             N=16, d=64, dvw=64, causal=1, eps=1e-6, dtype=1)
    a.update(case)
    st = b.lib.lt_linear_attn_bwd(a["q"], a["k"], a["v"], a["dout"], a["dq"], a["dk"], a["dv"],
                                  a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["dvw"],
                                  a["causal"], a["eps"], None, None, a["dtype"])
    assert st == expect


@pytest.mark.parametrize("case,expect", [
    (dict(phi=3), 1), (dict(phi=-1), 1), (dict(phi=1, d=64, dv=128), 2),
    (dict(dtype=2, d=128, dv=64), 2), (dict(phi=2, dtype=7), 2), (dict(q=None, phi=1), 1),
])
def test_fwd_ex_rejects_invalid_arguments(case, expect):
    """Unknown feature maps; the tensor-core variants (fp16 I/O, the other
    maps) take d = dv = 64 or 128 only.  Every case fails before a pointer
    is examined."""
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, Hq=8, Hkv=8, N=16, d=64, dv=64, causal=1,
             eps=1e-6, dtype=1, phi=0)
    a.update(case)
    st = b.lib.lt_linear_attn_fwd_ex(a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"],
                                     a["Hkv"], a["N"], a["d"], a["dv"], a["causal"], a["eps"],
                                     None, None, a["dtype"], a["phi"])
    assert st == expect


def test_fp16_plan_and_refusals():
    """fp16 inputs plan the two-launch general path; entry points other than
    the forward pass refuse LT_F16."""
    from causal_linear_attention_chunked_b200 import _binding as b
    nb, nl, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    assert b.lib.lt_linear_attn_fwd_plan(2, 8, 8, 4096, 64, 64, 1, 0, 2, 148, ctypes.byref(nb),
                                         ctypes.byref(nl), ctypes.byref(ws)) == 0
    assert (nb.value, nl.value) == (8, 2)
    assert b.lib.lt_linear_attn_fwd_plan(2, 8, 8, 4096, 64, 128, 1, 0, 2, 148, ctypes.byref(nb),
                                         ctypes.byref(nl), ctypes.byref(ws)) == 2
    assert b.lib.lt_linear_attn_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 8, 64, 64,
                                            1e-6, None, 2) == 2
    assert b.lib.lt_linear_attn_state(FAKE, FAKE, 1, 8, 16, 64, 64, None, None, None, FAKE, FAKE,
                                      None, 2) == 2


@pytest.mark.parametrize("case,expect", [
    (dict(window=0), 1), (dict(window=-3), 1), (dict(q=None), 1), (dict(B=0), 1),
    (dict(d=32), 2), (dict(dtype=9), 2), (dict(Hkv=3, Hq=8), 1),
])
def test_window_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, Hq=8, Hkv=8, N=16, d=64, dv=64, window=4,
             eps=1e-6, dtype=1)
    a.update(case)
    st = b.lib.lt_linear_attn_fwd_window(a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"],
                                         a["Hkv"], a["N"], a["d"], a["dv"], a["window"],
                                         a["eps"], None, None, a["dtype"])
    assert st == expect


def test_selftest_wait_rejects_invalid_limit():
    from causal_linear_attention_chunked_b200 import _binding as b
    assert b.lib.lt_selftest_wait_timeout(0, None) == 1
    assert b.lib.lt_selftest_wait_timeout(2000000, None) == 1


def test_oracle_and_library_share_no_code():
    """The oracle sources never include/import the CUDA path and vice versa."""
    osrc = open(os.path.join(ROOT, "oracle", "lt_oracle.c")).read()
    assert "#include \"" not in osrc
    opy = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    assert "causal_linear_attention_chunked_b200" not in opy
    pkg = os.path.join(ROOT, "causal_linear_attention_chunked_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "lt_oracle" not in txt, f


@pytest.mark.parametrize("shape,expect", [
    # (B, H_q, H_kv, N, d, dv, causal, packed, dtype), num_sms = 148
    # 9 -> 8 blocks of 4 chunks, 128 CTAs: one cooperative launch; the
    # workspace holds the aggregates
    ((2, 8, 8, 4096, 64, 64, 1, 0, 1), (8, 1, 2 * 8 * 8 * (64 * 64 + 64) * 4)),
    ((2, 8, 8, 8192, 64, 64, 1, 0, 1), (8, 2, 2 * 8 * 8 * (64 * 64 + 64) * 4)),  # blocks of 8
    ((1, 8, 8, 65536, 64, 64, 0, 0, 1), (18, 2, 8 * 18 * (64 * 64 + 64) * 4)),
    ((2, 32, 8, 16384, 128, 128, 1, 0, 1), (9, 2, 2 * 8 * 9 * (128 * 128 + 128) * 4)),
    ((1, 1, 1, 300, 64, 128, 1, 0, 1), (3, 2, 3 * (64 * 128 + 64) * 4)),   # capped by 3 chunks
    ((1, 1, 1, 100, 64, 64, 1, 0, 1), (1, 1, 0)),                            # one chunk
    ((64, 8, 8, 50000, 64, 64, 1, 1, 1), (1, 1, 0)),                         # packed
    ((2, 8, 8, 4096, 64, 64, 1, 0, 0), (1, 1, 0)),                           # fp32 path
    ((1, 2, 1, 8192, 64, 64, 1, 0, 1), (64, 1, 64 * (64 * 64 + 64) * 4)),  # 64 chunks, one launch
])
def test_fwd_plan_host_arithmetic(sched, shape, expect):
    """Blocks per sequence: the SM count over the (sequence, KV head) lanes,
    at most the chunk count; one launch when there is one block; the
    workspace holds one fp32 d x dv + d partial state per block."""
    from causal_linear_attention_chunked_b200 import _binding as b
    B, Hq, Hkv, N, d, dv, causal, packed, dt = shape
    nb, nl, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    st = b.lib.lt_linear_attn_fwd_plan(B, Hq, Hkv, N, d, dv, causal, packed, dt, 148,
                                       ctypes.byref(nb), ctypes.byref(nl), ctypes.byref(ws))
    assert st == 0
    assert (nb.value, nl.value, ws.value) == expect


def test_fwd_plan_pair_forced(sched):
    """The two-launch override keeps the state launch plus the forward launch
    where the one-launch path would apply."""
    sched(kernel="two_launch")
    from causal_linear_attention_chunked_b200 import _binding as b
    nb, nl, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    st = b.lib.lt_linear_attn_fwd_plan(2, 8, 8, 4096, 64, 64, 1, 0, 1, 148,
                                       ctypes.byref(nb), ctypes.byref(nl), ctypes.byref(ws))
    assert st == 0
    assert (nb.value, nl.value, ws.value) == (8, 2, 2 * 8 * 8 * (64 * 64 + 64) * 4)


@pytest.mark.parametrize("case,expect", [
    (dict(d=32), 2), (dict(dtype=3), 2), (dict(B=0), 1), (dict(Hkv=3, Hq=8), 1),
    (dict(causal=5), 1), (dict(packed=2), 1), (dict(out=None), 1), (dict(Hkv=70000, Hq=70000), 1),
])
def test_fwd_plan_rejects_invalid_arguments(case, expect):
    from causal_linear_attention_chunked_b200 import _binding as b
    a = dict(B=1, Hq=8, Hkv=8, N=16, d=64, dv=64, causal=1, packed=0, dtype=1, out=True)
    a.update(case)
    nb, nl, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    st = b.lib.lt_linear_attn_fwd_plan(a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["dv"],
                                       a["causal"], a["packed"], a["dtype"], 148,
                                       ctypes.byref(nb), ctypes.byref(nl),
                                       ctypes.byref(ws) if a["out"] else None)
    assert st == expect
