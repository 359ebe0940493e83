"""Throughput of the causal linear-attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lt|reference]

One step = one forward pass (all stages of the chunked path) over one batch
of the headline workload: bf16, B=2, H=8, N=4096, d=dv=64, causal (the
lineartile page's usage example: d_model 512 over 8 heads).  The metric is
B*H*N tokens per second over the whole job, with inputs resident in HBM.

Timing: W untimed warm-up steps, then exactly K steps replayed from CUDA
graphs on one stream, bracketed by a barrier and a device synchronisation,
timed with CUDA events; the maximum over ranks is used.  One workload
(33.6 MB) fits in L2, so the steps rotate over R input sets whose total is
at least 3x the L2 size.  N > 1 runs one rank per GPU, each on its own batch
(weak scaling, no data-path collective).

Rank 0 prints one JSON line.  Alongside the metric it carries
  roofline      achieved HBM GB/s of the forward kernel (algorithmic bytes /
                average launch time) against the measured copy bandwidth;
  cpu_baseline  the fp64 oracle timed on the host cores (bounded sample);
  e2e           the same metric through the C ABI with pinned host buffers,
                host<->device copies inside the timed region;
  clocks        SM clocks and throttle reasons sampled during the timed region;
  extra         the other workloads (long sequence, GQA d=128, packed,
                non-causal, decode) measured the same way, for context.
--impl reference times the fp64 CPU oracle on the same workload instead.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from causal_linear_attention_chunked_b200 import inputs  # noqa: E402

HEADLINE = "bf16_b2h8n4096d64"
METRIC = "causal linear-attn fwd tokens/s (B·H·N per s) and % of roofline on 1 B200"
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ helpers
def algorithmic_bytes(w, total_tokens=None):
    """Q, K, V read once and O written once (bytes per forward pass)."""
    es = 2 if w.dtype == torch.bfloat16 else 4
    T = total_tokens if total_tokens is not None else w.B * w.N
    return T * (w.Hq * w.d + w.Hkv * (w.d + w.dv) + w.Hq * w.dv) * es


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


FORWARD_SOURCES = (
    "causal_linear_attention_chunked_b200/csrc/state_bf16_sm100.cu",
    "causal_linear_attention_chunked_b200/csrc/fwd_bf16_block_sm100.cu",
    "causal_linear_attention_chunked_b200/csrc/fwd_bf16_fused_sm100.cu",
    "causal_linear_attention_chunked_b200/csrc/fwd_bf16_sm100.cu",
    "causal_linear_attention_chunked_b200/csrc/fwd_common.cuh",
    "causal_linear_attention_chunked_b200/csrc/lt_ptx.cuh")


def source_digest(files=FORWARD_SOURCES):
    h = hashlib.sha256()
    for rel in files:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload, kernel_label=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel it names (else None).  The summary
    lists the files its digest covers (`source_files`, default: every forward
    source) and the kernel it measured (`kernel`), which must be the kernel
    this run timed."""
    path = os.path.join(ROOT, "profiles", "traffic_lt_fwd_bf16_%s.txt" % workload)
    try:
        kv = {}
        for line in open(path):
            if "=" in line and not line.startswith("#"):
                a, b = line.split("=", 1)
                kv[a.strip()] = b.strip()
        files = kv["source_files"].split() if "source_files" in kv else FORWARD_SOURCES
        if kv.get("source_digest") != source_digest(files):
            return None
        if "kernel" in kv and (kernel_label is None or kv["kernel"] not in kernel_label):
            return None
        return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons every 100 ms in the background."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        try:
            self.idx = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.idx = str(device.index or 0)
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
        note = None
        if not inside and rows:
            # timed region shorter than the sampling interval: nearest samples
            inside = sorted(rows, key=lambda r: abs(r[0] - 0.5 * (t0 + t1)))[:2]
            note = "timed region shorter than the sampling interval; nearest samples"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inside:
            flags = r[3][1:5]
            for n, f in zip(names, flags):
                if f.lower().startswith("active"):
                    reasons.add(n)
        out = {"sm_mhz": statistics.median(r[1] for r in inside),
               "sm_max_mhz": max(r[2] for r in inside), "reasons": sorted(reasons),
               "samples": len(inside)}
        if note:
            out["note"] = note
        return out


# ----------------------------------------------------------- distributed
def dist_setup(want, backend=None):
    """One process per GPU under torchrun: (world, rank, local rank).  NCCL on
    GPUs; gloo when there is no GPU (the host-side tests of this path)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif want > 1:
        raise SystemExit("--gpus %d needs a torchrun launch (one process per GPU)" % want)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base, rank):
    """Each rank draws its own batch: the workload's seed offset by rank."""
    return base + 1000 * rank


def whole_job_rate(units_per_rank, world, ms_max):
    """Units of all ranks over the slowest rank's time (weak scaling)."""
    return units_per_rank * world / (ms_max / 1e3)


# --------------------------------------------------------------- GPU arm
def make_sets(w, R, seed_base, device, lengths=None):
    sets = []
    for r in range(R):
        q, k, v, cu = inputs.make(w, seed=seed_base + r, lengths=lengths)
        sets.append((q.to(device), k.to(device), v.to(device),
                     None if cu is None else cu.to(device),
                     torch.empty(q.shape[:-1] + (w.dv,), dtype=w.dtype, device=device)))
    return sets


def capture(fn_list, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        for fn in fn_list:
            fn()
    return g


def timed_graph_steps(step_fns, K, stream, world):
    """Replay exactly K steps (step i runs step_fns[i % R]) from CUDA graphs;
    returns (elapsed ms, max over ranks)."""
    R = len(step_fns)
    G = max(R, min(K, (4096 // R) * R))
    full, rem = divmod(K, G)
    g_full = capture([step_fns[i % R] for i in range(G)], stream) if full else None
    g_rem = capture([step_fns[i % R] for i in range(rem)], stream) if rem else None
    # untimed replays until the GPU has run for a while (clocks ramp up after
    # idle); the timed region below still covers exactly K steps
    warm = g_full if g_full is not None else g_rem
    t_end = time.time() + 0.25
    while time.time() < t_end:
        with torch.cuda.stream(stream):
            warm.replay()
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    ms = e0.elapsed_time(e1)
    return ms, max_over_ranks(ms, world), (t0, t1)


def fwd_step_fns(L, w, sets, stream):
    fns = []
    for (q, k, v, cu, out) in sets:
        def f(q=q, k=k, v=v, cu=cu, out=out):
            L.linear_attn_fwd(q, k, v, causal=w.causal, eps=w.eps, cu_seqlens=cu, out=out,
                              stream=stream)
        fns.append(f)
    return fns


def measure_workload(L, w, K, W, stream, device, world, l2_bytes, rank=0):
    """Throughput of one workload: (tokens/s, ms per step, bytes per step)."""
    q0, _, _, cu0 = inputs.make(w)
    total_tokens = int(cu0[-1]) if cu0 is not None else w.B * w.N
    nbytes = algorithmic_bytes(w, total_tokens)
    R = max(1, math.ceil(3 * l2_bytes / nbytes))
    lengths = None if cu0 is None else (cu0[1:] - cu0[:-1]).tolist()  # same lengths in every set
    sets = make_sets(w, R, rank_seed(w.seed, rank), device, lengths)
    fns = fwd_step_fns(L, w, sets, stream)
    with torch.cuda.stream(stream):
        for i in range(W):
            fns[i % R]()
    torch.cuda.synchronize()
    assert L.get_last_device_error(stream) == 0
    ms, ms_max, window = timed_graph_steps(fns, K, stream, world)
    assert L.get_last_device_error(stream) == 0
    units = total_tokens * w.Hq
    del sets
    return units, ms_max / K, nbytes, R, window


def measure_from_state(L, w, K, stream, device, l2_bytes, peak):
    """The headline shape through lt_linear_attn_fwd_state: every pass starts
    from a given state and returns the final state (prefill -> decode
    handoff).  Bytes: Q, K, V, O plus the state read and written."""
    total_tokens = w.B * w.N
    state_bytes = w.B * w.Hkv * (w.d * w.dv + w.d) * 4
    nbytes = algorithmic_bytes(w, total_tokens) + 2 * state_bytes
    R = max(1, math.ceil(3 * l2_bytes / nbytes))
    sets = make_sets(w, R, w.seed + 500, device)
    g = inputs.generator(w.seed + 499)
    S0 = torch.rand((w.B, w.Hkv, w.d, w.dv), generator=g).to(device)
    z0 = torch.rand((w.B, w.Hkv, w.d), generator=g).to(device) + 1.0
    S1 = torch.empty_like(S0)
    z1 = torch.empty_like(z0)
    fns = []
    for (q, k, v, _, out) in sets:
        def f(q=q, k=k, v=v, out=out):
            L.linear_attn_fwd_state(q, k, v, causal=w.causal, eps=w.eps, S0=S0, z0=z0, out=out,
                                    S_out=S1, z_out=z1, stream=stream)
        fns.append(f)
    with torch.cuda.stream(stream):
        for i in range(3):
            fns[i % R]()
    torch.cuda.synchronize()
    assert L.get_last_device_error(stream) == 0
    ms, _, _ = timed_graph_steps(fns, K, stream, 1)
    assert L.get_last_device_error(stream) == 0
    ms /= K
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"workload": w.name + "_from_state", "tokens_per_s": total_tokens * w.Hq / (ms / 1e3),
            "ms_per_step": ms, "achieved_gbs": ach, "roofline_frac": ach / peak,
            "algorithmic_bytes": nbytes,
            "note": "lt_linear_attn_fwd_state: given initial state, final state returned "
                    "(one cooperative launch: S0 folded into every block's carry, the last "
                    "block writes the final state)"}


def measure_decode(L, stream, device, steps=1000, reps=3):
    c = inputs.DECODE
    B, Hq, Hkv, d, dv = c["B"], c["Hq"], c["Hkv"], c["d"], c["dv"]
    g = inputs.generator(c["seed"])
    toks = [inputs.make_decode_step(B, Hq, Hkv, d, dv, c["dtype"], c["scale"], g)
            for _ in range(steps)]
    qs = torch.stack([t[0] for t in toks]).to(device)
    ks = torch.stack([t[1] for t in toks]).to(device)
    vs = torch.stack([t[2] for t in toks]).to(device)
    S = torch.zeros(B, Hkv, d, dv, device=device)
    z = torch.zeros(B, Hkv, d, device=device)
    out = torch.empty(B, Hq, dv, dtype=c["dtype"], device=device)
    fns = [lambda i=i: L.linear_attn_decode_step(qs[i], ks[i], vs[i], S, z, eps=c["eps"],
                                                 out=out, stream=stream) for i in range(steps)]
    with torch.cuda.stream(stream):
        fns[0]()
    torch.cuda.synchronize()
    gph = capture(fns, stream)
    best = None
    for _ in range(reps):
        S.zero_()
        z.zero_()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            gph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    us_step = best * 1000.0 / steps
    state_bytes = B * Hkv * (d * dv + d) * 4 * 2
    io_bytes = B * (Hq * d + Hkv * (d + dv) + Hq * dv) * 2
    # the launch floor: a graph of as many one-element fills, same stream
    one = torch.zeros(1, device=device)
    floor = capture([lambda: one.fill_(1.0)] * steps, stream)
    with torch.cuda.stream(stream):
        floor.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        floor.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    floor_us = e0.elapsed_time(e1) * 1000.0 / steps
    return {"workload": c["name"], "tokens_per_s": B * steps / (best / 1e3),
            "head_tokens_per_s": B * Hq * steps / (best / 1e3), "us_per_step": us_step,
            "bytes_per_step": state_bytes + io_bytes,
            "achieved_gbs": (state_bytes + io_bytes) / (us_step * 1e-6) / 1e9,
            "graph_floor_us_per_kernel": floor_us,
            "note": "1000 steps replayed as one CUDA graph; the 8.4 MB fp32 state is "
                    "L2-resident. graph_floor: the same graph shape of one-element fill kernels"}


def measure_backward(L, w, stream, device, peak, reps=10):
    """lt_linear_attn_bwd on the workload's shape: dQ, dK, dV for a random
    upstream gradient.  Algorithmic bytes: q, k, v and dO read once, dq, dk,
    dv written once."""
    q, k, v, _ = inputs.make(w, seed=w.seed + 700)
    q, k, v = q.to(device), k.to(device), v.to(device)
    g = inputs.generator(w.seed + 701)
    dout = torch.randn(q.shape[:-1] + (w.dv,), generator=g).to(w.dtype).to(device)
    fns = [lambda: L.linear_attn_bwd(q, k, v, dout, causal=w.causal, eps=w.eps, stream=stream)]
    with torch.cuda.stream(stream):
        for _ in range(2):
            fns[0]()
    torch.cuda.synchronize()
    assert L.get_last_device_error(stream) == 0
    # reps calls per graph (the stream-ordered workspace becomes graph memory
    # nodes); the best of three replays
    gph = capture(fns * reps, stream)
    best = None
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            gph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1)
        best = t if best is None else min(best, t)
    assert L.get_last_device_error(stream) == 0
    e_ms = best
    ms = e_ms / reps
    es = 2 if w.dtype == torch.bfloat16 else 4
    nbytes = w.B * w.N * (2 * w.Hq * w.d + 2 * w.Hkv * (w.d + w.dv) + w.Hq * w.dv) * es
    ach = nbytes / (ms * 1e-3) / 1e9
    fma = backward_fma(w)
    tflops = 2 * fma / (ms * 1e-3) / 1e12
    return {"workload": w.name + "_backward", "tokens_per_s": w.B * w.Hq * w.N / (ms / 1e3),
            "ms_per_step": ms, "achieved_gbs": ach, "roofline_frac": ach / peak,
            "algorithmic_bytes": nbytes, "executed_fma": fma, "achieved_tflops": tflops,
            "alu_peak_tflops": FP32_ALU_TFLOPS, "alu_frac": tflops / FP32_ALU_TFLOPS,
            "note": "lt_linear_attn_bwd: a block-sum launch and two fp32 FMA scans, one CTA per "
                    "(sequence, head, block); 10 calls replayed as one CUDA graph, best of three "
                    "replays; alu_frac: the "
                    "FMAs the kernels execute (masked tiles whole) against 148 SMs x 128 fp32 "
                    "lanes x 2 x 1.965 GHz"}


# fp32 FMA peak of the B200: 148 SMs x 128 lanes x 2 flops x 1.965 GHz (max SM clock)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_fma(w):
    """FMAs the backward kernels execute per call (32-token chunks, masked
    tiles computed whole): the block-sum launch, the dq scan per query head
    and the dk, dv scan per KV head."""
    C, d, dv, G = 32, w.d, w.dv, w.Hq // w.Hkv
    chunks = w.B * ((w.N + C - 1) // C)
    st = (d * dv + d) * C  # one chunk's phi^T [x | 1]
    if w.causal:
        k1 = C * C * d + C * (C + d) + C * dv * (C + d) + C * C * dv + C * d * (C + dv) + 2 * st
        k2 = 2 * C * d * dv + G * (2 * C * C * d + 2 * C * C * dv + st)
    else:
        k1 = C * d + 2 * C * d * dv + st
        k2 = 2 * C * d * dv
    return chunks * (w.Hkv * st + w.Hq * k1 + w.Hkv * k2)


def measure_e2e(L, w, steps, stream, device):
    q, k, v, cu = inputs.make(w)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty(q.shape[:-1] + (w.dv,), dtype=w.dtype).pin_memory()
    L.linear_attn_fwd_host(qh, kh, vh, causal=w.causal, eps=w.eps, device=device, stream=stream,
                           out_host=oh)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        L.linear_attn_fwd_host(qh, kh, vh, causal=w.causal, eps=w.eps, device=device,
                               stream=stream, out_host=oh)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = qh.numel() * qh.element_size() * 3
    d2h = oh.numel() * oh.element_size()
    return {"value": w.B * w.Hq * w.N / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": steps, "path": "lt_linear_attn_fwd via linear_attn_fwd_host (pinned host "
                                    "buffers, copies + kernel on one stream)"}


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def measure_eager(L, w, stream, device, calls=200):
    """Per-call cost of eager (not graph-captured) calls of the headline
    shape: the host time to issue one call through the C ABI (argument
    checks, plan, workspace, launch), and the device time per call when calls
    are issued back to back without a graph."""
    q, k, v, cu = inputs.make(w)
    q, k, v = q.to(device), k.to(device), v.to(device)
    out = torch.empty(q.shape[:-1] + (w.dv,), dtype=w.dtype, device=device)
    for _ in range(5):
        L.linear_attn_fwd(q, k, v, causal=w.causal, eps=w.eps, out=out, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    t0 = time.perf_counter()
    for _ in range(calls):
        L.linear_attn_fwd(q, k, v, causal=w.causal, eps=w.eps, out=out, stream=stream)
    t1 = time.perf_counter()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"workload": w.name + "_eager", "host_us_per_call": (t1 - t0) * 1e6 / calls,
            "device_us_per_call": e0.elapsed_time(e1) * 1e3 / calls, "calls": calls,
            "note": "eager calls through the Python binding and the C ABI, no CUDA graph; "
                    "host time covers marshalling, argument checks, plan, workspace and launch"}


def cpu_baseline(w, budget_s=10.0):
    import oracle  # the fp64 CPU oracle, as it stands (test infrastructure)
    q, k, v, _ = inputs.make(w)
    reps, t0 = 0, time.time()
    while True:
        oracle.fwd_recurrent(q, k, v, causal=w.causal, eps=w.eps)
        reps += 1
        if time.time() - t0 >= budget_s:
            break
    dt = time.time() - t0
    return {"value": reps * w.B * w.Hq * w.N / dt, "unit": "tokens/s",
            "cores": oracle.num_threads(), "cpu_model": cpu_model(), "kind": "oracle",
            "sample": "%d full passes of %s (fp64 recurrent form, OpenMP over (sequence, head)) "
                      "in %.1f s" % (reps, w.name, dt)}


def run_lt(args):
    world, rank, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import causal_linear_attention_chunked_b200 as L
    w = inputs.WORKLOADS[args.workload]
    props = torch.cuda.get_device_properties(device)
    l2 = props.L2_cache_size
    stream = torch.cuda.Stream(device)
    sampler = ClockSampler(device)
    sampler.start()
    units, ms_step, nbytes, R, window = measure_workload(L, w, args.steps, args.warmup, stream,
                                                         device, world, l2, rank)
    clocks = sampler.summary(*window)
    sampler.stop()
    value = whole_job_rate(units, world, ms_step)
    peak, peak_kind = peaks()
    achieved = nbytes / (ms_step * 1e-3) / 1e9
    packed = w.packed_len is not None
    nblk, per_step, ws_bytes = L.linear_attn_fwd_plan(w.B, w.Hq, w.Hkv, 1 if packed else w.N,
                                                      w.d, w.dv, causal=w.causal, packed=packed)
    d64 = w.d == 64 and w.dv == 64
    if per_step == 2:
        kern = "lt_block_state_kernel + " + ("lt_block_fwd_kernel" if d64 else "lt_fwd_bf16_kernel")
    elif d64 and nblk > 1:
        kern = "lt_fused_fwd_kernel (one cooperative launch)"
    else:
        kern = "lt_block_fwd_kernel" if d64 else "lt_fwd_bf16_kernel"
    traffic = committed_traffic(w.name, kern)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H_q": w.Hq, "H_kv": w.Hkv, "N": w.N, "d": w.d,
                   "dv": w.dv, "causal": w.causal, "eps": w.eps, "global_batch": w.B * world,
                   "seq_len": w.N, "parallelism": "dp%d (independent batches)" % world,
                   "l2": "rotating %d input sets (%.0f MB, >= 3x the %.0f MB L2)" % (
                       R, R * nbytes / 1e6, l2 / 1e6),
                   "timing": "CUDA events around exactly K steps replayed from CUDA graphs"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind
                     if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": "one forward pass (%s, %d block(s) per sequence)" % (kern, nblk),
                     "algorithmic_bytes_per_launch": nbytes,
                     "avg_launch_us": ms_step * 1e3},
        "clocks": clocks,
        "gpu_launches": args.steps * per_step,
    }
    if args.profile:
        pass
    elif rank == 0 and world == 1:
        line["e2e"] = measure_e2e(L, w, min(args.steps, 50), stream, device)
    elif rank == 0:
        line["e2e"] = measure_e2e(L, w, min(args.steps, 50), stream, device)
        line["e2e"]["value"] *= world
        line["e2e"]["note"] = "rank 0's end-to-end rate times the number of ranks"
    if rank == 0 and not args.no_extra and not args.profile:
        extra = []
        for name in args.extra:
            ew = inputs.WORKLOADS[name]
            u, ms, nb, RR, _ = measure_workload(L, ew, args.extra_steps, 3, stream, device, 1, l2)
            ach = nb / (ms * 1e-3) / 1e9
            extra.append({"workload": name, "tokens_per_s": u / (ms / 1e3), "ms_per_step": ms,
                          "achieved_gbs": ach, "roofline_frac": ach / peak,
                          "algorithmic_bytes": nb})
        extra.append(measure_from_state(L, inputs.WORKLOADS[HEADLINE], args.extra_steps, stream,
                                        device, l2, peak))
        extra.append(measure_decode(L, stream, device))
        extra.append(measure_eager(L, w, stream, device))
        extra.append(measure_backward(L, w, stream, device, peak))
        line["extra"] = extra
    if rank == 0 and world == 1 and not args.profile:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The fp64 oracle on the host cores, same workload and metric."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = inputs.WORKLOADS[args.workload]
    q, k, v, _ = inputs.make(w)
    # each step: a prefix of the workload (every batch row and head, first n
    # tokens; causal prefixes are exact sub-problems), sized so that the run
    # stays within about two minutes
    per_tok = None
    n = w.N
    t0 = time.time()
    oracle.fwd_recurrent(q, k, v, causal=w.causal, eps=w.eps)
    per_tok = (time.time() - t0) / w.N
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(16, min(w.N, budget / per_tok)))
    qs, ks, vs = (t[:, :n].contiguous() for t in (q, k, v))
    for _ in range(args.warmup):
        oracle.fwd_recurrent(qs, ks, vs, causal=w.causal, eps=w.eps)
    t0 = time.time()
    for _ in range(args.steps):
        oracle.fwd_recurrent(qs, ks, vs, causal=w.causal, eps=w.eps)
    dt = time.time() - t0
    value = args.steps * w.B * w.Hq * n / dt
    sample = "each step: the first %d of %d tokens of %s, all %d batch rows x %d heads " \
             "(fp64 recurrent form)" % (n, w.N, w.name, w.B, w.Hq)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "H_q": w.Hq, "H_kv": w.Hkv, "N": w.N,
                       "d": w.d, "dv": w.dv, "causal": w.causal, "eps": w.eps},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("lt", "reference"), default="lt")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--extra-steps", type=int, default=200)
    ap.add_argument("--profile", action="store_true",
                    help="headline workload only (no e2e, CPU baseline or extras): for ncu")
    ap.add_argument("--extra", nargs="*", default=[
        "bf16_b1h8n65536d64", "bf16_b1h8n65536d64_noncausal", "bf16_gqa_b2hq32hkv8n16384d128",
        "bf16_varlen64_h8d64"])
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_lt(args)


if __name__ == "__main__":
    main()
