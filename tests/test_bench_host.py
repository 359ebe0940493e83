"""Host logic of bench.py (CPU only): a committed DRAM-traffic figure is
reported only for the kernel it measured and only while the sources its
digest covers are unchanged."""
import os
import shutil

import bench

SRC = "causal_linear_attention_chunked_b200/csrc/fwd_bf16_fused_sm100.cu"


def _fake_root(tmp_path):
    os.makedirs(tmp_path / os.path.dirname(SRC))
    shutil.copy(os.path.join(bench.ROOT, SRC), tmp_path / SRC)
    os.makedirs(tmp_path / "profiles")
    return tmp_path


def _write_traffic(root, digest, kernel="lt_fused_fwd_kernel"):
    (root / "profiles" / "traffic_lt_fwd_bf16_wl.txt").write_text(
        "# test\nkernel = %s\nsource_files = %s\nsource_digest = %s\n"
        "dram_bytes_per_launch = 1234\n" % (kernel, SRC, digest))


def test_committed_traffic_matches_kernel_and_digest(tmp_path, monkeypatch):
    root = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    digest = bench.source_digest([SRC])
    _write_traffic(root, digest)
    assert bench.committed_traffic("wl", "lt_fused_fwd_kernel (one cooperative launch)") == 1234
    # another kernel timed: not this figure
    assert bench.committed_traffic("wl", "lt_block_state_kernel + lt_block_fwd_kernel") is None
    # a covered source changed since the capture: stale
    with open(root / SRC, "a") as f:
        f.write("\n// edited\n")
    assert bench.committed_traffic("wl", "lt_fused_fwd_kernel") is None
    # no summary at all
    assert bench.committed_traffic("other", "lt_fused_fwd_kernel") is None


def test_committed_headline_traffic_names_the_one_launch_kernel():
    kv = {}
    path = os.path.join(bench.ROOT, "profiles",
                        "traffic_lt_fwd_bf16_%s.txt" % bench.HEADLINE)
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            a, b = line.split("=", 1)
            kv[a.strip()] = b.strip()
    assert kv["kernel"] == "lt_fused_fwd_kernel"
    assert all(os.path.exists(os.path.join(bench.ROOT, f)) for f in kv["source_files"].split())
