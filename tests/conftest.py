"""Shared pytest configuration.

Markers: ``gpu`` for tests that need a CUDA device (run on the B200 machine);
everything else runs on the CPU.  The oracle library (plain C) and the CUDA
library are (re)built here when missing or older than their sources, so a
fresh checkout can run the suite directly.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    from oracle import build as obuild
    obuild.build()
    try:
        from causal_linear_attention_chunked_b200 import build as lbuild
    except ImportError:
        return
    lbuild.build()


def cuda_available():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture
def sched():
    """Set the library's diagnostic schedule override for one test:
    ``sched(kernel=..., blocks=...)`` updates the given fields (kernel
    "auto" | "two_launch" | "general"; blocks 0 = the library's choice); the
    override is reset to the library's choice when the test ends."""
    from causal_linear_attention_chunked_b200 import _binding as b
    state = {"kernel": "auto", "blocks": 0}

    def set_(kernel=None, blocks=None):
        if kernel is not None:
            state["kernel"] = kernel
        if blocks is not None:
            state["blocks"] = blocks
        b.set_schedule(state["kernel"], state["blocks"])

    set_()
    yield set_
    b.set_schedule("auto", 0)
