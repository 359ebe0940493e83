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
