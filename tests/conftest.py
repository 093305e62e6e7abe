"""Shared pytest set-up: the `gpu` marker and import paths.

Tests marked `gpu` need a CUDA device and the built library; everything else
runs on the CPU (`pytest -m "not gpu"`)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libmoeq.so")


@pytest.fixture(scope="session")
def ref():
    from oracle import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def syn():
    from synth import synth
    synth.build(device=False)
    return synth
