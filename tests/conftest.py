"""Shared pytest setup.

Markers: ``gpu`` marks tests that need a CUDA device (run with ``-m gpu``);
everything else runs on a CPU-only machine (``-m "not gpu"``).
"""
import ast
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def load_golden(name: str) -> dict:
    """Parse a ``key = python-literal`` fixture under ``tests/golden/``;
    ``#`` lines are the fixture's derivation and citations."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            s = line.strip()
            if not s or s.startswith("#"):
                continue
            key, _, val = s.partition("=")
            out[key.strip()] = ast.literal_eval(val.strip())
    return out


@pytest.fixture(scope="session")
def golden():
    return load_golden
