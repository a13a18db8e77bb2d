"""Shared pytest set-up: the ``gpu`` marker, import paths and the golden-file reader."""
from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name: str):
    """Return the non-comment lines of tests/golden/<name>: 'key: values' lines as a dict
    of float lists, other lines as lists of tokens under the key None."""
    out: dict = {None: []}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                out[k.strip()] = [float(t) for t in v.split()]
            else:
                out[None].append(line.split())
    return out


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
