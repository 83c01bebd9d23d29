"""Shared test set-up: the ``gpu`` marker, import paths and small helpers."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def rel_l2_per_slice(x, ref, axes):
    """max over slices of ||x - ref||_2 / max(||ref||_2, 1e-30), the norms
    taken over ``axes`` (the error metric every parity bar uses)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.sqrt(((x - ref) ** 2).sum(axis=axes))
    den = np.maximum(np.sqrt((ref ** 2).sum(axis=axes)), 1e-30)
    return float((num / den).max())


@pytest.fixture(scope="session")
def oracle_mod():
    from oracle import oracle
    oracle.load()
    return oracle
