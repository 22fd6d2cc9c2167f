import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
# The mutation test points this at a copy of the oracle package with one planted mistake.
if os.environ.get("R2L_ORACLE_PKG_DIR"):
    sys.path.insert(0, os.environ["R2L_ORACLE_PKG_DIR"])


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) and the built CUDA library")


def rel_err(got, ref):
    """Max over elements of |got - ref| / max(|ref|, rms(ref)).

    Element-wise relative error with a floor at the reference RMS so that outputs
    that cancel to ~0 do not blow the ratio up.
    """
    import numpy as np

    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    den = np.maximum(np.abs(ref), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(got - ref) / den))


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    oracle.build()
    return oracle
