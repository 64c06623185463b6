import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


def rel_err(got, ref):
    """max |got - ref| / RMS(ref) over the checked (non-NaN) elements."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    m = ~np.isnan(ref)
    rms = np.sqrt(np.mean(ref[m] ** 2))
    return float(np.max(np.abs(got[m] - ref[m])) / max(rms, 1e-300))


@pytest.fixture
def relerr():
    return rel_err


def bf16_storage_ratio(got, ref, allowance=4e-3, rms=None):
    """Worst ratio of |got - ref| to the error a bf16-stored result can carry:
    half a bf16 ulp of the exact value (2^-8 |ref|, rounding to 8 significant
    bits) plus an accumulation allowance times an RMS (of ref unless given).
    <= 1 passes."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    m = ~np.isnan(ref)
    if rms is None:
        rms = np.sqrt(np.mean(ref[m] ** 2))
    bound = 2.0 ** -8 * np.abs(ref[m]) + allowance * max(rms, 1e-300)
    return float(np.max(np.abs(got[m] - ref[m]) / bound))
