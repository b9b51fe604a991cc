import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Output tolerance for the additive-quantised product, per element:
#   |y_gpu - y_ref| <= RTOL * sum_i |s_o| |W_oi| |x_ib| + ATOL
# where y_ref is the fp64 oracle.  Dequantised weights and codes are compared
# bit for bit.
RTOL = 1e-2
ATOL = 1e-3


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def within_tolerance(y_gpu, y_ref, bound):
    import numpy as np
    err = np.abs(np.asarray(y_gpu, dtype=np.float64) - y_ref)
    lim = RTOL * bound + ATOL
    return err <= lim, err, lim


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
