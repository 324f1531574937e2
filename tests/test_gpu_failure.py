"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies runs out,
the kernel records OSC_ERR_TIMEOUT in the status word and exits, the host reads and clears it,
and the context stays usable for the next call."""
import time

import numpy as np
import pytest
import torch

from tests.conftest import to_dev, to_np
from w4a4_outlier_separated_b200 import inputs as I

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports(oracle, osc):
    assert osc.osc_status() == (0, 0)
    t0 = time.perf_counter()
    osc.osc_selftest_timeout(10_000)                 # 10 ms
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert osc.osc_status() == (-5, 1)               # OSC_ERR_TIMEOUT, device code 1
    assert osc.osc_status() == (0, 0)                # read and cleared
    # the context is still good: a small quantize matches the oracle
    c = I.tiny_case()
    QX, SX, B = osc.quantize(to_dev(c.X), 32, to_dev(c.planted), 16)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    Xz, Bref = oracle.extract(c.X, 32, c.planted, 16)
    assert np.array_equal(to_np(B), Bref)
