import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and libosc.so")


@pytest.fixture(scope="session")
def oracle():
    from oracle import oracle as O
    O.build()
    return O


@pytest.fixture(scope="session")
def osc():
    """The CUDA library's binding (built in-tree if stale); fails loudly without a GPU."""
    import torch
    from w4a4_outlier_separated_b200 import build as B
    B.build()
    from w4a4_outlier_separated_b200 import osc as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


def to_dev(a, dtype=None):
    """numpy -> CUDA tensor (bf16 bit patterns travel as int16)."""
    import numpy as np
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    t = torch.from_numpy(a).cuda()
    return t if dtype is None else t.to(dtype)


def to_np(t, dtype=None):
    import numpy as np
    import torch
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    a = t.detach().cpu().numpy()
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    return a if dtype is None else a.astype(dtype)
