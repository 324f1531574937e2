"""The largest table the quantize stages on chip (K/G = 1024 groups, every one protected, so
K_L = 1024 columns of B and 16 compensation stages in the product), checked against the oracle:
codes, scales and B bit for bit, Y within the product's tolerance."""
import numpy as np
import pytest
import torch

from tests.conftest import to_dev, to_np
from tests.test_gpu_linear import _compare
from tests.test_gpu_quantize import _check_quant
from w4a4_outlier_separated_b200 import inputs as I

pytestmark = pytest.mark.gpu


def test_largest_table_full_protection(oracle, osc):
    M, K, N, G = 130, 32768, 256, 32
    rng = np.random.default_rng(11)
    x = rng.standard_normal((M, K))
    L = rng.integers(0, G, K // G).astype(np.int8)          # every group protected
    x[:, np.arange(K // G) * G + L] *= 40.0                  # its outlier channel, on every row
    X = I.bf16_bits(x)
    W = I.gen_weights(N, K, seed=12)
    K_L = I.pad16(oracle.table_count(L))
    assert K_L == 1024
    _check_quant(oracle, osc, X, G, L, K_L)                  # codes, scales, B bit for bit
    Ld = to_dev(L)
    QX, SX, B = osc.quantize(to_dev(X), G, Ld, K_L)
    QW, SW, WL = osc.prepare_weight(to_dev(W), G, Ld, K_L)
    Y, Yf = osc.linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, want_f32=True)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    cw, ew, WLr = oracle.osc_prepare_weight(W, G, L, K_L)
    ref = oracle.osc_forward(X, G, L, K_L, cw, ew, WLr)["Y"]
    _compare(to_np(Y), to_np(Yf), ref)
