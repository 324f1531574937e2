"""osc_linear_splitk_noalloc, the allocation-free split product, against osc_linear_splitk.

Some callers of this library cannot allocate device memory at all: an inference-engine plugin
that is handed only its input and output buffers, or a serving loop that allows no allocation
once it runs. They cannot give osc_linear_splitk the workspace its fp32 partials need, so
osc_linear_splitk_noalloc keeps those partials in one fixed 16 MiB buffer inside the library.

This file calls it through the C ABI and compares its output with the workspace form's on the
same inputs, for two calls in a row: the second call uses a different, smaller problem, so any
partials the first call left in the shared buffer would show up in its result. The file is
named to be collected after every other test file, and it needs nothing from them: it passes
alone in a fresh process as well as after the rest of the suite."""
import numpy as np
import pytest
import torch

from tests._layout import bf16_ulp
from tests.conftest import to_dev, to_np
from w4a4_outlier_separated_b200 import inputs as I

pytestmark = pytest.mark.gpu
REL = 1e-3            # the tolerance of the product's parity tests


def _layer(osc, M):
    """QKV-shaped layer (K = 4096, N = 6144, G = 32) at M token rows: table by osc_build_table,
    weights by osc_prepare_weight, activations by osc_quantize, all on the GPU."""
    c = I.qkv_case(M)
    K, N, G = c.K, c.N, c.G
    Ld = torch.empty(K // G, dtype=torch.int8, device="cuda")
    osc.osc_build_table(to_dev(c.calib), G, 5.0, 5, Ld)
    K_L = osc.osc_table_kl(Ld.cpu().numpy())
    QW, SW, WL = osc.prepare_weight(to_dev(c.W), G, Ld, K_L)
    QX, SX, B = osc.quantize(to_dev(c.X), G, Ld, K_L)
    return dict(QX=QX, SX=SX, B=B, QW=QW, SW=SW, WL=WL, M=M, N=N, K=K, G=G, K_L=K_L)


def _both(osc, L):
    """(bf16 Y, fp32 Y) from the workspace form and from the allocation-free form."""
    M, N, K, G, K_L = L["M"], L["N"], L["K"], L["G"], L["K_L"]
    args = (L["QX"], L["SX"], L["B"], L["QW"], L["SW"], L["WL"], M, N, K, G, K_L)
    nbytes = osc.osc_linear_workspace_bytes(M, N, K, K_L)
    assert 0 < nbytes <= 16 << 20                   # the split is in use and fits the fixed buffer
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = []
    for noalloc in (False, True):
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
        if noalloc:
            osc.osc_linear_splitk_noalloc(*args, Y, Yf)
        else:
            osc.osc_linear_splitk(*args, Y, ws, Yf)
        out.append((Y, Yf))
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    return out


def _close(ref, got):
    (Yr, Yfr), (Yg, Yfg) = ref, got
    yr, yg = to_np(Yfr).astype(np.float64), to_np(Yfg).astype(np.float64)
    ymax = np.abs(yr).max()
    assert np.abs(yg - yr).max() <= REL * ymax
    br = I.bf16_to_f32(to_np(Yr)).astype(np.float64)
    bg = I.bf16_to_f32(to_np(Yg)).astype(np.float64)
    assert np.all(np.abs(bg - br) <= REL * ymax + bf16_ulp(br))


def test_noalloc_matches_the_workspace_form_on_two_calls_in_a_row(osc):
    first = _layer(osc, 16)                          # the most rows the split takes
    ref, got = _both(osc, first)
    _close(ref, got)
    second = _layer(osc, 5)                          # smaller: the first call's partials remain around it
    ref, got = _both(osc, second)
    _close(ref, got)
