"""Save and load of a layer's offline artifacts (table + prepared weights), on the CPU: the round
trip is exact, the header fields sit where the format says, and damaged or mismatched files are
rejected."""
import struct

import numpy as np
import pytest
import torch

from w4a4_outlier_separated_b200 import artifacts as A


def _layer(G=32, K=512, N=48, K_L=16, seed=0):
    from w4a4_outlier_separated_b200 import build
    build.build()
    from w4a4_outlier_separated_b200 import osc
    rng = np.random.default_rng(seed)
    L = torch.from_numpy(rng.integers(-1, G, size=K // G).astype(np.int8))
    if K_L == 0:
        L[:] = -1                                             # no compensation columns, no entries
    assert osc.osc_table_kl(L.numpy()) <= K_L
    QW = torch.from_numpy(rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8))
    SW = torch.from_numpy(rng.integers(0, 256, size=osc.osc_scale_bytes(N, K, G)).astype(np.uint8))
    WL = torch.from_numpy(rng.integers(-30000, 30000, size=(N, K_L)).astype(np.int16)) if K_L else None
    return dict(L=L, QW=QW, SW=SW, WL=WL, G=G, K=K, N=N, K_L=K_L)


@pytest.mark.parametrize("G,K_L", [(32, 16), (16, 32), (64, 0)])
def test_round_trip_is_exact(tmp_path, G, K_L):
    d = _layer(G=G, K_L=K_L)
    p = str(tmp_path / "layer.osc")
    A.save_layer(p, d["L"], d["QW"], d["SW"], d["WL"], G=G, K=d["K"], N=d["N"], K_L=K_L, alpha=6.0, min_hits=4)
    r = A.load_layer(p, device="cpu")
    for k in ("L", "QW", "SW"):
        assert torch.equal(r[k], d[k]), k
    assert (r["WL"] is None) == (K_L == 0) and (K_L == 0 or torch.equal(r["WL"], d["WL"]))
    assert (r["G"], r["K"], r["N"], r["K_L"], r["alpha"], r["min_hits"]) == (G, 512, 48, K_L, 6.0, 4)


def test_header_layout(tmp_path):
    d = _layer()
    p = str(tmp_path / "layer.osc")
    A.save_layer(p, d["L"], d["QW"], d["SW"], d["WL"], G=32, K=512, N=48, K_L=16)
    raw = open(p, "rb").read()
    assert raw[:8] == b"OSCLAYR1"
    version, G, K, N, K_L = struct.unpack_from("<5I", raw, 8)
    assert (version, G, K, N, K_L) == (1, 32, 512, 48, 16)
    assert struct.unpack_from("<f", raw, 28)[0] == 5.0
    sizes = struct.unpack_from("<4Q", raw, 40)
    assert sizes == (16, 48 * 256, d["SW"].numel(), 48 * 16 * 2)
    assert len(raw) == 72 + sum(sizes)
    assert raw[72:88] == d["L"].numpy().tobytes()             # the table follows the header


def test_damaged_or_mismatched_files_are_rejected(tmp_path):
    d = _layer()
    p = str(tmp_path / "layer.osc")
    A.save_layer(p, d["L"], d["QW"], d["SW"], d["WL"], G=32, K=512, N=48, K_L=16)
    raw = bytearray(open(p, "rb").read())
    bad = tmp_path / "bad.osc"
    bad.write_bytes(b"XXXXXXXX" + raw[8:])
    with pytest.raises(ValueError, match="not an OSC layer"):
        A.load_layer(str(bad), device="cpu")
    bad.write_bytes(raw[:-5])
    with pytest.raises(ValueError, match="length"):
        A.load_layer(str(bad), device="cpu")
    hacked = bytearray(raw)
    struct.pack_into("<I", hacked, 20, 96)                   # N changed: sizes no longer fit
    bad.write_bytes(bytes(hacked))
    with pytest.raises(ValueError, match="sizes"):
        A.load_layer(str(bad), device="cpu")
    with pytest.raises(ValueError, match="QW"):
        A.save_layer(p, d["L"], d["QW"][:10], d["SW"], d["WL"], G=32, K=512, N=48, K_L=16)


def test_tables_that_do_not_fit_the_layer_are_rejected(tmp_path):
    """Entries outside [-1, G) or more entries than K_L columns hold: refused on save, and on
    load of a file whose table bytes were changed after saving."""
    d = _layer()
    p = str(tmp_path / "layer.osc")
    bad_entry = d["L"].clone()
    bad_entry[3] = 32                                         # channel >= G
    with pytest.raises(ValueError, match="entries must lie"):
        A.save_layer(p, bad_entry, d["QW"], d["SW"], d["WL"], G=32, K=512, N=48, K_L=16)
    many = torch.arange(16, dtype=torch.int8)                 # 16 entries need K_L = 16 ...
    few = _layer(G=32, K_L=0)                                 # ... but this layer has K_L = 0
    with pytest.raises(ValueError, match="more than K_L"):
        A.save_layer(p, many, few["QW"], few["SW"], None, G=32, K=512, N=48, K_L=0)
    A.save_layer(p, d["L"], d["QW"], d["SW"], d["WL"], G=32, K=512, N=48, K_L=16)
    raw = bytearray(open(p, "rb").read())
    raw[72 + 2] = 0x7F                                         # entry 127 >= G in the stored table
    bad = tmp_path / "bad.osc"
    bad.write_bytes(bytes(raw))
    with pytest.raises(ValueError, match="entries must lie"):
        A.load_layer(str(bad), device="cpu")
    d0 = _layer(G=32, K_L=0)
    A.save_layer(p, d0["L"], d0["QW"], d0["SW"], None, G=32, K=512, N=48, K_L=0)
    raw = bytearray(open(p, "rb").read())
    raw[72] = 5                                               # one entry, but K_L = 0 in the header
    bad.write_bytes(bytes(raw))
    with pytest.raises(ValueError, match="more than K_L"):
        A.load_layer(str(bad), device="cpu")
