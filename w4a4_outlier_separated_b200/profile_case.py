"""Run the kernels of ONE workload of the OSC path a few times and exit: the process to put
under a profiler (one kernel, a few launches, a small device footprint), as opposed to
bench.py, which sweeps every row.

  python -m w4a4_outlier_separated_b200.profile_case CASE [--launches N] [--m M] [--g G]

CASE:
  qkv           osc_quantize + osc_linear, QKV projection (K=4096, N=6144), M=--m (2048), G=--g (32)
  weight_bound  osc_linear alone at few token rows (QKV weights, M=--m, default 16)
  weight_bound_split  osc_linear_splitk at few token rows (K split over SMs, chained reduction)
  qkv_rmsnorm   osc_rmsnorm_quantize + osc_linear at the QKV shape (M=--m, default 2048), G=--g
  ffn           osc_quantize + osc_linear, FFN up (K=4096, N=24576, M=4096), G=--g
  w2_osc        osc_quantize + osc_linear, down projection (K=12288, N=4096, M=4096), G=32
  w2_fp8        osc_quantize_fp8 + osc_linear_fp8_fallback on the down projection
  moe_gateup    osc_quantize_grouped + osc_linear_grouped, 128 experts, 2048 -> 1536
  moe_down      the same for the expert down projection, 768 -> 2048

Inputs are the seeded synthetic workloads of inputs.py; tables come from osc_build_table on
the GPU and weights from osc_prepare_weight (or osc_quantize_fp8), so the set-up launches come
first: skip them in the profiler with its launch filter (ncu -k regex:<kernel> -s <skip>).
Each launch round uses the same buffers; the device status word is checked at the end.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from w4a4_outlier_separated_b200 import inputs as I
from w4a4_outlier_separated_b200 import osc


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to("cuda")


def _table(calib, K, G):
    Ld = torch.empty(K // G, dtype=torch.int8, device="cuda")
    osc.osc_build_table(_dev(calib), G, 5.0, 5, Ld)
    return Ld, osc.osc_table_kl(Ld.cpu().numpy())


def _dense(case, G, launches, linear_only=False, M=None, split=False):
    X = case.X if M is None else case.X[:M]
    M, K = X.shape
    N = case.W.shape[0]
    Ld, K_L = _table(case.calib, K, G)
    QW, SW, WL = osc.prepare_weight(_dev(case.W), G, Ld, K_L)
    Xd = _dev(X)
    QX, SX, B = osc.quantize(Xd, G, Ld, K_L)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(16, osc.osc_linear_workspace_bytes(M, N, K, K_L)), dtype=torch.uint8, device="cuda")
    for _ in range(launches):
        if not linear_only:
            osc.osc_quantize(Xd, G, Ld, K_L, QX, SX, B)
        if split:
            osc.osc_linear_splitk(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y, ws)
        else:
            osc.osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y)


def _rmsnorm(case, G, launches):
    M, K = case.X.shape
    N = case.W.shape[0]
    gamma = torch.from_numpy((1.0 + 0.1 * np.random.default_rng(1).standard_normal(K)).astype(np.float32))
    gbits = gamma.to(torch.bfloat16).view(torch.int16).cuda()
    Ld, K_L = _table(case.calib, K, G)
    QW, SW, WL = osc.prepare_weight(_dev(case.W), G, Ld, K_L)
    Xd = _dev(case.X)
    QX, SX, B = osc.alloc_quantize_outputs(M, K, G, K_L, "cuda")
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(launches):
        osc.osc_rmsnorm_quantize(Xd, gbits, 1e-6, G, Ld, K_L, QX, SX, B)
        osc.osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y)


def _fp8(case, launches):
    M, K = case.X.shape
    N = case.W.shape[0]
    QW, SW, _ = osc.alloc_quantize_outputs(N, K, 32, 0, fp8=True)
    osc.osc_quantize_fp8(_dev(case.W), QW, SW)
    Xd = _dev(case.X)
    QX, SX, _ = osc.alloc_quantize_outputs(M, K, 32, 0, fp8=True)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(launches):
        osc.osc_quantize_fp8(Xd, QX, SX)
        osc.osc_linear_fp8_fallback(QX, SX, QW, SW, M, N, K, Y)


def _moe(which, launches):
    case = I.moe_case(which)
    E, K, N, G = case.E, case.K, case.N, 32
    Ld = torch.full((E, K // G), -1, dtype=torch.int8, device="cuda")
    for e in range(E):
        if case.calib[e].shape[0]:
            osc.osc_build_table(_dev(case.calib[e]), G, 5.0, 5, Ld[e])
    Lh = Ld.cpu().numpy()
    kls = np.array([osc.osc_table_kl(Lh[e]) for e in range(E)], np.int32)
    K_L = max(16, int(kls.max()))
    off, poff, mbe = osc.osc_grouped_plan(case.counts)
    Mp = int(poff[-1])
    offd, poffd, mbed, kld = off.cuda(), poff.cuda(), mbe.cuda(), torch.from_numpy(kls).cuda()
    QW = torch.empty((E, N, K // 2), dtype=torch.uint8, device="cuda")
    SW = torch.empty((E, osc.osc_scale_bytes(N, K, G)), dtype=torch.uint8, device="cuda")
    WL = torch.empty((E, N, K_L), dtype=torch.int16, device="cuda")
    for e in range(E):
        osc.osc_prepare_weight(_dev(case.W[e]), G, Ld[e], K_L, QW[e], SW[e], WL[e])
    Xd = _dev(case.X)
    QX = torch.empty((Mp, K // 2), dtype=torch.uint8, device="cuda")
    SX = torch.empty(osc.osc_scale_bytes(Mp, K, G), dtype=torch.uint8, device="cuda")
    B = torch.empty((Mp, K_L), dtype=torch.int16, device="cuda")
    Y = torch.empty((Mp, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(launches):
        osc.osc_quantize_grouped(Xd, E, offd, poffd, mbed, Mp, G, Ld, K_L, QX, SX, B)
        osc.osc_linear_grouped(QX, SX, B, QW, SW, WL, mbed, kld, E, Mp, N, K, G, K_L, Y)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("case", choices=["qkv", "qkv_rmsnorm", "weight_bound", "weight_bound_split", "ffn", "w2_osc",
                                     "w2_fp8", "moe_gateup", "moe_down"])
    ap.add_argument("--launches", type=int, default=4, help="rounds of the workload's kernels")
    ap.add_argument("--m", type=int, default=None, help="token rows (qkv: 2048, weight_bound: 16)")
    ap.add_argument("--g", type=int, default=32, help="group size (qkv, ffn)")
    a = ap.parse_args(argv)
    osc.lib()
    if a.case == "qkv":
        _dense(I.qkv_case(a.m or 2048), a.g, a.launches)
    elif a.case == "qkv_rmsnorm":
        _rmsnorm(I.qkv_case(a.m or 2048), a.g, a.launches)
    elif a.case in ("weight_bound", "weight_bound_split"):
        _dense(I.qkv_case(a.m or 16), 32, a.launches, linear_only=True, split=a.case.endswith("split"))
    elif a.case == "ffn":
        _dense(I.ffn_case(a.g), a.g, a.launches)
    elif a.case == "w2_osc":
        _dense(I.w2_case(), 32, a.launches)
    elif a.case == "w2_fp8":
        _fp8(I.w2_case(), a.launches)
    else:
        _moe(a.case[4:], a.launches)
    torch.cuda.synchronize()
    code, raw = osc.osc_status()
    if code != 0:
        raise SystemExit(f"device status {code} ({raw})")
    print(f"profile_case {a.case}: {a.launches} rounds done")


if __name__ == "__main__":
    main()
