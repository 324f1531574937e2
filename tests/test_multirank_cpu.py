"""Multi-rank host logic of bench.py on the CPU: two `gloo` ranks (world size 2) take the
element-wise max of their timings, every rank sees the same result, the whole-job throughput is
the weak-scaling sum, and under a launcher only rank 0 runs the reference arm."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["OSC_ROOT"])
import torch.distributed as dist
import bench
ws, rank, local = bench.dist_env()
dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
mine = [1.0 + rank, 10.0 - rank, 5.0 + 0.5 * rank]
out = bench.max_over_ranks(mine, "cpu")
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "local": local, "ws": ws, "out": out}))
"""


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(ws: int, code: str, extra_env=None):
    port = _free_port()
    procs = []
    for r in range(ws):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r), LOCAL_RANK=str(r),
                   WORLD_SIZE=str(ws), OSC_ROOT=ROOT, CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("a rank did not finish")
        assert p.returncode == 0, e[-2000:]
        outs.append(o)
    return outs


def test_max_over_ranks_gloo_world2():
    outs = _launch(2, WORKER)
    res = sorted((json.loads(o.strip().splitlines()[-1]) for o in outs), key=lambda d: d["rank"])
    assert [d["rank"] for d in res] == [0, 1] and all(d["ws"] == 2 for d in res)
    assert [d["local"] for d in res] == [0, 1]
    for d in res:
        assert d["out"] == [2.0, 10.0, 5.5]          # element-wise max, identical on every rank


def test_single_process_passthrough_and_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5], "cpu") == [3.0, 4.5]
    flops = 2.0 * 2048 * 6144 * 4096
    one = bench.weak_scaling_tflops(1, flops, 0.040)
    assert abs(one - flops / 40e-6 / 1e12) < 1e-9
    # N ranks, each with its own batch in the same (max) time: N times the work per second
    assert abs(bench.weak_scaling_tflops(4, flops, 0.040) - 4 * one) < 1e-9


REF_WORKER = r"""
import os, sys
sys.path.insert(0, os.environ["OSC_ROOT"])
import bench
args = type("A", (), {"steps": 1, "warmup": 0, "gpus": 2})()
res = bench.run_reference(args)
print("NONE" if res is None else "LINE")
"""


def test_reference_arm_runs_on_rank0_only():
    """Under a launcher the oracle arm runs on rank 0; other ranks return without work."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", OSC_ROOT=ROOT, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "-c", REF_WORKER], env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip().splitlines()[-1] == "NONE"


def test_algorithmic_bytes_and_row_record():
    """The quantize byte counts behind the HBM fractions: X read (bf16), codes, one E8M0 byte
    per 32 (or 16) elements, and B, written out for the QKV and W2 shapes."""
    import bench
    assert bench.quant_bytes(2048, 4096, 32, 96) == 2048 * 4096 * 2 + 2048 * 2048 + 2048 * 128 + 2048 * 96 * 2
    assert bench.quant_bytes(2048, 4096, 32, 96) == 21_626_880                  # ~21.6 MB per QKV launch
    assert bench.quant_bytes(2048, 4096, 16, 96) - bench.quant_bytes(2048, 4096, 32, 96) == 2048 * 128
    assert bench.quant_bytes(4096, 12288, 32, 0, fp8=True) == 152_567_808       # MXFP8 W2: ~3.03 B/elem
    peaks = {"hbm_gbs": 6450.0, "bf16_tflops": 1672.7}
    qkv_lbytes = 4_194_304 + 262_144 + 393_216 + 12_582_912 + 786_432 + 1_179_648 + 25_165_824
    r = bench._row_record("x", 2048, 4096, 6144, 32, 96, 0.0373, 0.0073, 0.0284, 2.0 * 2048 * 6144 * 4096,
                          21_626_880, 4 * 1672.7, peaks, 8, qkv_lbytes)
    assert abs(r["TFLOPs"] - 2764.2) < 1.0 and abs(r["linear_frac"] - 0.5425) < 1e-3
    assert abs(r["quantize_GBps"] - 2962.6) < 0.5 and abs(r["quantize_hbm_frac"] - 0.459) < 1e-3
    assert r["linear_bound"] == "tensor" and r["linear_roofline_frac"] == r["linear_frac"]
    # MoE gate+up: 404 MB to move at 6.45 TB/s (62.6 us) outlasts 253 GFLOP at 6.69 PFLOP/s (37.8 us)
    moe = bench._row_record("m", 32768, 2048, 1536, 32, 48, 0.174, 0.0759, 0.0998, 2.0 * 32768 * 1536 * 2048,
                            1, 4 * 1672.7, peaks, 1, 404_000_000, mma_flops=2.0 * 40192 * 1536 * 2048)
    assert moe["linear_bound"] == "hbm" and abs(moe["linear_roofline_frac"] - 0.6276) < 1e-3
    import torch
    assert bench.tensor_bytes(torch.empty(3, 5, dtype=torch.int16), None, torch.empty(7, dtype=torch.uint8)) == 37


def test_clock_sampler_samples_while_the_timed_work_runs():
    """Samples are taken from the host until the end event of the timed region completes, at
    least once; throttle reasons are collected by name."""
    import bench

    class NV:
        NVML_CLOCK_SM = 0

        @staticmethod
        def nvmlDeviceGetClockInfo(h, kind):
            return 1965

        @staticmethod
        def nvmlDeviceGetCurrentClocksThrottleReasons(h):
            return 0x4

    class Event:
        def __init__(self, done_after):
            self.calls, self.done_after = 0, done_after

        def query(self):
            self.calls += 1
            return self.calls >= self.done_after

    c = bench.ClockSampler(0)
    c.nv, c.h, c.samples, c.reasons = NV, None, [], set()
    c.sample_while(Event(3), 0.0)
    assert len(c.samples) == 3
    assert c.summary() == {"sm_mhz": 1965.0, "sm_max_mhz": c.max_mhz, "reasons": ["sw_power_cap"], "samples": 3}
    c.samples = []
    c.sample_while(Event(1), 0.0)                    # work already done: still one sample
    assert len(c.samples) == 1


def test_line_ends_with_the_kernel_figures():
    """The printed line keeps every required key and ends with the compact per-row summary,
    the headline kernels' figures and the weight-bound lines, so they fit a 1.5 kB log tail
    even after a long per-row section."""
    import json
    import bench
    row = {"ms_per_step": 0.0373, "linear_roofline_frac": 0.54, "quantize_hbm_frac": 0.46, "detail": "x" * 400}
    res = {"metric": "m", "value": 1.0, "kernels": {"osc_quantize_GBps": 2950.0, "osc_quantize_hbm_frac": 0.46},
           "weight_bound": {"unit": "GB/s", "peak": 6450.0, "what": "w",
                            "lines": [{"M": m, "us": 9.9, "GBps": 1490.0, "frac": 0.23, "us_one_part": 12.0,
                                       "frac_one_part": 0.19, "step_two_calls_us": 11.5,
                                       "step_one_call_us": 11.0} for m in (1, 16, 128)]},
           "roofline": {"frac": 0.5},
           "scope_rows": {f"row{i}": dict(row) for i in range(12)} | {"table2_osc_speedup_over_w8a8": {"G32": 1.35}},
           "cpu_baseline": {"value": 0.0035}}
    out = bench.tail_order(res)
    assert list(out)[-3:] == ["rows_brief", "kernels", "weight_bound"]
    assert out["rows_brief"]["row3"] == [37.3, 0.54, 0.46] and out["rows_brief"]["table2"] == {"G32": 1.35}
    line = json.dumps(out)
    tail = line[-1500:]
    assert '"osc_quantize_GBps": 2950.0' in tail and "[16, 9.9, 1490.0, 0.23, 12.0, 0.19, 11.5, 11.0]" in tail and '"row11"' in tail
    assert {"metric", "value", "roofline", "scope_rows", "cpu_baseline"} <= set(out)
