"""The benchmark's reference arm (the fp64 oracle on the host) prints the contract's line."""
import argparse
import io
import json
from contextlib import redirect_stdout

import bench
from quantized_mamba_ssd_b200 import workloads as W


def test_reference_arm_line():
    case = W.make_prefill(1, 128, 4, 64, 16, 1, 64, seed=3, name="tiny")
    args = argparse.Namespace(gpus=1, steps=2, warmup=1)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_arm(args, case)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["metric"] == bench.METRIC
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_algorithmic_work_of_the_long_prefill():
    case = W.PrefillCase("shape-only", 2, 16384, 128, 64, 128, 8, 256, *([None] * 9))
    # x + B + C + dt + int8 y + final state
    assert bench.prefill_alg_bytes(case, 1, True) == 629145600
    assert abs(bench.prefill_alg_ops(case) - 215.05e9) / 215.05e9 < 1e-3


def test_algorithmic_bytes_of_the_decode_steps():
    d = W.DecodeCase("shape-only", 128, 1, 128, 64, 128, 8, *([None] * 10))
    # fp32 state read and written, x, B, C, dt in, f16 y out: 65 748 B per (batch, head)
    assert bench.decode_alg_bytes(d, 2) == 65748 * 128 * 128
    # int8 codes read and written plus one fp32 scale each way: 16 604 B per (batch, head)
    assert bench.decode_alg_bytes(d, 2, state_bytes=1) == 16604 * 128 * 128


def test_captured_traffic_scales_with_the_work():
    # the captured DRAM bytes, when the kernel source matches the capture, grow with the tokens
    # (prefill) and the (batch, head) items (decode); a changed source reports none
    t = bench.captured_traffic(32768)
    if t is not None:
        assert abs(bench.captured_traffic(16384) * 2 - t) < 1e-6 * t
    for src in ("state_update.cu", "state_update_q8.cu"):
        v = bench.captured_decode_traffic(src, 128 * 128)
        if v is not None:
            assert abs(bench.captured_decode_traffic(src, 64 * 128) * 2 - v) < 1e-6 * v
