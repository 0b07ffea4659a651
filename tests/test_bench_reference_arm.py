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


def test_algorithmic_bytes_of_the_smaller_prefills():
    # x + B + C + dt + f16 y (SURVEY's roofline table: 104.9 MB and 522.2 MB), and with the
    # final states the legs write
    c1 = W.PrefillCase("shape-only", 4, 2048, 64, 64, 128, 1, 256, *([None] * 9))
    c2 = W.PrefillCase("shape-only", 8, 4096, 80, 64, 128, 1, 256, *([None] * 9))
    assert bench.prefill_alg_bytes(c1, 2, False) == 104857600
    assert bench.prefill_alg_bytes(c2, 2, False) == 522190848
    assert bench.prefill_alg_bytes(c1, 2, True) == 104857600 + 4 * 4 * 64 * 64 * 128
    assert bench.prefill_alg_bytes(c2, 2, True) == 522190848 + 4 * 8 * 80 * 64 * 128


def test_device_status_field_reports_ok_and_stops_on_a_timeout():
    # every timed chunk-scan leg reports its device status; a leg whose bounded wait gave up
    # ended early, so the run exits non-zero instead of printing its time
    assert bench.device_status_field({"main": None, "varlen_strided": None}) == "ok"
    import pytest
    with pytest.raises(SystemExit) as ei:
        bench.device_status_field({"main": None, "hadamard_out": 5})
    assert ei.value.code != 0


def test_bench_line_carries_the_device_status():
    # the field is part of the printed line, computed from the statuses of every timed leg
    src = open(bench.__file__).read()
    assert '"device_status": device_status_field(statuses)' in src
    for leg in ("main", "hadamard_out", "e2e_serial", "e2e_pipelined", "per_tensor_percentile",
                "varlen_strided"):
        assert f'statuses["{leg}"]' in src or f'"{leg}": scan_status' in src
