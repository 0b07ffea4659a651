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
