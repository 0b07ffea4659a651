"""Failure detection without a GPU fault: a CTA that never publishes its state hand-off.

The fault is injected from the host (ssd_i8_debug_inject): for one launch, CTA 0 skips its
hand-off and every device-side wait is bounded by a few milliseconds.  The waiting CTA gives
up, the launch still ends, ssd_i8_chunk_scan_status reports SSD_ERR_TIMEOUT, and the next call
on the same context and workspace runs normally and matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8
from quantized_mamba_ssd_b200 import workloads as W
from parity_util import check_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    qbuild.build()
    ssd_i8.library()


def test_dropped_handoff_is_reported_and_the_context_survives():
    # one sequence of 300 blocks of 128 tokens and one head: every CTA range splits it, so
    # every CTA but the first waits for its predecessor's hand-off
    case = W.make_prefill(1, 128 * 300, 1, 64, 128, 1, 128, law="laplace_outliers_all", seed=51)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    ins = [t(a) for a in (case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                          case.B_scale, case.C_scale)]
    ws = torch.empty(ssd_i8.ssd_i8_chunk_scan_workspace_size(1, case.seqlen, 1, 64, 128, 1, 128),
                     dtype=torch.uint8, device=DEV)
    ssd_i8.ssd_i8_debug_inject(0, 1 << 24)
    ssd_i8.ssd_i8_chunk_scan(*ins, 128, workspace=ws, y_dtype="f32")
    with pytest.raises(ssd_i8.SSDError) as ei:
        ssd_i8.ssd_i8_chunk_scan_status(ws)
    assert ei.value.status == 5  # SSD_ERR_TIMEOUT
    # same context, same workspace: a clean call is correct and reports no failure
    fs = torch.empty((1, 1, 64, 128), dtype=torch.float32, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan(*ins, 128, workspace=ws, final_state=fs, y_dtype="f32")
    ssd_i8.ssd_i8_chunk_scan_status(ws)
    yr, fr, _ = oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                            case.B_scale, case.C_scale)
    check_close(y.cpu().numpy(), yr, "y after recovery")
    check_close(fs.cpu().numpy(), fr, "final_state after recovery")
