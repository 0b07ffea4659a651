"""The allocation-free chunk scan, for callers that cannot allocate device memory.

Such callers (an engine whose memory pool is reserved in full before it serves, code that must
not risk the device synchronisation of a cudaMalloc, a plug-in whose host owns allocation) call
``ssd_i8_chunk_scan_noalloc``, which takes its scratch from the library's built-in 4 MiB device
array instead of a workspace.  These tests call it through the C ABI and compare it with the
workspace-taking ``ssd_i8_chunk_scan`` on the same inputs, with the parity tolerances, on two
calls in a row (so that the second call runs on scratch the first one left behind).

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

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


def _inputs(case):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    return [t(a) for a in (case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                           case.B_scale, case.C_scale)], \
        (None if case.init_state is None else t(case.init_state))


def _both(case, y_dtype):
    ins, init = _inputs(case)
    shape_s = (case.batch, case.nheads, case.headdim, case.dstate)
    fs_ref = torch.empty(shape_s, dtype=torch.float32, device=DEV)
    y_ref = ssd_i8.ssd_i8_chunk_scan(*ins, case.chunk_size, init_state=init, final_state=fs_ref,
                                     y_dtype=y_dtype)
    fs = torch.full(shape_s, float("nan"), dtype=torch.float32, device=DEV)
    y = torch.full_like(y_ref, 0)
    ssd_i8.ssd_i8_chunk_scan_noalloc(*ins, case.chunk_size, init_state=init, final_state=fs,
                                     y=y, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return (y.float().cpu().numpy(), fs.cpu().numpy(), y_ref.float().cpu().numpy(),
            fs_ref.cpu().numpy())


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    first = W.make_prefill(2, 700, 8, 64, 128, 2, 128, law="laplace_outliers_all", seed=41,
                           with_init_state=True)
    second = W.make_prefill(1, 517, 4, 64, 128, 4, 256, law="laplace_spread", seed=42,
                            with_init_state=True)
    for case, out in ((first, "f32"), (second, "f16")):
        need = ssd_i8.ssd_i8_chunk_scan_workspace_size(case.batch, case.seqlen, case.nheads,
                                                       case.headdim, case.dstate, case.ngroups,
                                                       case.chunk_size)
        assert 0 < need <= ssd_i8.NOALLOC_SCRATCH_BYTES
        y, fs, y_ref, fs_ref = _both(case, out)
        check_close(y, y_ref, "noalloc y")
        check_close(fs, fs_ref, "noalloc final_state")


def test_noalloc_refuses_problems_beyond_its_scratch():
    # more work items than the scratch has state slots for
    case = W.make_prefill(4, 2048, 64, 64, 128, 1, 256, seed=43)
    need = ssd_i8.ssd_i8_chunk_scan_workspace_size(4, 2048, 64, 64, 128, 1, 256)
    assert need > ssd_i8.NOALLOC_SCRATCH_BYTES
    ins, _ = _inputs(case)
    y = torch.zeros((4, 2048, 64, 64), dtype=torch.float16, device=DEV)
    with pytest.raises(ssd_i8.SSDError) as ei:
        ssd_i8.ssd_i8_chunk_scan_noalloc(*ins, 256, y=y)
    assert ei.value.status == 3  # SSD_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not y.any()  # refused before anything ran


def test_noalloc_limit_falls_at_127_blocks_of_128_tokens():
    # the built-in scratch holds the hand-off slots of 127 work items of 128 tokens, whatever
    # the chunk size: one sequence of 127 blocks (every CTA but the first waits for a hand-off)
    # runs and matches the workspace path; one more block is refused
    case = W.make_prefill(1, 127 * 128, 1, 64, 128, 1, 256, law="laplace_outliers_all", seed=44,
                          with_init_state=True)
    assert ssd_i8.ssd_i8_chunk_scan_workspace_size(1, 127 * 128, 1, 64, 128, 1, 64) <= \
        ssd_i8.NOALLOC_SCRATCH_BYTES
    y, fs, y_ref, fs_ref = _both(case, "f32")
    check_close(y, y_ref, "noalloc y, 127 blocks")
    check_close(fs, fs_ref, "noalloc final_state, 127 blocks")
    big = W.make_prefill(1, 127 * 128 + 1, 1, 64, 128, 1, 256, seed=45)
    assert ssd_i8.ssd_i8_chunk_scan_workspace_size(1, 127 * 128 + 1, 1, 64, 128, 1, 256) > \
        ssd_i8.NOALLOC_SCRATCH_BYTES
    ins, _ = _inputs(big)
    y = torch.zeros((1, 127 * 128 + 1, 1, 64), dtype=torch.float32, device=DEV)
    with pytest.raises(ssd_i8.SSDError) as ei:
        ssd_i8.ssd_i8_chunk_scan_noalloc(*ins, 256, y=y, y_dtype="f32")
    assert ei.value.status == 3  # SSD_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not y.any()


def test_noalloc_status_reports_a_device_side_timeout():
    # a caller without a workspace still learns of a bounded wait that gave up: the hook makes
    # CTA 0 skip its hand-off for one launch (waits bounded by 2^24 cycles), the allocation-free
    # status query reports the timeout, and the next clean call is correct and reports none
    case = W.make_prefill(1, 100 * 128, 1, 64, 128, 1, 128, law="laplace_outliers_all", seed=46)
    ins, _ = _inputs(case)
    ssd_i8.ssd_i8_chunk_scan_noalloc_status()  # nothing failed so far
    y = torch.empty((1, case.seqlen, 1, 64), dtype=torch.float32, device=DEV)
    ssd_i8.ssd_i8_debug_inject(0, 1 << 24)
    ssd_i8.ssd_i8_chunk_scan_noalloc(*ins, 128, y=y, y_dtype="f32")
    with pytest.raises(ssd_i8.SSDError) as ei:
        ssd_i8.ssd_i8_chunk_scan_noalloc_status()
    assert ei.value.status == 5  # SSD_ERR_TIMEOUT
    y, fs, y_ref, fs_ref = _both(case, "f32")
    ssd_i8.ssd_i8_chunk_scan_noalloc_status()
    check_close(y, y_ref, "noalloc y after a reported timeout")
    check_close(fs, fs_ref, "noalloc final_state after a reported timeout")
