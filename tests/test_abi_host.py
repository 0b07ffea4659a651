"""Host-side checks of the C-ABI library (no GPU needed, no compute launched).

The library must load, export every entry point ``include/*.h`` declares, and reject bad
arguments on the host before anything reaches the device.
"""
import ctypes
import glob
import os
import re
from pathlib import Path

import pytest

from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# These calls pass deliberately invalid arguments (placeholder pointers included) and expect
# the host-side checks to refuse them before any launch.  They are CPU tests: on a machine
# with a CUDA device they are skipped, so that a regression in the checks can never turn a
# placeholder pointer into a device access.
pytestmark = pytest.mark.skipif(__import__("torch").cuda.is_available(),
                                reason="host-only argument checks run where no GPU is present")


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return ssd_i8.library()


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names.update(re.findall(r"^SSD_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, re.M))
    return names


def test_header_declares_the_boundary():
    names = _declared_symbols()
    assert {"ssd_i8_chunk_scan", "ssd_i8_state_update"} <= names
    assert names == set(ssd_i8.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), f"{name} not exported"
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_abi_version_and_status_strings(lib):
    assert lib.ssd_i8_abi_version() >= 1
    for code, name in ssd_i8.STATUS_NAMES.items():
        assert lib.ssd_status_string(code).decode().startswith(name)
    assert lib.ssd_status_string(99).decode() == "SSD_ERR_UNKNOWN"


def test_workspace_size(lib):
    f = lib.ssd_i8_chunk_scan_workspace_size
    n = f(2, 16384, 128, 64, 128, 8, 256)
    assert n > 0 and n % 256 == 0
    assert f(-1, 10, 4, 64, 16, 1, 64) == 0
    assert f(1, 0, 4, 64, 16, 1, 64) < 4096  # no work: status word and flags only
    assert f(2, 16384, 128, 64, 128, 8, 256) <= 9 << 20  # bounded by the CTA count, not L


def _scan_args(**over):
    a = dict(x=256, B=256, C=256, dt=256, A=256, D=256, xs=256, bs=256, cs=256, batch=1, L=8, H=4,
             P=64, N=16, G=1, Q=64, init=None, final=None, y=256, yd=1, ys=1.0, ws=256,
             wsb=1 << 24, stream=None)
    a.update(over)
    return [a[k] for k in ("x", "B", "C", "dt", "A", "D", "xs", "bs", "cs", "batch", "L", "H",
                           "P", "N", "G", "Q", "init", "final", "y", "yd", "ys", "ws", "wsb",
                           "stream")]


@pytest.mark.parametrize("over,status", [
    (dict(H=6, G=4), 1),          # H % G != 0
    (dict(yd=7), 1),              # bad dtype code
    (dict(yd=2, ys=0.0), 1),      # int8 output needs y_scale > 0
    (dict(yd=2 | 32, ys=0.0), 1),  # the same with per-channel B/C scales (flag parsed)
    (dict(yd=64), 1),             # unknown flag bit
    (dict(yd=7 | 32), 1),         # bad dtype code under the per-channel flag
    (dict(A=None), 1),            # null pointer
    (dict(P=32), 2),              # headdim not implemented
    (dict(N=48), 2),              # dstate not implemented
    (dict(Q=100), 2),             # chunk size not implemented
    (dict(batch=1 << 24, H=256), 2),  # 2^32 (sequence, head) units: beyond 32-bit indexing
    (dict(ws=None), 3),           # workspace missing
    (dict(wsb=16), 3),            # workspace too small
    (dict(ws=257), 3),            # workspace misaligned
    (dict(batch=-1), 1),
    (dict(x=264), 1),             # x not 16-byte aligned (TMA source)
    (dict(y=1032), 1),            # y not 16-byte aligned (vector stores)
])
def test_chunk_scan_rejects_bad_arguments_on_host(lib, over, status):
    assert lib.ssd_i8_chunk_scan(*_scan_args(**over)) == status


def test_state_update_rejects_bad_arguments_on_host(lib):
    f = lib.ssd_i8_state_update
    base = [1] * 10 + [1, 4, 64, 16, 1, 1, 1, 1.0, None]
    bad_groups = list(base)
    bad_groups[11], bad_groups[14] = 6, 4
    assert f(*bad_groups) == 1
    bad_n = list(base)
    bad_n[13] = 12
    assert f(*bad_n) == 2
    null_state = list(base)
    null_state[0] = None
    assert f(*null_state) == 1


def test_per_channel_flag_reaches_the_decode_checks(lib):
    f = lib.ssd_i8_state_update
    base = [1] * 10 + [1, 4, 64, 16, 1, 1, 2 | 32, 0.0, None]  # int8 out with per-channel scales
    assert f(*base) == 1  # y_scale 0 refused: the flag combination is understood
    q8 = lib.ssd_i8_state_update_q8
    base = [1] * 11 + [1, 4, 64, 16, 1, 1, 7 | 32, 1.0, None]
    assert q8(*base) == 1  # a bad dtype code under the flag


def test_chunk_cb_rejects_bad_arguments_on_host(lib):
    f = lib.ssd_i8_chunk_cb
    assert f(256, 256, 1, 8, 1, 16, 100, 256, None) == 2
    assert f(None, 256, 1, 8, 1, 16, 64, 256, None) == 1
    assert f(256, 256, -1, 8, 1, 16, 64, 256, None) == 1
    assert f(264, 256, 1, 8, 1, 16, 64, 256, None) == 1  # misaligned C


def test_status_query_rejects_null_workspace(lib):
    assert lib.ssd_i8_chunk_scan_status(None, None) == 1


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 8, 4, 64, dtype=torch.int8)
    B = torch.zeros(1, 8, 1, 16, dtype=torch.int8)
    with pytest.raises(ValueError):
        ssd_i8.ssd_i8_chunk_cb(B, B, 64, cb=torch.zeros(1, 1, 1, 64, 64, dtype=torch.int32))
    with pytest.raises((ValueError, RuntimeError)):
        f = torch.zeros(4)
        ssd_i8.ssd_i8_chunk_scan(x, B, B, torch.zeros(1, 8, 4), f, f, f, torch.zeros(1),
                                 torch.zeros(1), 64, y=torch.zeros(1, 8, 4, 64, dtype=torch.float16),
                                 workspace=torch.zeros(1 << 20, dtype=torch.uint8))


def test_missing_library_fails_loudly():
    """Without libssd_i8.so the binding raises; there is no CPU or library fallback.  (A fresh
    interpreter: the loaded library is cached per process.)"""
    import subprocess
    import sys
    code = ("import quantized_mamba_ssd_b200.ssd_i8 as m\n"
            "m.LIB_PATH = '/nonexistent/libssd_i8.so'\n"
            "try:\n"
            "    m.library()\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n")
    root = Path(__file__).resolve().parent.parent
    out = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    assert "raised:" in out.stdout and "no fallback" in out.stdout
