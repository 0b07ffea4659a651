"""Shared helpers of the parity tests: tolerance checks and oracle sampling.

Tolerances are the ones the target states for the int8 SSD scan:
  y (and the final state): max-abs error <= 2e-3 * max|ref| and relative L2 <= 1e-3;
  int8 requantized y: within +-1 LSB on >= 99.99 % of the elements;
  ChunkBMM int32 tiles: bit-exact.
"""
from __future__ import annotations

import json
import os

import numpy as np

MAXABS_REL = 2e-3
REL_L2 = 1e-3
I8_LSB_FRACTION = 0.9999


def _log_margin(record: dict) -> None:
    """With SSD_PARITY_LOG set to a file path, append the check's achieved error as a fraction
    of its tolerance (one JSON line per check, tagged with the running test)."""
    path = os.environ.get("SSD_PARITY_LOG")
    if not path:
        return
    record["test"] = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    with open(path, "a") as f:
        f.write(json.dumps(record) + "\n")


def check_close(got, ref, what: str = "y"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} != {ref.shape}"
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    maxabs = err.max() if err.size else 0.0
    nrm = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / nrm if nrm > 0 else np.linalg.norm(got - ref)
    _log_margin({"what": what, "maxabs_of_tol": float(maxabs / (MAXABS_REL * scale)) if scale > 0
                 else 0.0, "relL2_of_tol": float(rel / REL_L2)})
    assert maxabs <= MAXABS_REL * scale + 1e-30, \
        f"{what}: max-abs err {maxabs:.3e} > {MAXABS_REL} * max|ref| ({scale:.3e})"
    assert rel <= REL_L2, f"{what}: rel-L2 err {rel:.3e} > {REL_L2}"
    return maxabs / scale if scale > 0 else 0.0, rel


def check_i8(got, ref_q):
    got = np.asarray(got).astype(np.int32)
    ref_q = np.asarray(ref_q).astype(np.int32)
    assert got.shape == ref_q.shape
    assert got.min() >= -127 and got.max() <= 127, "int8 output outside the symmetric range"
    d = np.abs(got - ref_q)
    within = (d <= 1).mean() if d.size else 1.0
    _log_margin({"what": "int8", "differ_fraction": float((d != 0).mean()) if d.size else 0.0,
                 "max_lsb": int(d.max()) if d.size else 0})
    assert within >= I8_LSB_FRACTION, f"only {within:.6f} of int8 outputs within +-1 LSB"
    return within, int(d.max()) if d.size else 0


def head_subset(case, heads, batches=None, seqlen=None):
    """Oracle inputs restricted to some (batch, head) pairs, with B/C re-indexed so that head
    i of the subset reads its own copy of its original group."""
    H, G = case.nheads, case.ngroups
    heads = np.asarray(heads)
    groups = heads // (H // G)
    bsel = slice(None) if batches is None else np.asarray(batches)
    L = case.seqlen if seqlen is None else seqlen
    x = case.x[bsel][:, :L][:, :, heads]
    B = case.B[bsel][:, :L][:, :, groups]
    C = case.C[bsel][:, :L][:, :, groups]
    dt = case.dt[bsel][:, :L][:, :, heads]
    init = None if case.init_state is None else case.init_state[bsel][:, heads]
    return dict(x=x, B=B, C=C, dt=dt, A=case.A[heads], D=case.D[heads],
                x_scale=case.x_scale[heads], B_scale=case.B_scale[groups],
                C_scale=case.C_scale[groups], init_state=init)
