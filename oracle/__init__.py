"""CPU oracle for the int8 SSD scan -- TEST INFRASTRUCTURE, not part of the product path.

Only ``tests/``, the package's ``smoke()`` check and the benchmark's CPU-baseline leg may
import this package.  It wraps ``ssd_oracle.c`` (plain fp64 C, built with gcc) through
ctypes and shares no code with the CUDA library.

Functions follow the pages' statement of the problem (see ``ssd_oracle.c`` for the
definitions and their sources):

* :func:`scan` -- sequential fp64 recurrence over a prefill, with optional initial state,
  final state and an additive per-step state perturbation (for the error-accumulation check);
  B and C scales per group, or per group and dstate channel.
* :func:`step` -- one decode step on an fp64 state.
* :func:`chunk_cb` -- SSDi8's ChunkBMM matrix CB = Cq Bq^T per chunk and group, int64.
* :func:`requant` -- static symmetric int8 requantization of an output.
* :func:`quantize_state` / :func:`step_q8` -- the int8 cached decode state (one scale per
  (batch, head), max|h| / 127) and one decode step on it: dequantize, fp64 step, requantize.
* :func:`hadamard` -- the orthonormal Walsh-Hadamard transform of the SSD output over headdim.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lock = threading.Lock()
_lib = None

__all__ = ["build", "load", "scan", "step", "chunk_cb", "requant", "quantize_state", "step_q8",
           "hadamard"]


def build(force: bool = False) -> str:
    """Compile ``ssd_oracle.c`` into ``libssd_oracle.so`` next to it (gcc, -O2, pthreads).

    -O2 without -ffast-math keeps IEEE fp64 semantics (no reassociation, no FMA contraction).
    """
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            vp = ctypes.c_void_p
            ci = ctypes.c_int
            lib.ssd_oracle_scan.restype = ci
            lib.ssd_oracle_scan.argtypes = [vp] * 9 + [ci] * 6 + [vp] * 4 + [ci]
            lib.ssd_oracle_scan_pern.restype = ci
            lib.ssd_oracle_scan_pern.argtypes = [vp] * 9 + [ci] * 6 + [vp] * 4 + [ci]
            lib.ssd_oracle_step.restype = ci
            lib.ssd_oracle_step.argtypes = [vp] * 10 + [ci] * 5 + [vp, ci]
            lib.ssd_oracle_chunk_cb.restype = ci
            lib.ssd_oracle_chunk_cb.argtypes = [vp, vp] + [ci] * 5 + [vp]
            lib.ssd_oracle_requant.restype = ci
            lib.ssd_oracle_requant.argtypes = [vp, ctypes.c_int64, ctypes.c_double, vp]
            _lib = lib
    return _lib


def _arr(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _opt(a, dtype):
    if a is None:
        return None, None
    return _arr(a, dtype)


def scan(x, B, C, dt, A, D, x_scale, B_scale, C_scale, *, init_state=None, eps=None,
         want_final_state=True, nthreads: int = 0):
    """fp64 sequential scan.  Shapes: x [b,l,h,p] int8, B/C [b,l,g,n] int8, dt [b,l,h] f32,
    A/D/x_scale [h] f32, B_scale/C_scale [g] f32 -- or both [g, n], one scale per dstate
    channel --, init_state [b,h,p,n] (any float), eps [b,l,h,p,n] (any float).  Returns
    (y f64 [b,l,h,p], final_state f64 or None, threads used)."""
    lib = load()
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    per_n = np.ndim(B_scale) == 2
    if np.shape(B_scale) != ((G, N) if per_n else (G,)) or np.shape(C_scale) != np.shape(B_scale):
        raise ValueError("B_scale and C_scale must both be [g] or both be [g, n]")
    keep = []
    args = []
    for a, t in ((x, np.int8), (B, np.int8), (C, np.int8), (dt, np.float32), (A, np.float32),
                 (D, np.float32), (x_scale, np.float32), (B_scale, np.float32),
                 (C_scale, np.float32)):
        arr, p = _arr(a, t)
        keep.append(arr)
        args.append(p)
    init, pinit = _opt(init_state, np.float64)
    ep, peps = _opt(eps, np.float64)
    y = np.zeros((bsz, L, H, P), dtype=np.float64)
    fs = np.zeros((bsz, H, P, N), dtype=np.float64) if want_final_state else None
    fn = lib.ssd_oracle_scan_pern if per_n else lib.ssd_oracle_scan
    r = fn(*args, bsz, L, H, P, N, G, pinit, peps,
           None if fs is None else fs.ctypes.data_as(ctypes.c_void_p),
           y.ctypes.data_as(ctypes.c_void_p), nthreads)
    if r < 0:
        raise ValueError(f"ssd_oracle_scan failed ({r})")
    del keep, init, ep
    return y, fs, r


def step(state, x, B, C, dt, A, D, x_scale, B_scale, C_scale, *, nthreads: int = 0):
    """One decode step.  state [b,h,p,n] f64 is updated in place (it must be a contiguous
    float64 array); x [b,h,p] int8; B/C [b,g,n] int8; dt [b,h] f32.  Returns y f64 [b,h,p]."""
    lib = load()
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64 and state.flags.c_contiguous):
        raise TypeError("state must be a C-contiguous float64 numpy array")
    bsz, H, P, N = state.shape
    G = B.shape[1]
    keep = []
    args = []
    for a, t in ((x, np.int8), (B, np.int8), (C, np.int8), (dt, np.float32), (A, np.float32),
                 (D, np.float32), (x_scale, np.float32), (B_scale, np.float32),
                 (C_scale, np.float32)):
        arr, p = _arr(a, t)
        keep.append(arr)
        args.append(p)
    y = np.zeros((bsz, H, P), dtype=np.float64)
    r = lib.ssd_oracle_step(state.ctypes.data_as(ctypes.c_void_p), *args, bsz, H, P, N, G,
                            y.ctypes.data_as(ctypes.c_void_p), nthreads)
    if r < 0:
        raise ValueError(f"ssd_oracle_step failed ({r})")
    del keep
    return y


def chunk_cb(C, B, chunk_size: int):
    """ChunkBMM matrices CB[b, c, g, t, s] = sum_n Cq[t,n] Bq[s,n] per chunk, int64."""
    lib = load()
    bsz, L, G, N = C.shape
    nchunks = (L + chunk_size - 1) // chunk_size
    Ca, pc = _arr(C, np.int8)
    Ba, pb = _arr(B, np.int8)
    cb = np.zeros((bsz, nchunks, G, chunk_size, chunk_size), dtype=np.int64)
    r = lib.ssd_oracle_chunk_cb(pc, pb, bsz, L, G, N, chunk_size, cb.ctypes.data_as(ctypes.c_void_p))
    if r < 0:
        raise ValueError(f"ssd_oracle_chunk_cb failed ({r})")
    del Ca, Ba
    return cb


def requant(y, y_scale: float):
    """q = clamp(rne(y / s_y), -127, 127), decided in fp64."""
    lib = load()
    ya, py = _arr(y, np.float64)
    q = np.zeros(ya.shape, dtype=np.int8)
    r = lib.ssd_oracle_requant(py, ya.size, float(y_scale), q.ctypes.data_as(ctypes.c_void_p))
    if r < 0:
        raise ValueError("ssd_oracle_requant failed")
    return q


def quantize_state(state):
    """int8 cached state: per (batch, head) scale = max|h| / 127 over [p, n] and codes
    clamp(rne(h / scale), -127, 127) decided in fp64 (an all-zero state gets scale 0 and codes
    0).  state [b,h,p,n]; returns (codes int8 [b,h,p,n], scales float64 [b,h])."""
    st = np.asarray(state, dtype=np.float64)
    bsz, H = st.shape[:2]
    scales = np.abs(st).reshape(bsz, H, -1).max(axis=2) / 127.0
    codes = np.zeros(st.shape, dtype=np.int8)
    for b in range(bsz):
        for h in range(H):
            if scales[b, h] > 0:
                codes[b, h] = requant(st[b, h], scales[b, h])
    return codes, scales


def step_q8(codes, scales, x, B, C, dt, A, D, x_scale, B_scale, C_scale):
    """One decode step on an int8 cached state: h = scale * code (fp64), the fp64 step of
    :func:`step`, then :func:`quantize_state` of the updated state.  Returns (y, codes, scales)."""
    state = np.ascontiguousarray(np.asarray(codes, dtype=np.float64)
                                 * np.asarray(scales, dtype=np.float64)[:, :, None, None])
    y = step(state, x, B, C, dt, A, D, x_scale, B_scale, C_scale)
    c2, s2 = quantize_state(state)
    return y, c2, s2


def hadamard(y):
    """Orthonormal Walsh-Hadamard transform over the last axis (length a power of two, Sylvester
    order): y' = H y / sqrt(P), H from scipy.linalg.hadamard.  The transform of the SSD output
    ahead of out_proj used with the Table R10 runs of the Quamba2 OpenReview rebuttal."""
    from scipy.linalg import hadamard as _sylvester
    y = np.asarray(y, dtype=np.float64)
    P = y.shape[-1]
    Hm = _sylvester(P).astype(np.float64) / np.sqrt(P)
    return y @ Hm.T
