"""Python binding of ``libssd_i8.so``: argument marshalling only.

Each function takes torch CUDA tensors, checks dtype / shape / contiguity, and passes their
device pointers to the C entry point of the same name (declared in ``include/ssd_i8.h``) on
the current torch stream.  All arithmetic runs in the library's CUDA kernels; if the library
is missing or fails to load, the calls raise -- there is no fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd_i8.so")

SSD_OK = 0
STATUS_NAMES = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED",
                3: "SSD_ERR_WORKSPACE", 4: "SSD_ERR_CUDA", 5: "SSD_ERR_TIMEOUT"}
OUT_DTYPES = {"f32": (0, torch.float32), "f16": (1, torch.float16), "i8": (2, torch.int8)}
OUT_HADAMARD = 16  # flag: y' = H y / 8 over headdim before the conversion (include/ssd_i8.h)
SCALES_PER_N = 32  # flag: B_scale / C_scale are [ngroups, dstate] (include/ssd_i8.h)

# names of every extern "C" symbol include/ssd_i8.h declares
EXPORTED = ("ssd_i8_abi_version", "ssd_status_string", "ssd_i8_chunk_scan_workspace_size",
            "ssd_i8_chunk_scan", "ssd_i8_state_update", "ssd_i8_chunk_cb",
            "ssd_i8_chunk_scan_noalloc", "ssd_i8_chunk_scan_status", "ssd_i8_debug_inject",
            "ssd_i8_chunk_scan_varlen_workspace_size", "ssd_i8_chunk_scan_varlen",
            "ssd_i8_state_quantize", "ssd_i8_state_update_q8", "ssd_i8_chunk_scan_noalloc_status")

# built-in scratch of ssd_i8_chunk_scan_noalloc (bytes); larger problems are refused
NOALLOC_SCRATCH_BYTES = 4 << 20

# kernels one ssd_i8_chunk_scan call launches (the fused persistent scan); the benchmark
# reports launches from it and a GPU test checks it against a profiler count
KERNELS_PER_CHUNK_SCAN = 1
KERNELS_PER_STATE_UPDATE = 1

_lock = threading.Lock()
_lib: Optional[ctypes.CDLL] = None
_tls = threading.local()  # device of the call being marshalled


class SSDError(RuntimeError):
    """A non-OK status returned by the library."""

    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg}")
        self.status = status


def library() -> ctypes.CDLL:
    """Load ``libssd_i8.so`` (built by ``quantized_mamba_ssd_b200.build``) and declare types."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m quantized_mamba_ssd_b200.build` (no fallback exists)")
        lib = ctypes.CDLL(LIB_PATH)
        vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.ssd_i8_abi_version.restype = ci
        lib.ssd_i8_abi_version.argtypes = []
        lib.ssd_status_string.restype = ctypes.c_char_p
        lib.ssd_status_string.argtypes = [ci]
        lib.ssd_i8_chunk_scan_workspace_size.restype = sz
        lib.ssd_i8_chunk_scan_workspace_size.argtypes = [ci] * 7
        lib.ssd_i8_chunk_scan.restype = ci
        lib.ssd_i8_chunk_scan.argtypes = [vp] * 9 + [ci] * 7 + [vp, vp, vp, ci, cf, vp, sz, vp]
        lib.ssd_i8_state_update.restype = ci
        lib.ssd_i8_state_update.argtypes = [vp] * 10 + [ci] * 5 + [vp, ci, cf, vp]
        lib.ssd_i8_chunk_cb.restype = ci
        lib.ssd_i8_chunk_cb.argtypes = [vp, vp] + [ci] * 5 + [vp, vp]
        lib.ssd_i8_debug_inject.restype = ci
        lib.ssd_i8_debug_inject.argtypes = [ci, ctypes.c_longlong]
        lib.ssd_i8_chunk_scan_status.restype = ci
        lib.ssd_i8_chunk_scan_status.argtypes = [vp, vp]
        ll = ctypes.c_longlong
        lib.ssd_i8_chunk_scan_varlen_workspace_size.restype = sz
        lib.ssd_i8_chunk_scan_varlen_workspace_size.argtypes = [ci]
        lib.ssd_i8_chunk_scan_varlen.restype = ci
        lib.ssd_i8_chunk_scan_varlen.argtypes = ([vp, ll, vp, vp, ll, vp, ll] + [vp] * 5 +
                                                 [vp, ci, ll] + [ci] * 5 +
                                                 [vp, vp, vp, ci, cf, vp, sz, vp])
        lib.ssd_i8_state_quantize.restype = ci
        lib.ssd_i8_state_quantize.argtypes = [vp, vp, vp] + [ci] * 4 + [vp]
        lib.ssd_i8_state_update_q8.restype = ci
        lib.ssd_i8_state_update_q8.argtypes = [vp] * 11 + [ci] * 5 + [vp, ci, cf, vp]
        lib.ssd_i8_chunk_scan_noalloc.restype = ci
        lib.ssd_i8_chunk_scan_noalloc.argtypes = [vp] * 9 + [ci] * 7 + [vp, vp, vp, ci, cf, vp]
        lib.ssd_i8_chunk_scan_noalloc_status.restype = ci
        lib.ssd_i8_chunk_scan_noalloc_status.argtypes = [vp]
        _lib = lib
        return lib


def _check(fn: str, status: int) -> None:
    if status != SSD_OK:
        msg = library().ssd_status_string(status).decode()
        raise SSDError(fn, status, msg)


@contextlib.contextmanager
def _on_device_of(t: torch.Tensor):
    """Run one library call with ``t``'s GPU as the current device: the library launches on the
    current device, and every tensor of the call must live on that one."""
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError("the library's tensors must be CUDA tensors")
    prev = getattr(_tls, "device", None)
    _tls.device = t.device
    try:
        with torch.cuda.device(t.device):
            yield
    finally:
        _tls.device = prev


def _device_call(fn):
    """Decorator: the wrapped call marshals and launches on the GPU of its first tensor."""
    import functools

    @functools.wraps(fn)
    def wrapper(first, *args, **kwargs):
        with _on_device_of(first):
            return fn(first, *args, **kwargs)
    return wrapper


def _ptr(t: Optional[torch.Tensor], name: str, dtype: torch.dtype, shape=None) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    dev = getattr(_tls, "device", None)
    if dev is not None and t.device != dev:
        raise ValueError(f"{name} is on {t.device}, the call's other tensors on {dev}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr() if t.numel() else None


def _bc_scales(B_scale: torch.Tensor, C_scale: torch.Tensor, G: int, N: int) -> tuple:
    """Pointers of the B and C scales, [G] per group or [G, N] per group and dstate channel,
    and the y_dtype flag that says which."""
    per_n = isinstance(B_scale, torch.Tensor) and B_scale.dim() == 2
    shape = (G, N) if per_n else (G,)
    return (_ptr(B_scale, "B_scale", torch.float32, shape),
            _ptr(C_scale, "C_scale", torch.float32, shape),
            SCALES_PER_N if per_n else 0)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def ssd_i8_chunk_scan_workspace_size(batch: int, seqlen: int, nheads: int, headdim: int,
                                     dstate: int, ngroups: int, chunk_size: int) -> int:
    return int(library().ssd_i8_chunk_scan_workspace_size(batch, seqlen, nheads, headdim, dstate,
                                                          ngroups, chunk_size))


@_device_call
def ssd_i8_chunk_scan(x: torch.Tensor, B: torch.Tensor, C: torch.Tensor, dt: torch.Tensor,
                      A: torch.Tensor, D: torch.Tensor, x_scale: torch.Tensor,
                      B_scale: torch.Tensor, C_scale: torch.Tensor, chunk_size: int, *,
                      init_state: Optional[torch.Tensor] = None,
                      final_state: Optional[torch.Tensor] = None,
                      y: Optional[torch.Tensor] = None, y_dtype: str = "f16",
                      y_scale: float = 1.0, workspace: Optional[torch.Tensor] = None,
                      stream=None, hadamard: bool = False) -> torch.Tensor:
    """Chunked int8 SSD scan (see ``ssd_i8_chunk_scan`` in include/ssd_i8.h).  ``hadamard``
    applies the output transform y' = H y / 8 over headdim (``SSD_OUT_HADAMARD``).

    x int8 [b,l,h,p]; B, C int8 [b,l,g,n]; dt f32 [b,l,h]; A, D, x_scale f32 [h];
    B_scale, C_scale f32 [g] (or [g, n]: per dstate channel, ``SSD_SCALES_PER_N``); optional
    init_state / final_state f32 [b,h,p,n]; returns y
    [b,l,h,p] of ``y_dtype`` ("f32", "f16" or "i8"; "i8" uses ``y_scale``).  ``workspace`` is
    a uint8 CUDA tensor of at least ``ssd_i8_chunk_scan_workspace_size`` bytes; one is
    allocated through torch when omitted.
    """
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,l,h,p] and B/C [b,l,g,n]")
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    code, tdt = OUT_DTYPES[y_dtype]
    if y is None:
        y = torch.empty((bsz, L, H, P), dtype=tdt, device=x.device)
    need = ssd_i8_chunk_scan_workspace_size(bsz, L, H, P, N, G, chunk_size)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    pb, pc, flag = _bc_scales(B_scale, C_scale, G, N)
    args = [
        _ptr(x, "x", torch.int8, (bsz, L, H, P)),
        _ptr(B, "B", torch.int8, (bsz, L, G, N)),
        _ptr(C, "C", torch.int8, (bsz, L, G, N)),
        _ptr(dt, "dt", torch.float32, (bsz, L, H)),
        _ptr(A, "A", torch.float32, (H,)),
        _ptr(D, "D", torch.float32, (H,)),
        _ptr(x_scale, "x_scale", torch.float32, (H,)),
        pb, pc,
        bsz, L, H, P, N, G, int(chunk_size),
        _ptr(init_state, "init_state", torch.float32, (bsz, H, P, N)),
        _ptr(final_state, "final_state", torch.float32, (bsz, H, P, N)),
        _ptr(y, "y", tdt, (bsz, L, H, P)),
        code | (OUT_HADAMARD if hadamard else 0) | flag, float(y_scale),
        _ptr(workspace, "workspace", torch.uint8),
        workspace.numel(),
        _stream(stream),
    ]
    _check("ssd_i8_chunk_scan", library().ssd_i8_chunk_scan(*args))
    return y


def _rows_ptr(t: torch.Tensor, name: str, dtype: torch.dtype, inner_shape) -> tuple:
    """Pointer and token stride (elements) of a [T, *inner_shape] view whose inner dims are
    contiguous (a column slice of a wider row-major buffer is accepted)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape[1:]) != tuple(inner_shape):
        raise ValueError(f"{name} must have shape [T, {', '.join(map(str, inner_shape))}], "
                         f"got {tuple(t.shape)}")
    inner = 1
    for d in range(t.dim() - 1, 0, -1):
        if t.shape[d] > 1 and t.stride(d) != inner:
            raise ValueError(f"{name}: the dims after the token dim must be contiguous")
        inner *= t.shape[d]
    return (t.data_ptr() if t.numel() else None), (t.stride(0) if t.shape[0] > 1 else inner)


def ssd_i8_chunk_scan_varlen_workspace_size(nseq: int) -> int:
    return int(library().ssd_i8_chunk_scan_varlen_workspace_size(int(nseq)))


@_device_call
def ssd_i8_chunk_scan_varlen(x: torch.Tensor, B: torch.Tensor, C: torch.Tensor, dt: torch.Tensor,
                             A: torch.Tensor, D: torch.Tensor, x_scale: torch.Tensor,
                             B_scale: torch.Tensor, C_scale: torch.Tensor, cu_seqlens,
                             chunk_size: int, *, init_state: Optional[torch.Tensor] = None,
                             final_state: Optional[torch.Tensor] = None,
                             y: Optional[torch.Tensor] = None, y_dtype: str = "f16",
                             y_scale: float = 1.0, workspace: Optional[torch.Tensor] = None,
                             stream=None, hadamard: bool = False) -> torch.Tensor:
    """Chunked int8 SSD scan over packed variable-length sequences (see
    ``ssd_i8_chunk_scan_varlen`` in include/ssd_i8.h).

    x int8 [T,h,p], B, C int8 [T,g,n], dt f32 [T,h]: token-major views whose inner dims are
    contiguous (column slices of a projection output are fine; B and C share a token stride);
    ``cu_seqlens``: host sequence of nseq + 1 token offsets; init_state / final_state f32
    [nseq,h,p,n]; returns y [T,h,p] of ``y_dtype``.
    """
    if x.dim() != 3 or B.dim() != 3 or C.dim() != 3 or dt.dim() != 2:
        raise ValueError("x must be [T,h,p], B/C [T,g,n] and dt [T,h]")
    T, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    nseq = len(cu) - 1
    if nseq < 0:
        raise ValueError("cu_seqlens needs at least one entry")
    code, tdt = OUT_DTYPES[y_dtype]
    if y is None:
        y = torch.empty((T, H, P), dtype=tdt, device=x.device)
    xp, xs = _rows_ptr(x, "x", torch.int8, (H, P))
    bp, bs = _rows_ptr(B, "B", torch.int8, (G, N))
    cp, cs = _rows_ptr(C, "C", torch.int8, (G, N))
    dp, ds = _rows_ptr(dt, "dt", torch.float32, (H,))
    if bs != cs:
        raise ValueError("B and C must have the same token stride")
    if B.shape[0] != T or C.shape[0] != T or dt.shape[0] != T:
        raise ValueError("x, B, C and dt must have the same number of tokens")
    need = ssd_i8_chunk_scan_varlen_workspace_size(nseq)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    cu_arr = (ctypes.c_int32 * len(cu))(*cu)
    pbs, pcs, flag = _bc_scales(B_scale, C_scale, G, N)
    args = [
        xp, xs, bp, cp, bs, dp, ds,
        _ptr(A, "A", torch.float32, (H,)),
        _ptr(D, "D", torch.float32, (H,)),
        _ptr(x_scale, "x_scale", torch.float32, (H,)),
        pbs, pcs,
        ctypes.cast(cu_arr, ctypes.c_void_p), nseq, T, H, P, N, G, int(chunk_size),
        _ptr(init_state, "init_state", torch.float32, (nseq, H, P, N)),
        _ptr(final_state, "final_state", torch.float32, (nseq, H, P, N)),
        _ptr(y, "y", tdt, (T, H, P)),
        code | (OUT_HADAMARD if hadamard else 0) | flag, float(y_scale),
        _ptr(workspace, "workspace", torch.uint8),
        workspace.numel(),
        _stream(stream),
    ]
    _check("ssd_i8_chunk_scan_varlen", library().ssd_i8_chunk_scan_varlen(*args))
    return y


@_device_call
def ssd_i8_state_update(state: torch.Tensor, x: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
                        dt: torch.Tensor, A: torch.Tensor, D: torch.Tensor,
                        x_scale: torch.Tensor, B_scale: torch.Tensor, C_scale: torch.Tensor, *,
                        y: Optional[torch.Tensor] = None, y_dtype: str = "f16",
                        y_scale: float = 1.0, stream=None, hadamard: bool = False) -> torch.Tensor:
    """One decode step, state f32 [b,h,p,n] updated in place; x int8 [b,h,p]; B, C int8
    [b,g,n]; dt f32 [b,h].  Returns y [b,h,p] of ``y_dtype`` (``hadamard``: y' = H y / 8 over
    headdim, ``SSD_OUT_HADAMARD``)."""
    bsz, H, P, N = state.shape
    G = B.shape[1]
    code, tdt = OUT_DTYPES[y_dtype]
    if y is None:
        y = torch.empty((bsz, H, P), dtype=tdt, device=state.device)
    pb, pc, flag = _bc_scales(B_scale, C_scale, G, N)
    args = [
        _ptr(state, "state", torch.float32, (bsz, H, P, N)),
        _ptr(x, "x", torch.int8, (bsz, H, P)),
        _ptr(B, "B", torch.int8, (bsz, G, N)),
        _ptr(C, "C", torch.int8, (bsz, G, N)),
        _ptr(dt, "dt", torch.float32, (bsz, H)),
        _ptr(A, "A", torch.float32, (H,)),
        _ptr(D, "D", torch.float32, (H,)),
        _ptr(x_scale, "x_scale", torch.float32, (H,)),
        pb, pc,
        bsz, H, P, N, G,
        _ptr(y, "y", tdt, (bsz, H, P)),
        code | (OUT_HADAMARD if hadamard else 0) | flag, float(y_scale),
        _stream(stream),
    ]
    _check("ssd_i8_state_update", library().ssd_i8_state_update(*args))
    return y


@_device_call
def ssd_i8_state_quantize(state: torch.Tensor, state_q: Optional[torch.Tensor] = None,
                          state_scale: Optional[torch.Tensor] = None, stream=None):
    """fp32 state [b,h,p,n] -> (int8 codes [b,h,p,n], float32 scales [b,h]) with scale =
    max|h| / 127 per (batch, head) (see ``ssd_i8_state_quantize`` in include/ssd_i8.h)."""
    bsz, H, P, N = state.shape
    if state_q is None:
        state_q = torch.empty((bsz, H, P, N), dtype=torch.int8, device=state.device)
    if state_scale is None:
        state_scale = torch.empty((bsz, H), dtype=torch.float32, device=state.device)
    _check("ssd_i8_state_quantize", library().ssd_i8_state_quantize(
        _ptr(state, "state", torch.float32, (bsz, H, P, N)),
        _ptr(state_q, "state_q", torch.int8, (bsz, H, P, N)),
        _ptr(state_scale, "state_scale", torch.float32, (bsz, H)), bsz, H, P, N,
        _stream(stream)))
    return state_q, state_scale


@_device_call
def ssd_i8_state_update_q8(state_q: torch.Tensor, state_scale: torch.Tensor, x: torch.Tensor,
                           B: torch.Tensor, C: torch.Tensor, dt: torch.Tensor, A: torch.Tensor,
                           D: torch.Tensor, x_scale: torch.Tensor, B_scale: torch.Tensor,
                           C_scale: torch.Tensor, *, y: Optional[torch.Tensor] = None,
                           y_dtype: str = "f16", y_scale: float = 1.0,
                           stream=None, hadamard: bool = False) -> torch.Tensor:
    """One decode step on the int8 cached state, in place (see ``ssd_i8_state_update_q8``).

    state_q int8 [b,h,p,n] and state_scale f32 [b,h] are updated; x int8 [b,h,p]; B, C int8
    [b,g,n]; dt f32 [b,h]; returns y [b,h,p] of ``y_dtype`` (``hadamard``: y' = H y / 8 over
    headdim)."""
    bsz, H, P, N = state_q.shape
    G = B.shape[1]
    code, tdt = OUT_DTYPES[y_dtype]
    if y is None:
        y = torch.empty((bsz, H, P), dtype=tdt, device=state_q.device)
    pb, pc, flag = _bc_scales(B_scale, C_scale, G, N)
    args = [
        _ptr(state_q, "state_q", torch.int8, (bsz, H, P, N)),
        _ptr(state_scale, "state_scale", torch.float32, (bsz, H)),
        _ptr(x, "x", torch.int8, (bsz, H, P)),
        _ptr(B, "B", torch.int8, (bsz, G, N)),
        _ptr(C, "C", torch.int8, (bsz, G, N)),
        _ptr(dt, "dt", torch.float32, (bsz, H)),
        _ptr(A, "A", torch.float32, (H,)),
        _ptr(D, "D", torch.float32, (H,)),
        _ptr(x_scale, "x_scale", torch.float32, (H,)),
        pb, pc,
        bsz, H, P, N, G,
        _ptr(y, "y", tdt, (bsz, H, P)),
        code | (OUT_HADAMARD if hadamard else 0) | flag, float(y_scale),
        _stream(stream),
    ]
    _check("ssd_i8_state_update_q8", library().ssd_i8_state_update_q8(*args))
    return y


@_device_call
def ssd_i8_chunk_cb(C: torch.Tensor, B: torch.Tensor, chunk_size: int, *,
                    cb: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """ChunkBMM export: int32 [b, ceil(l/Q), g, Q, Q] = Cq Bq^T per chunk and group."""
    bsz, L, G, N = C.shape
    Q = int(chunk_size)
    nch = (L + Q - 1) // Q
    if cb is None:
        cb = torch.empty((bsz, nch, G, Q, Q), dtype=torch.int32, device=C.device)
    args = [
        _ptr(C, "C", torch.int8, (bsz, L, G, N)),
        _ptr(B, "B", torch.int8, (bsz, L, G, N)),
        bsz, L, G, N, Q,
        _ptr(cb, "cb", torch.int32, (bsz, nch, G, Q, Q)),
        _stream(stream),
    ]
    _check("ssd_i8_chunk_cb", library().ssd_i8_chunk_cb(*args))
    return cb


def ssd_i8_debug_inject(drop_publish_cta: int, wait_cycles: int) -> None:
    """Test hook: arm a one-shot hand-off fault for the next chunk scan (see include/ssd_i8.h)."""
    _check("ssd_i8_debug_inject", library().ssd_i8_debug_inject(int(drop_publish_cta), int(wait_cycles)))


@_device_call
def ssd_i8_chunk_scan_status(workspace: torch.Tensor, stream=None) -> None:
    """Raise SSDError (SSD_ERR_TIMEOUT) if a chunk scan that ran on ``workspace`` since the
    previous status query on it (with none, since its first call) reported a device-side wait
    that gave up; synchronises the stream."""
    _check("ssd_i8_chunk_scan_status",
           library().ssd_i8_chunk_scan_status(_ptr(workspace, "workspace", torch.uint8),
                                              _stream(stream)))


@_device_call
def ssd_i8_chunk_scan_noalloc(x: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
                              dt: torch.Tensor, A: torch.Tensor, D: torch.Tensor,
                              x_scale: torch.Tensor, B_scale: torch.Tensor,
                              C_scale: torch.Tensor, chunk_size: int, *,
                              init_state: Optional[torch.Tensor] = None,
                              final_state: Optional[torch.Tensor] = None,
                              y: Optional[torch.Tensor] = None, y_dtype: str = "f16",
                              y_scale: float = 1.0, stream=None) -> torch.Tensor:
    """The chunk scan without a workspace, for callers that cannot allocate device memory:
    the library's built-in 4 MiB scratch (shared by all calls on a device) is used instead.
    Pass ``y`` to keep the call itself free of allocations; larger problems raise SSDError
    (SSD_ERR_WORKSPACE).  See ``ssd_i8_chunk_scan_noalloc`` in include/ssd_i8.h."""
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,l,h,p] and B/C [b,l,g,n]")
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    code, tdt = OUT_DTYPES[y_dtype]
    if y is None:
        y = torch.empty((bsz, L, H, P), dtype=tdt, device=x.device)
    args = [
        _ptr(x, "x", torch.int8, (bsz, L, H, P)),
        _ptr(B, "B", torch.int8, (bsz, L, G, N)),
        _ptr(C, "C", torch.int8, (bsz, L, G, N)),
        _ptr(dt, "dt", torch.float32, (bsz, L, H)),
        _ptr(A, "A", torch.float32, (H,)),
        _ptr(D, "D", torch.float32, (H,)),
        _ptr(x_scale, "x_scale", torch.float32, (H,)),
        *_bc_scales(B_scale, C_scale, G, N)[:2],
        bsz, L, H, P, N, G, int(chunk_size),
        _ptr(init_state, "init_state", torch.float32, (bsz, H, P, N)),
        _ptr(final_state, "final_state", torch.float32, (bsz, H, P, N)),
        _ptr(y, "y", tdt, (bsz, L, H, P)),
        code | _bc_scales(B_scale, C_scale, G, N)[2], float(y_scale),
        _stream(stream),
    ]
    _check("ssd_i8_chunk_scan_noalloc", library().ssd_i8_chunk_scan_noalloc(*args))
    return y


def ssd_i8_chunk_scan_noalloc_status(stream=None) -> None:
    """Raise SSDError (SSD_ERR_TIMEOUT) if the last allocation-free chunk scan on the current
    device reported a device-side wait that gave up; synchronises the stream.  See
    ``ssd_i8_chunk_scan_noalloc_status`` in include/ssd_i8.h."""
    _check("ssd_i8_chunk_scan_noalloc_status",
           library().ssd_i8_chunk_scan_noalloc_status(_stream(stream)))
