"""Seeded synthetic inputs for the int8 SSD chunk scan and its decode state update.

This module only draws random numbers and quantizes the drawn activations to the int8
inputs the op consumes; it holds none of the scan's arithmetic.  It is shared by the
CPU oracle tests, the GPU parity tests and ``bench.py``; it imports neither side.

Workloads follow the shapes the pages measure on (Mamba-2 1.3B / 2.7B / 8B SSD layers):

* x, B, C arrive as int8 with static symmetric scales: per tensor (Quamba project page,
  "static per-tensor quantization") or per head for x and per group for B/C
  (SSDi8 page, Table 10 "quantization axis": per-H(G)).  The per-tensor Mamba-2 baseline of
  the Quamba2 OpenReview rebuttal (the response listing Table R9) clips x at a percentile of
  |x| and quantizes B and C per tensor by their absmax: ``scales="percentile"``.
* x is head-structured with outlier channels (SSDi8 page, Figure 2; Quamba2 rebuttal,
  channel persistence), stood in for by Laplace values with 1 % of the (h, p) channels
  scaled x20, or a head-wise magnitude spread.
* dt = softplus(N(-2, 0.5)), A_h = -exp(U(0, ln 16)), D ~ N(0, 1): typical Mamba-2 ranges.

Random draws use numpy's PCG64 (``default_rng(seed)``), seed = 1000 + config index by
default, in the fixed order A, D, dt, x, B, C, outlier mask, magnitude spread.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "PrefillCase",
    "DecodeCase",
    "PREFILL_CONFIGS",
    "DECODE_CONFIG",
    "quantize_symmetric",
    "percentile_scale",
    "make_prefill",
    "make_prefill_config",
    "make_decode",
    "make_decode_config",
    "varlen_lengths",
    "make_varlen_config",
]

F32 = np.float32


@dataclasses.dataclass
class PrefillCase:
    """One prefill problem: int8 x/B/C plus fp32 dt, A, D and the static scales."""

    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk_size: int
    x: np.ndarray  # int8 [b, l, h, p]
    B: np.ndarray  # int8 [b, l, g, n]
    C: np.ndarray  # int8 [b, l, g, n]
    dt: np.ndarray  # f32 [b, l, h]
    A: np.ndarray  # f32 [h]
    D: np.ndarray  # f32 [h]
    x_scale: np.ndarray  # f32 [h]
    B_scale: np.ndarray  # f32 [g] (or [g, n] for scales="channel")
    C_scale: np.ndarray  # f32 [g] (or [g, n] for scales="channel")
    out_dtype: str = "f16"  # "f32" | "f16" | "i8"
    init_state: Optional[np.ndarray] = None  # f32 [b, h, p, n]

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


@dataclasses.dataclass
class DecodeCase:
    """A sequence of single-token state updates on one fp32 state."""

    name: str
    batch: int
    steps: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    state: np.ndarray  # f32 [b, h, p, n]
    x: np.ndarray  # int8 [steps, b, h, p]
    B: np.ndarray  # int8 [steps, b, g, n]
    C: np.ndarray  # int8 [steps, b, g, n]
    dt: np.ndarray  # f32 [steps, b, h]
    A: np.ndarray  # f32 [h]
    D: np.ndarray  # f32 [h]
    x_scale: np.ndarray  # f32 [h]
    B_scale: np.ndarray  # f32 [g]
    C_scale: np.ndarray  # f32 [g]
    out_dtype: str = "f16"


# name, batch, seqlen, nheads, headdim, dstate, ngroups, chunk, x/B/C law, scale axes, out dtype
PREFILL_CONFIGS = {
    0: dict(name="tiny-ssd-prefill b1 L256 h4 p64 n16 g1 Q64", batch=1, seqlen=256, nheads=4,
            headdim=64, dstate=16, ngroups=1, chunk_size=64, law="normal", scales="tensor",
            out_dtype="f16"),
    1: dict(name="mamba2-1.3b-ssd-prefill b4 L2048 h64 p64 n128 g1 Q256", batch=4, seqlen=2048,
            nheads=64, headdim=64, dstate=128, ngroups=1, chunk_size=256,
            law="laplace_outliers_x", scales="head", out_dtype="f16"),
    2: dict(name="mamba2-2.7b-ssd-prefill b8 L4096 h80 p64 n128 g1 Q256", batch=8, seqlen=4096,
            nheads=80, headdim=64, dstate=128, ngroups=1, chunk_size=256,
            law="laplace_spread", scales="head", out_dtype="f16"),
    3: dict(name="mamba2-8b-ssd-long-prefill b2 L16384 h128 p64 n128 g8 Q256 int8-out", batch=2,
            seqlen=16384, nheads=128, headdim=64, dstate=128, ngroups=8, chunk_size=256,
            law="laplace_outliers_all", scales="head", out_dtype="i8"),
    # the same layer and activations under the per-tensor static recipe: x clipped at the
    # 99.99th percentile of |x|, B and C per-tensor absmax
    4: dict(name="mamba2-8b-ssd-long-prefill per-tensor x-p99.99 b2 L16384 h128 p64 n128 g8 Q256 "
                 "int8-out", batch=2, seqlen=16384, nheads=128, headdim=64, dstate=128,
            ngroups=8, chunk_size=256, law="laplace_outliers_all", scales="percentile",
            out_dtype="i8"),
}

# tokens of a large activation that calibrate a percentile scale (a calibration set's worth)
CALIB_TOKENS = 2048

DECODE_CONFIG = dict(name="mamba2-8b-ssd-decode b128 x512 steps h128 p64 n128 g8", batch=128,
                     steps=512, nheads=128, headdim=64, dstate=128, ngroups=8, out_dtype="f16")


def quantize_symmetric(v: np.ndarray, scale_axis) -> tuple[np.ndarray, np.ndarray]:
    """Static symmetric int8 quantization: s = absmax / 127, q = clamp(rne(v / s), -127, 127).

    ``scale_axis`` is the axis that keeps its own scale (per head / per group), or a tuple of
    axes (per group and dstate channel); ``None`` gives one per-tensor scale.  Returns
    (q int8, s f32[...]); s has one entry per index of the kept axes (or a single entry).
    """
    v = np.asarray(v, dtype=F32)
    if v.ndim == 0:
        raise ValueError("quantize_symmetric expects an array")
    shape = [1] * v.ndim
    if scale_axis is None:
        amax = np.array([np.abs(v).max() if v.size else 0.0], dtype=np.float64)
    else:
        keep = (scale_axis,) if isinstance(scale_axis, int) else tuple(scale_axis)
        axes = tuple(i for i in range(v.ndim) if i not in keep)
        amax = (np.abs(v).max(axis=axes).astype(np.float64) if v.size
                else np.zeros(tuple(v.shape[k] for k in keep)))
        for k in keep:
            shape[k] = v.shape[k]
    s = np.where(amax > 0, amax / 127.0, 1.0).astype(F32)
    sb = s.reshape(shape)
    q = np.empty(v.shape, dtype=np.int8)
    # slabs along the first axis bound the host memory used at the large workloads
    for i in range(v.shape[0]):
        si = sb[i] if shape[0] > 1 else sb[0]
        r = np.rint(v[i] / si)  # round half to even, in fp32
        np.clip(r, -127, 127, out=r)
        q[i] = r.astype(np.int8)
    return q, s


def percentile_scale(v: np.ndarray, percentile: float) -> np.float32:
    """Static per-tensor scale clipped at a percentile: s = P_percentile(|v|) / 127 (numpy's
    linear interpolation between order statistics).  Values above the percentile saturate at
    +-127 when quantized with it.

    ``v`` is [batch, tokens, ...]; at most CALIB_TOKENS tokens, evenly spaced, calibrate the
    percentile (every token when there are fewer), all channels of each.
    """
    v = np.asarray(v, dtype=F32)
    step = max(1, -(-v.shape[1] // CALIB_TOKENS))
    sample = np.abs(v[:, ::step]).reshape(-1)
    t = float(np.percentile(sample, percentile)) if sample.size else 0.0
    return F32(t / 127.0) if t > 0 else F32(1.0)


def _quantize_with(v: np.ndarray, s: np.float32) -> np.ndarray:
    """q = clamp(rne(v / s), -127, 127) with one fp32 scale, in slabs along axis 0."""
    q = np.empty(v.shape, dtype=np.int8)
    for i in range(v.shape[0]):
        r = np.rint(v[i] / s)
        np.clip(r, -127, 127, out=r)
        q[i] = r.astype(np.int8)
    return q


def _laplace(rng: np.random.Generator, shape) -> np.ndarray:
    """Laplace(0, 1) in fp32: an Exp(1) magnitude with a fair random sign."""
    out = np.empty(shape, dtype=F32)
    rng.standard_exponential(dtype=F32, out=out)
    sign = rng.integers(0, 2, size=shape, dtype=np.int8)
    out *= (sign.astype(F32) * 2.0 - 1.0)
    return out


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    out = np.empty(shape, dtype=F32)
    rng.standard_normal(dtype=F32, out=out)
    return out


def _dt_A_D(rng: np.random.Generator, dt_shape, nheads: int):
    A = (-np.exp(rng.uniform(0.0, math.log(16.0), size=nheads))).astype(F32)
    D = rng.standard_normal(nheads).astype(F32)
    raw = rng.normal(-2.0, 0.5, size=dt_shape)
    dt = np.log1p(np.exp(raw)).astype(F32)  # softplus
    return A, D, dt


def make_prefill(batch: int, seqlen: int, nheads: int, headdim: int, dstate: int, ngroups: int,
                 chunk_size: int, *, law: str = "normal", scales: str = "head",
                 out_dtype: str = "f16", seed: int = 0, with_init_state: bool = False,
                 name: Optional[str] = None, clip_percentile: float = 99.99) -> PrefillCase:
    """Draw one seeded prefill problem.

    law: "normal" (x, B, C ~ N(0,1)); "laplace_outliers_x" (x Laplace with 1 % outlier
    channels x20 over (h,p); B, C ~ N(0,1)); "laplace_spread" (x, B, C Laplace, x scaled
    per head and B, C per group by U(0.5, 8)); "laplace_outliers_all" (x, B, C Laplace with
    1 % outlier channels x20: x over (h,p), B and C over (g,n)).
    scales: "tensor" (one scale per tensor, broadcast), "head" (x per head, B/C per group),
    "channel" (x per head, B/C per group and dstate channel, [g, n]: the per-P(N) axis, taken
    by the kernels with SSD_SCALES_PER_N) or "percentile" (per tensor; x clipped at
    ``clip_percentile`` of |x|, B/C by absmax).
    """
    if nheads % ngroups:
        raise ValueError("nheads must be a multiple of ngroups")
    rng = np.random.default_rng(seed)
    A, D, dt = _dt_A_D(rng, (batch, seqlen, nheads), nheads)
    xs = (batch, seqlen, nheads, headdim)
    bs = (batch, seqlen, ngroups, dstate)
    if law == "normal" or law == "laplace_outliers_x":
        x = _laplace(rng, xs) if law == "laplace_outliers_x" else _normal(rng, xs)
        Bf = _normal(rng, bs)
        Cf = _normal(rng, bs)
    elif law in ("laplace_spread", "laplace_outliers_all"):
        x = _laplace(rng, xs)
        Bf = _laplace(rng, bs)
        Cf = _laplace(rng, bs)
    else:
        raise ValueError(f"unknown law {law!r}")
    # outlier mask, then magnitude spread (fixed draw order)
    if law in ("laplace_outliers_x", "laplace_outliers_all"):
        xm = rng.random(nheads * headdim) < 0.01
        x *= np.where(xm, 20.0, 1.0).astype(F32).reshape(1, 1, nheads, headdim)
        if law == "laplace_outliers_all":
            bm = rng.random(ngroups * dstate) < 0.01
            cm = rng.random(ngroups * dstate) < 0.01
            Bf *= np.where(bm, 20.0, 1.0).astype(F32).reshape(1, 1, ngroups, dstate)
            Cf *= np.where(cm, 20.0, 1.0).astype(F32).reshape(1, 1, ngroups, dstate)
    if law == "laplace_spread":
        hs = rng.uniform(0.5, 8.0, size=nheads).astype(F32)
        gs_b = rng.uniform(0.5, 8.0, size=ngroups).astype(F32)
        gs_c = rng.uniform(0.5, 8.0, size=ngroups).astype(F32)
        x *= hs.reshape(1, 1, nheads, 1)
        Bf *= gs_b.reshape(1, 1, ngroups, 1)
        Cf *= gs_c.reshape(1, 1, ngroups, 1)
    if scales == "tensor":
        xq, sx = quantize_symmetric(x, None)
        Bq, sb = quantize_symmetric(Bf, None)
        Cq, sc = quantize_symmetric(Cf, None)
        sx = np.full(nheads, sx[0], dtype=F32)
        sb = np.full(ngroups, sb[0], dtype=F32)
        sc = np.full(ngroups, sc[0], dtype=F32)
    elif scales == "percentile":
        s_x = percentile_scale(x, clip_percentile)
        xq = _quantize_with(x, s_x)
        Bq, sb = quantize_symmetric(Bf, None)
        Cq, sc = quantize_symmetric(Cf, None)
        sx = np.full(nheads, s_x, dtype=F32)
        sb = np.full(ngroups, sb[0], dtype=F32)
        sc = np.full(ngroups, sc[0], dtype=F32)
    elif scales == "head":
        xq, sx = quantize_symmetric(x, 2)
        Bq, sb = quantize_symmetric(Bf, 2)
        Cq, sc = quantize_symmetric(Cf, 2)
    elif scales == "channel":  # x per head; B and C per group and dstate channel: [g, n]
        xq, sx = quantize_symmetric(x, 2)
        Bq, sb = quantize_symmetric(Bf, (2, 3))
        Cq, sc = quantize_symmetric(Cf, (2, 3))
    else:
        raise ValueError(f"unknown scales {scales!r}")
    del x, Bf, Cf
    init = None
    if with_init_state:
        init = (0.1 * rng.standard_normal((batch, nheads, headdim, dstate))).astype(F32)
    return PrefillCase(
        name=name or f"prefill b{batch} L{seqlen} h{nheads} p{headdim} n{dstate} g{ngroups} Q{chunk_size}",
        batch=batch, seqlen=seqlen, nheads=nheads, headdim=headdim, dstate=dstate,
        ngroups=ngroups, chunk_size=chunk_size, x=xq, B=Bq, C=Cq, dt=dt, A=A, D=D,
        x_scale=sx, B_scale=sb, C_scale=sc, out_dtype=out_dtype, init_state=init)


def make_exact_readout(batch: int, seqlen: int, ngroups: int, dstate: int, chunk_size: int = 256,
                       seed: int = 0, dt_log2: int = -3, headdim: int = 64) -> PrefillCase:
    """A prefill whose every intermediate is exactly representable, so that y reads out the
    ChunkBMM products one by one.

    B and C codes are drawn uniformly from {-1, 0, 1}; x is one-hot: head j of a group (there
    are ceil(seqlen / headdim) heads per group) carries a 1 at token headdim * j + p in column p
    and 0 elsewhere.  dt is 2^dt_log2 everywhere, A = D = 0 (no decay, no skip term), and the
    scales are powers of two (s_x = 1/2, s_B = 1/4, s_C = 1/2).  With the state starting at
    zero, the SSM recurrence then gives
        y[b, t, h, p] = dt s_x s_B s_C (C_t . B_s),  s = headdim * j + p <= t  (0 for s > t)
    for head h = j of group g, an integer times a power of two."""
    if seqlen < 1 or headdim < 1:
        raise ValueError("need seqlen >= 1 and headdim >= 1")
    rng = np.random.default_rng(seed)
    per_group = -(-seqlen // headdim)
    H = ngroups * per_group
    x = np.zeros((batch, seqlen, H, headdim), dtype=np.int8)
    for h in range(H):
        j = h % per_group
        for p in range(headdim):
            s = headdim * j + p
            if s < seqlen:
                x[:, s, h, p] = 1
    B = rng.integers(-1, 2, size=(batch, seqlen, ngroups, dstate)).astype(np.int8)
    C = rng.integers(-1, 2, size=(batch, seqlen, ngroups, dstate)).astype(np.int8)
    dt = np.full((batch, seqlen, H), 2.0 ** dt_log2, dtype=np.float32)
    zeros_h = np.zeros(H, dtype=np.float32)
    return PrefillCase(
        name=f"exact readout b{batch} L{seqlen} h{H} p{headdim} n{dstate} g{ngroups} Q{chunk_size}",
        batch=batch, seqlen=seqlen, nheads=H, headdim=headdim, dstate=dstate, ngroups=ngroups,
        chunk_size=chunk_size, x=x, B=B, C=C, dt=dt, A=zeros_h, D=zeros_h.copy(),
        x_scale=np.full(H, 0.5, dtype=np.float32), B_scale=np.full(ngroups, 0.25, dtype=np.float32),
        C_scale=np.full(ngroups, 0.5, dtype=np.float32), out_dtype="f32")


def make_exact_readout_varlen(lengths, ngroups: int, dstate: int, chunk_size: int = 256,
                              seed: int = 0, headdim: int = 64):
    """The exact-readout family (``make_exact_readout``) over packed sequences of the given
    lengths: one row of sum(lengths) tokens, and in sequence i head j of a group carries a 1 at
    the sequence's token headdim * j + p in column p.  Every sequence shares the head count
    ngroups * ceil(max length / headdim).  Returns (case with batch 1, cu_seqlens int32)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    if lengths.ndim != 1 or (lengths < 0).any():
        raise ValueError("lengths must be a 1-D sequence of non-negative integers")
    T = int(lengths.sum())
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    per_group = max(1, -(-int(lengths.max(initial=0)) // headdim))
    H = ngroups * per_group
    rng = np.random.default_rng(seed)
    x = np.zeros((1, max(T, 1), H, headdim), dtype=np.int8)
    for i, L in enumerate(lengths):
        for h in range(H):
            j = h % per_group
            for p in range(headdim):
                t = headdim * j + p
                if t < L:
                    x[0, cu[i] + t, h, p] = 1
    B = rng.integers(-1, 2, size=(1, max(T, 1), ngroups, dstate)).astype(np.int8)
    C = rng.integers(-1, 2, size=(1, max(T, 1), ngroups, dstate)).astype(np.int8)
    dt = np.full((1, max(T, 1), H), 0.125, dtype=np.float32)
    zeros_h = np.zeros(H, dtype=np.float32)
    case = PrefillCase(
        name=f"exact readout packed T{T} nseq{len(lengths)} h{H} p{headdim} n{dstate} g{ngroups}",
        batch=1, seqlen=max(T, 1), nheads=H, headdim=headdim, dstate=dstate, ngroups=ngroups,
        chunk_size=chunk_size, x=x, B=B, C=C, dt=dt, A=zeros_h, D=zeros_h.copy(),
        x_scale=np.full(H, 0.5, dtype=np.float32), B_scale=np.full(ngroups, 0.25, dtype=np.float32),
        C_scale=np.full(ngroups, 0.5, dtype=np.float32), out_dtype="f32")
    return case, cu


def make_prefill_config(index: int, seed: Optional[int] = None, **overrides) -> PrefillCase:
    """The prefill workload ``index`` (0..4) with its default seed 1000 + index."""
    spec = dict(PREFILL_CONFIGS[index])
    spec.update(overrides)
    name = spec.pop("name")
    if overrides:  # a smaller case of the same shape (profiling captures) says so in its name
        name += " [" + ", ".join(f"{k}={v}" for k, v in sorted(overrides.items())) + "]"
    return make_prefill(seed=1000 + index if seed is None else seed, name=name, **spec)


def make_decode(batch: int, steps: int, nheads: int, headdim: int, dstate: int, ngroups: int, *,
                out_dtype: str = "f16", seed: int = 0, name: Optional[str] = None,
                scales: str = "head") -> DecodeCase:
    """Draw a seeded decode run: an fp32 state ~ N(0, 0.1^2) and ``steps`` fresh tokens.

    Per step x, B, C ~ N(0, 1), quantized with static scales (x per head, B/C per group, or
    with ``scales="channel"`` per group and dstate channel, [g, n]) calibrated over all steps;
    dt, A, D as in the prefill workloads.
    """
    if nheads % ngroups:
        raise ValueError("nheads must be a multiple of ngroups")
    rng = np.random.default_rng(seed)
    A, D, dt = _dt_A_D(rng, (steps, batch, nheads), nheads)
    x = _normal(rng, (steps, batch, nheads, headdim))
    Bf = _normal(rng, (steps, batch, ngroups, dstate))
    Cf = _normal(rng, (steps, batch, ngroups, dstate))
    state = (0.1 * _normal(rng, (batch, nheads, headdim, dstate))).astype(F32)
    xq, sx = quantize_symmetric(x, 2)
    if scales == "head":
        Bq, sb = quantize_symmetric(Bf, 2)
        Cq, sc = quantize_symmetric(Cf, 2)
    elif scales == "channel":
        Bq, sb = quantize_symmetric(Bf, (2, 3))
        Cq, sc = quantize_symmetric(Cf, (2, 3))
    else:
        raise ValueError(f"unknown scales {scales!r}")
    return DecodeCase(
        name=name or f"decode b{batch} x{steps} h{nheads} p{headdim} n{dstate} g{ngroups}",
        batch=batch, steps=steps, nheads=nheads, headdim=headdim, dstate=dstate,
        ngroups=ngroups, state=state, x=xq, B=Bq, C=Cq, dt=dt, A=A, D=D, x_scale=sx,
        B_scale=sb, C_scale=sc, out_dtype=out_dtype)


def make_decode_config(seed: Optional[int] = None, **overrides) -> DecodeCase:
    """The decode workload (batch 128, 512 steps, Mamba-2-8B head shape), seed 1004."""
    spec = dict(DECODE_CONFIG)
    spec.update(overrides)
    name = spec.pop("name")
    if overrides:
        name += " [" + ", ".join(f"{k}={v}" for k, v in sorted(overrides.items())) + "]"
    return make_decode(seed=1004 if seed is None else seed, name=name, **spec)


# the packed serving prefill: the 8B layer's 32768 tokens as a batch of prompts of mixed length
VARLEN_CONFIG = dict(total_tokens=32768, min_len=64, max_len=8192, nheads=128, headdim=64,
                     dstate=128, ngroups=8, chunk_size=256, law="laplace_outliers_all",
                     scales="head", out_dtype="i8")


def varlen_lengths(total: int, min_len: int, max_len: int, seed: int) -> np.ndarray:
    """Sequence lengths drawn log-uniformly from [min_len, max_len] until they fill ``total``
    tokens (the last one is cut to fit); int32."""
    if total < 0 or min_len < 1 or max_len < min_len:
        raise ValueError("need total >= 0 and 1 <= min_len <= max_len")
    rng = np.random.default_rng(seed)
    out = []
    left = total
    while left > 0:
        n = int(np.exp(rng.uniform(np.log(min_len), np.log(max_len + 1))))
        n = max(1, min(n, max_len, left))
        out.append(n)
        left -= n
    return np.asarray(out, dtype=np.int32)


def make_varlen_config(seed: Optional[int] = None, **overrides):
    """The packed serving prefill of the Mamba-2-8B layer: one row of ``total_tokens`` tokens
    (the activation laws of the 8B long prefill), cut into sequences whose lengths are drawn
    log-uniformly from [min_len, max_len].  Returns (case with batch 1, cu_seqlens int32)."""
    spec = dict(VARLEN_CONFIG)
    spec.update(overrides)
    seed = 1005 if seed is None else seed
    T = spec.pop("total_tokens")
    lengths = varlen_lengths(T, spec.pop("min_len"), spec.pop("max_len"), seed + 1)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    name = (f"mamba2-8b-ssd-packed-serving-prefill T{T} nseq{len(lengths)} "
            f"h{spec['nheads']} p{spec['headdim']} n{spec['dstate']} g{spec['ngroups']} "
            f"Q{spec['chunk_size']} int8-out strided")
    case = make_prefill(1, max(T, 1), spec.pop("nheads"), spec.pop("headdim"), spec.pop("dstate"),
                        spec.pop("ngroups"), spec.pop("chunk_size"), seed=seed, name=name, **spec)
    return case, cu
