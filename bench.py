"""Benchmark of the int8 SSD chunk scan (and its decode state update) on B200.

One JSON line on rank 0.  A "step" is one ``ssd_i8_chunk_scan`` call over the Mamba-2-8B
shaped long prefill (batch 2 x 16384 tokens, 128 heads x 64, dstate 128, 8 groups, chunk
256, int8 output): chunk_cumsum, ChunkBMM, chunk_state, state passing, chunk_scan and the
requantizing epilogue.  ``value`` = tokens/s with inputs resident in HBM; ``e2e`` = the same
through the public call with pinned-host inputs copied in and the int8 output copied back in
every step.  The decode state update (batch 128, 512 steps) is reported beside it under
``decode``; the packed serving prefill (prompts of mixed length as strided views of one
projection buffer, ``ssd_i8_chunk_scan_varlen``) under ``varlen_strided``.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch under torch.distributed.run; every rank scans its own batch (weak scaling,
no collective on the data path; the only collective is the max-over-ranks of the timings).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from quantized_mamba_ssd_b200 import workloads as W  # noqa: E402
from quantized_mamba_ssd_b200.dist_util import aggregate_tokens_per_s, max_over_ranks, rank_seed  # noqa: E402

PREFILL_CFG = 3
PER_TENSOR_CFG = 4  # the same layer under the per-tensor percentile-clipped recipe
METRIC = "SSD scan tokens/s (int8 in) at 1 B200; achieved fraction of HBM/int8 roofline"
UNIT = "tokens/s"
INT8_PER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput ratio on B200 (4.5 : 2.25)
NOMINAL_HBM_GBS = 7700.0  # B200 HBM3e datasheet bandwidth (HGX), context for the measured peak


# ------------------------------------------------------------------------------------------
# algorithmic work of one call (bytes moved once, int8 MMA ops of the causal contractions)
# ------------------------------------------------------------------------------------------
# DRAM traffic (read + write) per token of the fused chunk-scan kernel, from one ncu capture,
# keyed by the SHA-256 of the kernel source that ran under it; see
# profiles/ncu_fused_chunk_scan_b2_L8192.md.  The traffic grows in proportion to the tokens of a
# launch, so the bench scales it to the workload.  A changed kernel reports null.
_CAPTURED_TRAFFIC_PER_TOKEN = {
    "f49754942ee3a1e403d29bf7941f7579f5176cb7effce65f49bab0607a1226b3": (179.271424e6 + 108.001792e6) / 16384,
}


# The same for the decode kernels, per (batch, head) item of one step; see
# profiles/ncu_state_update_decode_b32.md and profiles/ncu_state_update_q8_decode_b128.md.
_CAPTURED_DECODE_TRAFFIC_PER_ITEM = {
    "state_update.cu": {
        "dbcc58a871c5d4171d5134d6be749c7661410af95c3498b2f3f5b0a99ad2ffdc": (134.594304e6 + 75.850496e6) / (32 * 128),
    },
    "state_update_q8.cu": {
        # captured on the source 5b540318...; this one differs by comments and an unused helper
        "163058fc1d5ec17c0f39aa41cbe624d32d1f0c9b841046783ff8da9fefcc7881": (135.700480e6 + 77.127680e6) / (128 * 128),
    },
}


def _source_sha(name: str) -> str:
    import hashlib
    src = Path(__file__).resolve().parent / "quantized_mamba_ssd_b200" / "csrc" / name
    return hashlib.sha256(src.read_bytes()).hexdigest()


def captured_traffic(tokens: int):
    per_token = _CAPTURED_TRAFFIC_PER_TOKEN.get(_source_sha("chunk_scan_fused.cu"))
    return None if per_token is None else per_token * tokens


def captured_decode_traffic(kernel_source: str, items: int):
    per_item = _CAPTURED_DECODE_TRAFFIC_PER_ITEM[kernel_source].get(_source_sha(kernel_source))
    return None if per_item is None else per_item * items


def prefill_alg_bytes(c: W.PrefillCase, out_bytes: int, final_state: bool) -> int:
    b, L, H, P, N, G = c.batch, c.seqlen, c.nheads, c.headdim, c.dstate, c.ngroups
    n = b * L * H * P  # x in (int8)
    n += 2 * b * L * G * N  # B, C in (int8)
    n += 4 * b * L * H  # dt (f32)
    n += out_bytes * b * L * H * P  # y out
    if final_state:
        n += 4 * b * H * P * N
    return n


def prefill_alg_ops(c: W.PrefillCase) -> float:
    """2 x MACs: causal CB per group, causal M.x, chunk state B^T x and C.H_prev per head."""
    b, L, H, P, N, G, Q = c.batch, c.seqlen, c.nheads, c.headdim, c.dstate, c.ngroups, c.chunk_size
    nch = -(-L // Q)
    causal = Q * (Q + 1) / 2
    cb = b * nch * G * causal * N
    mx = b * nch * H * causal * P
    st = b * L * H * P * N
    ch = b * L * H * N * P
    return 2.0 * (cb + mx + st + ch)


def decode_alg_bytes(d: W.DecodeCase, out_bytes: int, state_bytes: int = 4) -> int:
    """Bytes one decode step moves: the state read and written once (fp32, or int8 codes plus
    one fp32 scale per (batch, head) read and written), x, B, C, dt and y."""
    b, H, P, N, G = d.batch, d.nheads, d.headdim, d.dstate, d.ngroups
    state = 2 * state_bytes * b * H * P * N + (2 * 4 * b * H if state_bytes == 1 else 0)
    return state + b * H * P + 2 * b * G * N + 4 * b * H + out_bytes * b * H * P


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


def device_status_field(statuses: dict) -> str:
    """The line's ``device_status``: "ok" when every timed chunk-scan leg reported SSD_OK
    after its loop.  A leg whose bounded device-side wait gave up ended early, so its time
    means nothing: the run stops with a non-zero exit instead of printing a number.
    ``statuses`` maps a leg name to None (OK) or the failing status code."""
    bad = {k: v for k, v in statuses.items() if v is not None}
    if bad:
        print(json.dumps({"error": "device-side wait gave up in the timed region",
                          "legs": bad}), file=sys.stderr, flush=True)
        raise SystemExit(3)
    return "ok"


def scan_status(ssd_i8, workspace):
    """None if the last chunk scan on ``workspace`` reported no device-side failure, else its
    status code (the call synchronises the stream)."""
    try:
        ssd_i8.ssd_i8_chunk_scan_status(workspace)
    except ssd_i8.SSDError as e:
        return e.status
    return None


# ------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report clocks as unavailable
            self.ok = False

    def _handle(self, device_index):
        import torch
        pynvml = self.nvml
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(device_index)

    def _run(self):
        pynvml = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
                self.reasons |= pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------
# CPU baseline / reference arm: the oracle on a bounded sample of the same workload
# ------------------------------------------------------------------------------------------
def oracle_tokens_per_s(case: W.PrefillCase, target_s: float = 15.0):
    import oracle
    oracle.build()
    probe = min(case.seqlen, 64)

    def run(Ls):
        t0 = time.perf_counter()
        _, _, nt = oracle.scan(case.x[:, :Ls], case.B[:, :Ls], case.C[:, :Ls], case.dt[:, :Ls],
                               case.A, case.D, case.x_scale, case.B_scale, case.C_scale,
                               want_final_state=False)
        return time.perf_counter() - t0, nt

    tp, _ = run(probe)
    Ls = int(min(case.seqlen, max(probe, probe * target_s / max(tp, 1e-6))))
    t, nt = run(Ls)
    tokens = case.batch * Ls
    return tokens / t, nt, (f"first {Ls} of {case.seqlen} tokens of every (batch, head) pair of "
                            f"the workload ({tokens} tokens x {case.nheads} heads), fp64 oracle")


def reference_arm(args, case: W.PrefillCase):
    """--impl reference: the fp64 CPU oracle, as it stands, on bounded samples."""
    import oracle
    oracle.build()
    Ls = min(case.seqlen, 512)
    xs = (case.x[:, :Ls], case.B[:, :Ls], case.C[:, :Ls], case.dt[:, :Ls])
    times = []
    nt = 0
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        _, _, nt = oracle.scan(*xs, case.A, case.D, case.x_scale, case.B_scale, case.C_scale,
                               want_final_state=False)
        dtm = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dtm)
    tot = sum(times)
    tokens = case.batch * Ls * len(times)
    value = tokens / tot
    sample = (f"first {Ls} of {case.seqlen} tokens of every (batch, head) pair per step "
              f"({case.batch * Ls} tokens x {case.nheads} heads), fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, shapes and value laws of the workload)",
        "config": {"workload": case.name, "global_batch": case.batch, "seq_len": case.seqlen,
                   "sample_seq_len": Ls, "parallelism": "cpu threads over (batch, head)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nt, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------
def prefill_leg(args, index, rank, world, dev, ssd_i8, barrier, hbm_peak, int8_peak_tops, cpu,
                **overrides):
    """Time ssd_i8_chunk_scan on prefill workload ``index`` (with ``overrides`` of its recipe,
    e.g. per-channel B/C scales) in its own output dtype, with the final states written:
    (report dict, device status of the leg)."""
    import torch
    case = W.make_prefill_config(index, seed=rank_seed(1000 + index, rank), **overrides)
    x, B, C = (torch.from_numpy(a).to(dev) for a in (case.x, case.B, case.C))
    dt = torch.from_numpy(case.dt).to(dev)
    A, Dp, sx, sb, sc = (torch.from_numpy(a).to(dev) for a in
                         (case.A, case.D, case.x_scale, case.B_scale, case.C_scale))
    bsz, L, H, P, N, G, Q = (case.batch, case.seqlen, case.nheads, case.headdim, case.dstate,
                             case.ngroups, case.chunk_size)
    out = case.out_dtype
    ob = {"f32": 4, "f16": 2, "i8": 1}[out]
    y = torch.empty((bsz, L, H, P), dtype=ssd_i8.OUT_DTYPES[out][1], device=dev)
    fs = torch.empty((bsz, H, P, N), dtype=torch.float32, device=dev)
    ws = torch.empty(ssd_i8.ssd_i8_chunk_scan_workspace_size(bsz, L, H, P, N, G, Q),
                     dtype=torch.uint8, device=dev)

    def step():
        ssd_i8.ssd_i8_chunk_scan(x, B, C, dt, A, Dp, sx, sb, sc, Q, final_state=fs, y=y,
                                 y_dtype=out, y_scale=0.05, workspace=ws)

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    status = scan_status(ssd_i8, ws)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
    alg_bytes = prefill_alg_bytes(case, ob, True)
    alg_ops = prefill_alg_ops(case)
    t_hbm = alg_bytes / (hbm_peak * 1e9)
    t_ops = alg_ops / (int8_peak_tops * 1e12)
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    per_n = case.B_scale.ndim == 2
    leg = {
        "metric": f"SSD scan tokens/s (int8 in), {out} out"
                  + (", B/C scales per dstate channel" if per_n else ""), "workload": case.name,
        "value": aggregate_tokens_per_s(bsz * L, world, ms), "unit": UNIT, "ms_per_step": ms,
        "gpu_launches": args.steps * ssd_i8.KERNELS_PER_CHUNK_SCAN,
        "roofline": {"bound": "hbm" if t_hbm >= t_ops else "tensor", "achieved": gbs,
                     "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak, "traffic": None,
                     "alg_bytes_per_launch": alg_bytes,
                     "alg_bytes_without_final_state": prefill_alg_bytes(case, ob, False),
                     "alg_int8_ops_per_launch": alg_ops,
                     "roofline_us": 1e6 * max(t_hbm, t_ops)},
        "clocks": clocks.summary(),
        "cpu_baseline": None,
    }
    del x, B, C, dt, y, fs, ws
    if cpu:
        v, nt, sample = oracle_tokens_per_s(case, target_s=8.0)
        leg["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": nt, "kind": "oracle",
                               "sample": sample}
    return leg, status


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-passes", type=int, default=3,
                    help="timed passes of the 512-step decode run (0 skips the decode report)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) leg")
    ap.add_argument("--no-per-tensor", action="store_true",
                    help="skip the per-tensor percentile-clipped workload leg")
    ap.add_argument("--no-varlen", action="store_true",
                    help="skip the packed variable-length (strided) serving prefill leg")
    ap.add_argument("--no-smaller", action="store_true",
                    help="skip the 1.3B- and 2.7B-shaped prefill legs")
    ap.add_argument("--no-per-channel", action="store_true",
                    help="skip the per-dstate-channel B/C scale leg")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="decode batch per rank (default: the workload's 128); smaller batches "
                         "of the same shape serve profiling captures")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per rank (default: the workload's batch of 2); a smaller "
                         "batch of the same shape serves profiling captures")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="tokens per sequence (default: the workload's 16384); a shorter "
                         "sequence of the same shape serves profiling captures")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        reference_arm(args, W.make_prefill_config(PREFILL_CFG))
        return

    import torch
    import torch.distributed as dist
    from quantized_mamba_ssd_b200 import ssd_i8

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    ssd_i8.library()

    hbm_peak, bf16_peak, bf16_sus, peak_kind = load_peaks()
    int8_peak_tops = bf16_peak * INT8_PER_BF16

    # ---- prefill workload: this rank's own batch (seeded per rank) ----
    overrides = {}
    if args.batch is not None:
        overrides["batch"] = args.batch
    if args.seqlen is not None:
        overrides["seqlen"] = args.seqlen
    case = W.make_prefill_config(PREFILL_CFG, seed=rank_seed(1000 + PREFILL_CFG, rank), **overrides)
    x, B, C = (torch.from_numpy(a).to(dev) for a in (case.x, case.B, case.C))
    dt = torch.from_numpy(case.dt).to(dev)
    A, Dp, sx, sb, sc = (torch.from_numpy(a).to(dev) for a in
                         (case.A, case.D, case.x_scale, case.B_scale, case.C_scale))
    bsz, L, H, P, N, G, Q = (case.batch, case.seqlen, case.nheads, case.headdim, case.dstate,
                             case.ngroups, case.chunk_size)
    y = torch.empty((bsz, L, H, P), dtype=torch.int8, device=dev)
    fs = torch.empty((bsz, H, P, N), dtype=torch.float32, device=dev)
    ws = torch.empty(ssd_i8.ssd_i8_chunk_scan_workspace_size(bsz, L, H, P, N, G, Q),
                     dtype=torch.uint8, device=dev)
    # static output scale: a fixed calibration constant for the int8 output (the parity tests
    # calibrate it on the oracle; here it only sets the clamp range)
    y_scale = 0.05

    def step():
        ssd_i8.ssd_i8_chunk_scan(x, B, C, dt, A, Dp, sx, sb, sc, Q, final_state=fs, y=y,
                                 y_dtype="i8", y_scale=y_scale, workspace=ws)

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    statuses = {"main": scan_status(ssd_i8, ws)}
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, dev)
    tokens_all = bsz * L * world
    value = aggregate_tokens_per_s(bsz * L, world, ms_max)

    # ---- the same call with the Hadamard-transformed output (SSD_OUT_HADAMARD) ----
    def step_had():
        ssd_i8.ssd_i8_chunk_scan(x, B, C, dt, A, Dp, sx, sb, sc, Q, final_state=fs, y=y,
                                 y_dtype="i8", y_scale=y_scale, workspace=ws, hadamard=True)

    for _ in range(args.warmup):
        step_had()
    torch.cuda.synchronize()
    barrier()
    ev0.record(stream)
    for _ in range(args.steps):
        step_had()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    statuses["hadamard_out"] = scan_status(ssd_i8, ws)
    had_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)

    # ---- end to end: pinned host inputs in, int8 output back, every step ----
    hx, hB, hC, hdt = (torch.from_numpy(a).pin_memory() for a in (case.x, case.B, case.C, case.dt))
    hys = [torch.empty((bsz, L, H, P), dtype=torch.int8).pin_memory() for _ in range(2)]
    h2d = sum(t_.numel() * t_.element_size() for t_ in (hx, hB, hC, hdt))
    d2h = hys[0].numel() * hys[0].element_size()

    def e2e_step():
        x.copy_(hx, non_blocking=True)
        B.copy_(hB, non_blocking=True)
        C.copy_(hC, non_blocking=True)
        dt.copy_(hdt, non_blocking=True)
        step()
        hys[0].copy_(y, non_blocking=True)

    e2e = None
    if not args.no_e2e:
        e2e_steps = max(3, min(args.steps, 10))
        # serial: copy in, scan, copy out, one after the other on one stream
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        statuses["e2e_serial"] = scan_status(ssd_i8, ws)
        serial_ms = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps, dev)
        # pipelined: step i's inputs go up on one copy stream while step i - 1 computes and step
        # i - 2's output comes down on another (two device buffer sets, two host output buffers)
        bufs = [(x, B, C, dt, y), tuple(torch.empty_like(t_) for t_ in (x, B, C, dt, y))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_pipe(i):
            j = i % 2
            bx, bB, bC, bdt, by = bufs[j]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_done[j])  # the scan of step i - 2 has read buffer j
                for dst, src in ((bx, hx), (bB, hB), (bC, hC), (bdt, hdt)):
                    dst.copy_(src, non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            stream.wait_event(ev_out[j])  # step i - 2's output has left buffer j
            ssd_i8.ssd_i8_chunk_scan(bx, bB, bC, bdt, A, Dp, sx, sb, sc, Q, final_state=fs, y=by,
                                     y_dtype="i8", y_scale=y_scale, workspace=ws)
            ev_done[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[j])
                hys[j].copy_(by, non_blocking=True)
                ev_out[j].record(s_out)

        for i in range(3):
            e2e_pipe(i)
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        s_in.wait_event(ev0)
        for i in range(e2e_steps):
            e2e_pipe(i)
        for j in range(2):
            stream.wait_event(ev_out[j])
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        statuses["e2e_pipelined"] = scan_status(ssd_i8, ws)
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps, dev)
        e2e = {"value": aggregate_tokens_per_s(bsz * L, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms, "pipelined": True,
               "serial_value": aggregate_tokens_per_s(bsz * L, world, serial_ms),
               "serial_ms_per_step": serial_ms}
        del bufs

    # ---- the per-tensor static recipe on the same layer: x clipped at the 99.99th percentile,
    # B and C per-tensor absmax (same shapes, so the same algorithmic bytes) ----
    per_tensor = None
    if not args.no_per_tensor:
        pcase = W.make_prefill_config(PER_TENSOR_CFG, seed=rank_seed(1000 + PER_TENSOR_CFG, rank),
                                      **overrides)
        px, pB, pC = (torch.from_numpy(a).to(dev) for a in (pcase.x, pcase.B, pcase.C))
        pdt = torch.from_numpy(pcase.dt).to(dev)
        pA, pD, psx, psb, psc = (torch.from_numpy(a).to(dev) for a in
                                 (pcase.A, pcase.D, pcase.x_scale, pcase.B_scale, pcase.C_scale))

        def step_pt():
            ssd_i8.ssd_i8_chunk_scan(px, pB, pC, pdt, pA, pD, psx, psb, psc, Q, final_state=fs,
                                     y=y, y_dtype="i8", y_scale=y_scale, workspace=ws)

        for _ in range(args.warmup):
            step_pt()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step_pt()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        statuses["per_tensor_percentile"] = scan_status(ssd_i8, ws)
        pt_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
        pt_gbs = prefill_alg_bytes(pcase, 1, True) / (pt_ms * 1e-3) / 1e9
        per_tensor = {
            "metric": "SSD scan tokens/s (int8 in), per-tensor static scales, x clipped at the "
                      "99.99th percentile", "workload": pcase.name,
            "value": aggregate_tokens_per_s(bsz * L, world, pt_ms), "unit": UNIT,
            "ms_per_step": pt_ms, "gpu_launches": args.steps * ssd_i8.KERNELS_PER_CHUNK_SCAN,
            "saturated_x_fraction": float((np.abs(pcase.x.astype(np.int16)) == 127).mean()),
            "roofline": {"bound": "hbm", "achieved": pt_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": pt_gbs / hbm_peak, "traffic": None},
        }
        del px, pB, pC, pdt, pcase

    # ---- packed serving prefill: the layer's tokens as prompts of mixed length, read as
    # strided column slices of one projection buffer (ssd_i8_chunk_scan_varlen) ----
    varlen = None
    if not args.no_varlen:
        vcase, cu = W.make_varlen_config(seed=rank_seed(1005, rank),
                                         **({} if args.seqlen is None and args.batch is None
                                            else {"total_tokens": bsz * L}))
        T = int(cu[-1])
        nseq = len(cu) - 1
        xw = H * P + 2 * G * N  # one projection row: x | B | C
        proj = torch.empty((T, xw), dtype=torch.int8, device=dev)
        proj[:, :H * P] = torch.from_numpy(vcase.x.reshape(T, H * P)).to(dev)
        proj[:, H * P:H * P + G * N] = torch.from_numpy(vcase.B.reshape(T, G * N)).to(dev)
        proj[:, H * P + G * N:] = torch.from_numpy(vcase.C.reshape(T, G * N)).to(dev)
        vx = proj[:, :H * P].view(T, H, P)
        vB = proj[:, H * P:H * P + G * N].view(T, G, N)
        vC = proj[:, H * P + G * N:].view(T, G, N)
        vdt = torch.from_numpy(vcase.dt.reshape(T, H)).to(dev)
        vA, vD, vsx, vsb, vsc = (torch.from_numpy(a).to(dev) for a in
                                 (vcase.A, vcase.D, vcase.x_scale, vcase.B_scale, vcase.C_scale))
        vy = torch.empty((T, H, P), dtype=torch.int8, device=dev)
        vfs = torch.empty((nseq, H, P, N), dtype=torch.float32, device=dev)
        vws = torch.empty(ssd_i8.ssd_i8_chunk_scan_varlen_workspace_size(nseq), dtype=torch.uint8,
                          device=dev)

        def step_vl():
            ssd_i8.ssd_i8_chunk_scan_varlen(vx, vB, vC, vdt, vA, vD, vsx, vsb, vsc, cu, Q,
                                            final_state=vfs, y=vy, y_dtype="i8",
                                            y_scale=y_scale, workspace=vws)

        for _ in range(args.warmup):
            step_vl()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step_vl()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        statuses["varlen_strided"] = scan_status(ssd_i8, vws)
        vl_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
        vl_bytes = (T * (H * P + 2 * G * N + 4 * H + H * P)  # x, B, C, dt in; y out (int8)
                    + 4 * nseq * H * P * N)  # final states
        vl_gbs = vl_bytes / (vl_ms * 1e-3) / 1e9
        blocks = int(sum(-(-int(n) // 128) for n in (cu[1:] - cu[:-1])))
        varlen = {
            "metric": "SSD scan tokens/s (int8 in), packed variable-length sequences read as "
                      "strided views of one projection buffer, int8 out",
            "workload": vcase.name, "value": aggregate_tokens_per_s(T, world, vl_ms),
            "unit": UNIT, "ms_per_step": vl_ms, "sequences": nseq,
            "length_mix": "log-uniform in [64, 8192] tokens, last cut to fill",
            "min_len": int((cu[1:] - cu[:-1]).min()), "max_len": int((cu[1:] - cu[:-1]).max()),
            "token_blocks_of_128": blocks, "padded_token_fraction": 1.0 - T / (128.0 * blocks),
            "x_token_stride_bytes": xw, "gpu_launches": args.steps * ssd_i8.KERNELS_PER_CHUNK_SCAN,
            "roofline": {"bound": "hbm", "achieved": vl_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": vl_gbs / hbm_peak, "traffic": None,
                         "alg_bytes_per_launch": vl_bytes},
        }
        del proj, vx, vB, vC, vdt, vy, vfs, vws, vcase

    # ---- the 1.3B- and 2.7B-shaped prefills (f16 out, final states written) ----
    smaller = {}
    if not args.no_smaller:
        for idx, key in ((1, "prefill_1p3b"), (2, "prefill_2p7b")):
            smaller[key], statuses[key] = prefill_leg(
                args, idx, rank, world, dev, ssd_i8, barrier, hbm_peak, int8_peak_tops,
                cpu=(rank == 0 and world == 1 and not args.no_cpu_baseline))

    # ---- the 8B-shaped long prefill with B and C scales per dstate channel ([g, n]) ----
    per_channel = None
    if not args.no_per_channel:
        per_channel, statuses["per_channel_scales"] = prefill_leg(
            args, PREFILL_CFG, rank, world, dev, ssd_i8, barrier, hbm_peak, int8_peak_tops,
            cpu=False, scales="channel", **overrides)

    # ---- roofline of the timed call ----
    alg_bytes = prefill_alg_bytes(case, 1, True)
    alg_ops = prefill_alg_ops(case)
    t_hbm = alg_bytes / (hbm_peak * 1e9)
    t_ops = alg_ops / (int8_peak_tops * 1e12)
    bound = "hbm" if t_hbm >= t_ops else "tensor"
    achieved_gbs = alg_bytes / (ms * 1e-3) / 1e9
    roofline = {
        "bound": bound, "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
        "frac": achieved_gbs / hbm_peak, "traffic": captured_traffic(bsz * L),
        "peak_kind": f"{peak_kind} HBM copy bandwidth",
        "alg_bytes_per_launch": alg_bytes, "alg_int8_ops_per_launch": alg_ops,
        "roofline_us": 1e6 * max(t_hbm, t_ops), "frac_of_roofline_time": 1e6 * max(t_hbm, t_ops) / (ms * 1e3),
        "int8_peak_tops": int8_peak_tops,
        "nominal_hbm_gbs": NOMINAL_HBM_GBS, "frac_of_nominal_hbm": achieved_gbs / NOMINAL_HBM_GBS,
    }

    had_gbs = alg_bytes / (had_ms * 1e-3) / 1e9
    hadamard_out = {
        "metric": "SSD scan tokens/s (int8 in), output y' = H y / 8 over headdim, int8",
        "value": aggregate_tokens_per_s(bsz * L, world, had_ms), "unit": UNIT,
        "ms_per_step": had_ms, "gpu_launches": args.steps * ssd_i8.KERNELS_PER_CHUNK_SCAN,
        "roofline": {"bound": "hbm", "achieved": had_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": had_gbs / hbm_peak, "traffic": None},
    }

    # ---- decode state update, 512 steps of batch 128 (CUDA graph replay) ----
    decode = None
    if args.decode_passes > 0:
        dover = {} if args.decode_batch is None else {"batch": args.decode_batch}
        d = W.make_decode_config(seed=rank_seed(1004, rank), **dover)
        st = torch.from_numpy(d.state).to(dev)
        dx, dB, dC, ddt = (torch.from_numpy(a).to(dev) for a in (d.x, d.B, d.C, d.dt))
        dA, dD, dsx, dsb, dsc = (torch.from_numpy(a).to(dev) for a in
                                 (d.A, d.D, d.x_scale, d.B_scale, d.C_scale))
        dy = torch.empty((d.steps, d.batch, d.nheads, d.headdim), dtype=torch.float16, device=dev)

        def decode_pass():
            for s in range(d.steps):
                ssd_i8.ssd_i8_state_update(st, dx[s], dB[s], dC[s], ddt[s], dA, dD, dsx, dsb, dsc,
                                           y=dy[s], y_dtype="f16")

        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            decode_pass()  # warm up on the capture stream
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode_pass()
        for _ in range(max(1, args.warmup // 2)):
            graph.replay()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(args.decode_passes):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        dms = max_over_ranks(ev0.elapsed_time(ev1) / args.decode_passes, dev)
        dbytes = decode_alg_bytes(d, 2) * d.steps
        dgbs = dbytes / (dms * 1e-3) / 1e9
        decode = {
            "metric": "SSD decode state-update tokens/s (int8 in, fp32 state)",
            "value": d.batch * d.steps * world / (dms * 1e-3), "unit": UNIT,
            "ms_per_512_steps": dms, "us_per_step": 1e3 * dms / d.steps,
            "workload": d.name, "gpu_launches_per_pass": d.steps,
            "roofline": {"bound": "hbm", "achieved": dgbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": dgbs / hbm_peak,
                         "traffic": captured_decode_traffic("state_update.cu", d.batch * d.nheads),
                         "alg_bytes_per_launch": decode_alg_bytes(d, 2)},
        }
        del graph

        # the same 512 steps on the int8 cached state (one byte per state element)
        sq, ss = ssd_i8.ssd_i8_state_quantize(torch.from_numpy(d.state).to(dev))

        def decode_pass_q8():
            for s in range(d.steps):
                ssd_i8.ssd_i8_state_update_q8(sq, ss, dx[s], dB[s], dC[s], ddt[s], dA, dD, dsx,
                                              dsb, dsc, y=dy[s], y_dtype="f16")

        side.wait_stream(stream)
        with torch.cuda.stream(side):
            decode_pass_q8()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode_pass_q8()
        for _ in range(max(1, args.warmup // 2)):
            graph.replay()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(args.decode_passes):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        qms = max_over_ranks(ev0.elapsed_time(ev1) / args.decode_passes, dev)
        qstep = decode_alg_bytes(d, 2, state_bytes=1)
        qgbs = qstep * d.steps / (qms * 1e-3) / 1e9
        decode["int8_state"] = {
            "metric": "SSD decode state-update tokens/s (int8 in, int8 cached state)",
            "value": d.batch * d.steps * world / (qms * 1e-3), "unit": UNIT,
            "ms_per_512_steps": qms, "us_per_step": 1e3 * qms / d.steps,
            "gpu_launches_per_pass": d.steps,
            "roofline": {"bound": "hbm", "achieved": qgbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": qgbs / hbm_peak,
                         "traffic": captured_decode_traffic("state_update_q8.cu", d.batch * d.nheads),
                         "alg_bytes_per_launch": qstep},
        }
        del graph

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, nt, sample = oracle_tokens_per_s(case)
        cpu = {"value": v, "unit": UNIT, "cores": nt, "kind": "oracle", "sample": sample}

    if rank != 0:
        device_status_field(statuses)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic (seeded; shapes and value laws of the Mamba-2-8B SSD workload)",
            "config": {"workload": case.name, "global_batch": bsz * world, "seq_len": L,
                       "nheads": H, "headdim": P, "dstate": N, "ngroups": G, "chunk_size": Q,
                       "out_dtype": "i8", "parallelism": f"batch-sharded x{world}, no collective",
                       "l2": "inputs larger than L2 (x 268 MB + B,C 67 MB + dt 17 MB per rank)"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * ssd_i8.KERNELS_PER_CHUNK_SCAN,
            "clocks": clocks.summary(),
            "hadamard_out": hadamard_out, "per_tensor_percentile": per_tensor,
            "varlen_strided": varlen,
            "prefill_1p3b": smaller.get("prefill_1p3b"),
            "prefill_2p7b": smaller.get("prefill_2p7b"),
            "per_channel_scales": per_channel,
            "decode": decode,
            "device_status": device_status_field(statuses),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
