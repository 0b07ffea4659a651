"""Seeded random shapes for the chunk scan and both decode steps, each against the oracle.

Each case draws batch, length (ragged, down to one token), heads, groups, dstate, chunk size,
value law, scale recipe, output dtype, Hadamard flag and initial state from a fixed seed, so a
failure names a reproducible case.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8
from quantized_mamba_ssd_b200 import workloads as W
from parity_util import check_close, check_i8

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LAWS = ["normal", "laplace_outliers_x", "laplace_spread", "laplace_outliers_all"]
SCALES = ["head", "tensor", "percentile"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    qbuild.build()
    ssd_i8.library()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def draw_scan_case(seed):
    r = np.random.default_rng(seed)
    G = int(r.choice([1, 2, 3, 4]))
    H = G * int(r.integers(1, 5))
    return dict(b=int(r.integers(1, 4)), L=int(r.integers(1, 700)), H=H, G=G,
                N=int(r.choice([16, 32, 64, 128])), Q=int(r.choice([64, 128, 256])),
                law=str(r.choice(LAWS)), scales=str(r.choice(SCALES)),
                out=str(r.choice(["f32", "f16", "i8"])), had=bool(r.integers(0, 2)),
                init=bool(r.integers(0, 2)))


@pytest.mark.parametrize("seed", range(24))
def test_random_chunk_scan(seed):
    k = draw_scan_case(5000 + seed)
    c = W.make_prefill(k["b"], k["L"], k["H"], 64, k["N"], k["G"], k["Q"], law=k["law"],
                       scales=k["scales"], seed=seed, with_init_state=k["init"])
    yr, fr, _ = oracle.scan(c.x, c.B, c.C, c.dt, c.A, c.D, c.x_scale, c.B_scale, c.C_scale,
                            init_state=c.init_state)
    if k["had"]:
        yr = oracle.hadamard(yr)
    s_y = float(np.abs(yr).max() / 127.0) if np.abs(yr).max() > 0 else 1.0
    fs = torch.empty((k["b"], k["H"], 64, k["N"]), dtype=torch.float32, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan(dev(c.x), dev(c.B), dev(c.C), dev(c.dt), dev(c.A), dev(c.D),
                                 dev(c.x_scale), dev(c.B_scale), dev(c.C_scale), k["Q"],
                                 init_state=None if c.init_state is None else dev(c.init_state),
                                 final_state=fs, y_dtype=k["out"], y_scale=s_y,
                                 hadamard=k["had"])
    torch.cuda.synchronize()
    if k["out"] == "i8":
        check_i8(y.cpu().numpy(), oracle.requant(yr, s_y))
    else:
        check_close(y.float().cpu().numpy(), yr, f"y {k}")
    check_close(fs.cpu().numpy(), fr, f"final state {k}")


@pytest.mark.parametrize("seed", range(12))
def test_random_decode_steps(seed):
    r = np.random.default_rng(7000 + seed)
    G = int(r.choice([1, 2, 4]))
    H = G * int(r.integers(1, 5))
    N = int(r.choice([16, 32, 64, 128, 256]))
    bsz = int(r.integers(1, 40))
    out = str(r.choice(["f32", "f16"]))
    had = bool(r.integers(0, 2))
    d = W.make_decode(bsz, 1, H, 64, N, G, seed=seed)
    tok = [d.x[0], d.B[0], d.C[0], d.dt[0]]
    rest = [d.A, d.D, d.x_scale, d.B_scale, d.C_scale]
    # fp32 state
    ref_state = d.state.astype(np.float64)
    yr = oracle.step(ref_state, *tok, *rest)
    st = dev(d.state)
    y = ssd_i8.ssd_i8_state_update(st, *(dev(a) for a in tok), *(dev(a) for a in rest),
                                   y_dtype=out, hadamard=had)
    torch.cuda.synchronize()
    check_close(y.float().cpu().numpy(), oracle.hadamard(yr) if had else yr, "decode y")
    check_close(st.cpu().numpy(), ref_state, "decode state")
    # int8 cached state (shapes it supports)
    codes, scales = oracle.quantize_state(d.state)
    scales32 = scales.astype(np.float32)
    q, s = dev(codes), dev(scales32)
    yq = ssd_i8.ssd_i8_state_update_q8(q, s, *(dev(a) for a in tok), *(dev(a) for a in rest),
                                       y_dtype=out, hadamard=had)
    torch.cuda.synchronize()
    yqr = oracle.step_q8(codes, scales32, *tok, *rest)[0]
    check_close(yq.float().cpu().numpy(), oracle.hadamard(yqr) if had else yqr, "int8-state y")
