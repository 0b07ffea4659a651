"""GPU parity of the Hadamard-transformed SSD output (y_dtype | SSD_OUT_HADAMARD).

The kernel applies y' = H y / 8 over the 64 head channels (Sylvester order) in its epilogue,
before the dtype conversion.  The oracle is the fp64 scan followed by the orthonormal transform
from scipy; both tolerances carry over unchanged because the transform is orthonormal (it keeps
the L2 norm of the error).  The state path does not see the flag, so final states must be
bit-identical to a call without it.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8
from quantized_mamba_ssd_b200 import workloads as W
from parity_util import check_close, check_i8, head_subset

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    qbuild.build()
    ssd_i8.library()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def run(case, y_dtype="f32", y_scale=1.0, hadamard=True):
    bsz, H, P, N = case.batch, case.nheads, case.headdim, case.dstate
    fs = torch.empty((bsz, H, P, N), dtype=torch.float32, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan(
        dev(case.x), dev(case.B), dev(case.C), dev(case.dt), dev(case.A), dev(case.D),
        dev(case.x_scale), dev(case.B_scale), dev(case.C_scale), case.chunk_size,
        init_state=None if case.init_state is None else dev(case.init_state), final_state=fs,
        y_dtype=y_dtype, y_scale=y_scale, hadamard=hadamard)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), fs.cpu().numpy()


def oracle_hy(case):
    yr, fr = oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                         case.B_scale, case.C_scale, init_state=case.init_state)[:2]
    return oracle.hadamard(yr), fr


CASES = [
    # b, L, H, G, N, Q, law, init
    (2, 300, 8, 2, 128, 256, "laplace_outliers_all", True),
    (1, 517, 4, 4, 64, 128, "laplace_spread", False),
    (3, 130, 4, 1, 16, 64, "normal", True),
    (1, 1, 2, 1, 128, 256, "laplace_outliers_x", True),
]


@pytest.mark.parametrize("b,L,H,G,N,Q,law,init", CASES)
@pytest.mark.parametrize("out", ["f32", "f16"])
def test_hadamard_output_matches_oracle(b, L, H, G, N, Q, law, init, out):
    case = W.make_prefill(b, L, H, 64, N, G, Q, law=law, seed=L + N + Q,
                          with_init_state=init)
    y, fs = run(case, y_dtype=out)
    yr, fr = oracle_hy(case)
    check_close(y, yr, "H y / 8")
    check_close(fs, fr, "final_state")


@pytest.mark.parametrize("Q", [64, 256])
def test_hadamard_int8_output(Q):
    case = W.make_prefill(2, 700, 8, 64, 128, 2, Q, law="laplace_outliers_all", seed=Q,
                          with_init_state=True)
    yr, _ = oracle_hy(case)
    s_y = float(np.abs(yr).max() / 127.0)
    yq, _ = run(case, y_dtype="i8", y_scale=s_y)
    check_i8(yq, oracle.requant(yr, s_y))


def test_transform_is_applied_to_the_plain_output():
    # the kernel's own untransformed fp32 output, transformed in fp64, agrees with its
    # transformed output to fp32 rounding (a wrong sign, order or scale would not)
    case = W.make_prefill(2, 400, 8, 64, 128, 2, 256, law="laplace_outliers_all", seed=5,
                          with_init_state=True)
    y_plain, f_plain = run(case, hadamard=False)
    y_had, f_had = run(case, hadamard=True)
    ref = oracle.hadamard(y_plain)
    err = np.abs(y_had - ref).max()
    assert err <= 4e-6 * np.abs(ref).max(), f"transform error {err:.3e}"
    assert np.array_equal(f_plain, f_had), "the flag changed the final state"


def test_int8_hadamard_is_the_fp32_hadamard_requantized():
    case = W.make_prefill(1, 600, 4, 64, 128, 1, 256, law="laplace_spread", seed=8)
    y32, _ = run(case, y_dtype="f32")
    s_y = np.float32(np.abs(y32).max() / 100.0)
    yq, _ = run(case, y_dtype="i8", y_scale=float(s_y))
    # the per-block scale and the 1/8 are powers of two, so scaling commutes with rounding and
    # the int8 output is exactly the f32 output times fp32(1 / s_y), the product taken exactly
    # (fp64 holds the product of two fp32 values) and rounded once
    inv = np.float32(1.0) / s_y
    expect = np.clip(np.rint(y32.astype(np.float64) * np.float64(inv)), -127, 127)
    assert np.array_equal(yq, expect)


def test_hadamard_varlen():
    lengths = [300, 1, 129, 0, 1000, 57]
    T = sum(lengths)
    case = W.make_prefill(1, T, 8, 64, 128, 2, 256, law="laplace_outliers_all", seed=21)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    init = np.random.default_rng(22).normal(0.0, 0.5, size=(len(lengths), 8, 64, 128))
    init = init.astype(np.float32)
    y = ssd_i8.ssd_i8_chunk_scan_varlen(
        dev(case.x[0]), dev(case.B[0]), dev(case.C[0]), dev(case.dt[0]), dev(case.A),
        dev(case.D), dev(case.x_scale), dev(case.B_scale), dev(case.C_scale), cu, 256,
        init_state=dev(init), y_dtype="f32", hadamard=True)
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    for s in range(len(lengths)):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        yr = oracle.scan(case.x[:, a:b], case.B[:, a:b], case.C[:, a:b], case.dt[:, a:b],
                         case.A, case.D, case.x_scale, case.B_scale, case.C_scale,
                         init_state=init[s][None])[0][0]
        check_close(y[a:b], oracle.hadamard(yr), f"H y / 8 of sequence {s}")


def test_hadamard_at_workload_size_sampled():
    # the int8-output prefill workload (batch 2, 16384 tokens, 128 heads, dstate 128, 8 groups,
    # chunk 256) in the benchmark's launch configuration, with the transform on; the oracle
    # runs sampled (batch, head) pairs whole
    case = W.make_prefill_config(3)
    pairs = [(0, 0), (1, 77), (0, 127)]
    refs = {}
    for b, h in pairs:
        yr, _, _ = oracle.scan(**head_subset(case, [h], batches=[b]))
        refs[(b, h)] = oracle.hadamard(yr[0, :, 0, :])
    s_y = float(max(np.abs(r).max() for r in refs.values()) / 127.0)
    yq, _ = run(case, y_dtype="i8", y_scale=s_y)
    for (b, h), r in refs.items():
        check_i8(yq[b, :, h, :], oracle.requant(r, s_y))


# ---------------------------------------------------------------------------------------
# decode: the same transform of the single-token output, on the fp32 and the int8 state
# ---------------------------------------------------------------------------------------
def _decode_case(seed):
    d = W.make_decode(8, 1, 16, 64, 128, 4, seed=seed)
    return d, dict(x=d.x[0], B=d.B[0], C=d.C[0], dt=d.dt[0])


def _dec_args(d, tok):
    return (dev(tok["x"]), dev(tok["B"]), dev(tok["C"]), dev(tok["dt"]), dev(d.A), dev(d.D),
            dev(d.x_scale), dev(d.B_scale), dev(d.C_scale))


@pytest.mark.parametrize("out", ["f32", "f16", "i8"])
def test_hadamard_decode_fp32_state(out):
    d, tok = _decode_case(61)
    ref_state = d.state.astype(np.float64)
    yr = oracle.hadamard(oracle.step(ref_state, tok["x"], tok["B"], tok["C"], tok["dt"], d.A,
                                     d.D, d.x_scale, d.B_scale, d.C_scale))
    s_y = float(np.abs(yr).max() / 127.0)
    st = dev(d.state)
    y = ssd_i8.ssd_i8_state_update(st, *_dec_args(d, tok), y_dtype=out, y_scale=s_y,
                                   hadamard=True)
    st_plain = dev(d.state)
    ssd_i8.ssd_i8_state_update(st_plain, *_dec_args(d, tok), y_dtype="f32")
    torch.cuda.synchronize()
    if out == "i8":
        check_i8(y.cpu().numpy(), oracle.requant(yr, s_y))
    else:
        check_close(y.float().cpu().numpy(), yr, "H y / 8 (decode)")
    assert torch.equal(st, st_plain), "the flag changed the state update"


@pytest.mark.parametrize("out", ["f32", "i8"])
def test_hadamard_decode_int8_state(out):
    d, tok = _decode_case(62)
    codes, scales = oracle.quantize_state(d.state)
    scales32 = scales.astype(np.float32)
    yr = oracle.hadamard(oracle.step_q8(codes, scales32, tok["x"], tok["B"], tok["C"],
                                        tok["dt"], d.A, d.D, d.x_scale, d.B_scale,
                                        d.C_scale)[0])
    s_y = float(np.abs(yr).max() / 127.0)
    q, s = dev(codes), dev(scales32)
    y = ssd_i8.ssd_i8_state_update_q8(q, s, *_dec_args(d, tok), y_dtype=out, y_scale=s_y,
                                      hadamard=True)
    q2, s2 = dev(codes), dev(scales32)
    ssd_i8.ssd_i8_state_update_q8(q2, s2, *_dec_args(d, tok), y_dtype="f32")
    torch.cuda.synchronize()
    if out == "i8":
        check_i8(y.cpu().numpy(), oracle.requant(yr, s_y))
    else:
        check_close(y.cpu().numpy(), yr, "H y / 8 (int8-state decode)")
    assert torch.equal(q, q2) and torch.equal(s, s2), "the flag changed the cached state"


def test_hadamard_needs_headdim_64():
    d = W.make_decode(2, 1, 4, 32, 16, 1, seed=63)
    st = dev(d.state)
    with pytest.raises(ssd_i8.SSDError):
        ssd_i8.ssd_i8_state_update(st, dev(d.x[0]), dev(d.B[0]), dev(d.C[0]), dev(d.dt[0]),
                                   dev(d.A), dev(d.D), dev(d.x_scale), dev(d.B_scale),
                                   dev(d.C_scale), y_dtype="f32", hadamard=True)
