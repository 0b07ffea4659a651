"""GPU parity of B and C scales per dstate channel (SSD_SCALES_PER_N) against the oracle.

The per-P(N) quantization axis of the SSDi8 page (Table 10): B_t[n] = s_B[g, n] Bq[t, g, n] and
C_t[n] = s_C[g, n] Cq[t, g, n].  The oracle's scan takes [g, n] scales directly (its pins are in
test_oracle_pins.py).  In the chunk scan the channel products s_C s_B sit inside ChunkBMM, which
then runs on f16 tensor cores, so y and the states are compared with the tolerances of every
other floating-point output; with scales constant over n the per-channel path must reproduce the
per-group kernel bit for bit (its ChunkBMM products are then exact integers in fp32).
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


def gpu_scan(case, y_dtype="f32", y_scale=1.0, hadamard=False, B_scale=None, C_scale=None,
             final=True):
    bsz, L, H, P, N = case.batch, case.seqlen, case.nheads, case.headdim, case.dstate
    fs = torch.empty((bsz, H, P, N), dtype=torch.float32, device=DEV) if final else None
    y = ssd_i8.ssd_i8_chunk_scan(
        dev(case.x), dev(case.B), dev(case.C), dev(case.dt), dev(case.A), dev(case.D),
        dev(case.x_scale), dev(case.B_scale if B_scale is None else B_scale),
        dev(case.C_scale if C_scale is None else C_scale), case.chunk_size,
        init_state=None if case.init_state is None else dev(case.init_state),
        final_state=fs, y_dtype=y_dtype, y_scale=y_scale, hadamard=hadamard)
    torch.cuda.synchronize()
    return y.cpu().numpy(), (fs.cpu().numpy() if final else None)


def oracle_scan(case):
    assert case.B_scale.ndim == 2  # the per-channel scan
    return oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                       case.B_scale, case.C_scale, init_state=case.init_state)[:2]


SMALL = [
    # b, L, H, G, N, Q, law, init, out
    (2, 300, 8, 2, 128, 64, "laplace_outliers_all", True, "f32"),
    (2, 300, 8, 2, 128, 128, "laplace_outliers_all", False, "f16"),
    (1, 517, 4, 4, 128, 256, "laplace_spread", True, "f32"),
    (3, 200, 6, 3, 16, 64, "normal", True, "f16"),
    (2, 130, 4, 1, 32, 128, "laplace_outliers_x", True, "f32"),
    (2, 257, 4, 2, 64, 256, "laplace_outliers_all", False, "f32"),
    (1, 1, 4, 2, 128, 256, "normal", True, "f32"),
    (1, 63, 2, 1, 128, 64, "normal", True, "f32"),
]


@pytest.mark.parametrize("b,L,H,G,N,Q,law,init,out", SMALL)
def test_small_prefill_per_n_matches_oracle(b, L, H, G, N, Q, law, init, out):
    case = W.make_prefill(b, L, H, 64, N, G, Q, law=law, scales="channel", seed=L + 7 * H + N,
                          with_init_state=init)
    assert case.B_scale.shape == (G, N)
    y, fs = gpu_scan(case, y_dtype=out)
    yr, fr = oracle_scan(case)
    check_close(y, yr, "y")
    check_close(fs, fr, "final_state")


def test_per_n_int8_output():
    case = W.make_prefill(2, 400, 8, 64, 128, 2, 256, law="laplace_outliers_all", scales="channel",
                          seed=78, with_init_state=True)
    yr, _ = oracle_scan(case)
    s_y = float(np.abs(yr).max() / 127.0)
    yq, _ = gpu_scan(case, y_dtype="i8", y_scale=s_y)
    check_i8(yq, oracle.requant(yr, s_y))


def test_per_n_constant_over_channels_is_the_per_group_kernel_bit_for_bit():
    # u~_n = 1 for every channel: ChunkBMM's f16 products are exact integers, and every other
    # step takes the same values as the per-group kernel
    case = W.make_prefill(2, 700, 8, 64, 128, 2, 128, law="laplace_outliers_all", scales="head",
                          seed=79, with_init_state=True)
    N = case.dstate
    sb = np.repeat(case.B_scale[:, None], N, axis=1)
    sc = np.repeat(case.C_scale[:, None], N, axis=1)
    for out in ("f32", "i8"):
        y_g, f_g = gpu_scan(case, y_dtype=out, y_scale=0.05)
        y_n, f_n = gpu_scan(case, y_dtype=out, y_scale=0.05, B_scale=sb, C_scale=sc)
        assert np.array_equal(y_g, y_n), out
        assert np.array_equal(f_g, f_n), out


def test_per_n_scale_of_one_channel_acts_on_its_state_column():
    # doubling s_B[g, k] doubles column k of the final states of group g's heads (the state is
    # linear in B), and nothing else, on the GPU as in the oracle
    case = W.make_prefill(1, 300, 4, 64, 128, 2, 128, law="laplace_outliers_all",
                          scales="channel", seed=80)
    g, k = 1, 37
    sb = case.B_scale.copy()
    sb[g, k] *= 2
    _, f0 = gpu_scan(case)
    _, f1 = gpu_scan(case, B_scale=sb)
    heads = np.arange(case.nheads)[np.arange(case.nheads) // (case.nheads // case.ngroups) == g]
    expect = f0.copy()
    expect[:, heads, :, k] *= 2
    check_close(f1, expect, "final_state after doubling one channel's B scale")
    others = np.setdiff1d(np.arange(case.nheads), heads)
    check_close(f1[:, others], f0[:, others], "other groups' states")


def test_per_n_hadamard_output():
    case = W.make_prefill(2, 333, 4, 64, 128, 2, 128, law="laplace_outliers_all",
                          scales="channel", seed=81, with_init_state=True)
    y, _ = gpu_scan(case, y_dtype="f32", hadamard=True)
    yr, _ = oracle_scan(case)
    check_close(y, oracle.hadamard(yr), "Hadamard y")


def test_per_n_varlen_strided():
    H, P, N, G = 8, 64, 128, 2
    lens = [300, 1, 0, 517, 129]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    case = W.make_prefill(1, T, H, P, N, G, 128, law="laplace_outliers_all", scales="channel",
                          seed=82)
    init = (0.1 * np.random.default_rng(83).standard_normal((len(lens), H, P, N))).astype(np.float32)
    # x, B and C as column slices of one projection row
    xw = H * P + 2 * G * N
    proj = torch.zeros((T, xw), dtype=torch.int8, device=DEV)
    proj[:, :H * P] = dev(case.x.reshape(T, H * P))
    proj[:, H * P:H * P + G * N] = dev(case.B.reshape(T, G * N))
    proj[:, H * P + G * N:] = dev(case.C.reshape(T, G * N))
    fs = torch.empty((len(lens), H, P, N), dtype=torch.float32, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan_varlen(
        proj[:, :H * P].view(T, H, P), proj[:, H * P:H * P + G * N].view(T, G, N),
        proj[:, H * P + G * N:].view(T, G, N), dev(case.dt.reshape(T, H)), dev(case.A),
        dev(case.D), dev(case.x_scale), dev(case.B_scale), dev(case.C_scale), cu, 128,
        init_state=dev(init), final_state=fs, y_dtype="f32")
    torch.cuda.synchronize()
    y, fs = y.cpu().numpy(), fs.cpu().numpy()
    for s, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        if e == a:
            assert np.array_equal(fs[s], init[s])
            continue
        yr, fr, _ = oracle.scan(case.x[:, a:e], case.B[:, a:e], case.C[:, a:e], case.dt[:, a:e],
                                case.A, case.D, case.x_scale, case.B_scale, case.C_scale,
                                init_state=init[s:s + 1])
        check_close(y[a:e], yr[0], f"y of sequence {s}")
        check_close(fs[s], fr[0], f"final_state of sequence {s}")


def test_per_n_long_prefill_at_workload_size():
    # the Mamba-2-8B-shaped long prefill with per-channel B/C scales, int8 out, in the launch
    # configuration the benchmark times; sampled (batch, head) pairs whole
    case = W.make_prefill_config(3, scales="channel")
    pairs = [(0, 0), (1, 127), (0, 77), (1, 35)]
    refs = {}
    for b, h in pairs:
        yr, fr, _ = oracle.scan(**head_subset(case, [h], batches=[b]))
        refs[(b, h)] = (yr[0, :, 0, :], fr[0, 0])
    s_y = float(max(np.abs(r[0]).max() for r in refs.values()) / 127.0)
    yq, fs = gpu_scan(case, y_dtype="i8", y_scale=s_y)
    for (b, h), (yr, fr) in refs.items():
        check_i8(yq[b, :, h, :], oracle.requant(yr, s_y))
        check_close(fs[b, h], fr, f"final_state[b={b},h={h}]")
    y32, _ = gpu_scan(case, y_dtype="f32", final=False)
    for (b, h), (yr, _) in refs.items():
        check_close(y32[b, :, h, :], yr, f"y[b={b},h={h}]")


# ---- decode steps with per-channel scales ----

@pytest.mark.parametrize("N,G", [(128, 8), (64, 2), (16, 1)])
def test_decode_step_per_n_matches_oracle(N, G):
    # a decode step is a length-1 prefill from the given state (the oracle's per-N scan)
    d = W.make_decode(4, 3, 16, 64, N, G, seed=84 + N, scales="channel")
    assert d.B_scale.shape == (G, N)
    st = dev(d.state)
    h64 = d.state.astype(np.float64)
    for t in range(d.steps):
        y = ssd_i8.ssd_i8_state_update(st, dev(d.x[t]), dev(d.B[t]), dev(d.C[t]), dev(d.dt[t]),
                                       dev(d.A), dev(d.D), dev(d.x_scale), dev(d.B_scale),
                                       dev(d.C_scale), y_dtype="f32")
        torch.cuda.synchronize()
        yr, fr, _ = oracle.scan(d.x[t][:, None], d.B[t][:, None], d.C[t][:, None],
                                d.dt[t][:, None], d.A, d.D, d.x_scale, d.B_scale, d.C_scale,
                                init_state=h64)
        check_close(y.cpu().numpy(), yr[:, 0], f"y step {t}")
        check_close(st.cpu().numpy(), fr, f"state step {t}")
        h64 = fr


def test_decode_step_q8_per_n_matches_oracle():
    d = W.make_decode(4, 1, 16, 64, 128, 4, seed=90, scales="channel")
    codes, scales = oracle.quantize_state(d.state)
    sq, ss = dev(codes), dev(scales.astype(np.float32))
    y = ssd_i8.ssd_i8_state_update_q8(sq, ss, dev(d.x[0]), dev(d.B[0]), dev(d.C[0]),
                                      dev(d.dt[0]), dev(d.A), dev(d.D), dev(d.x_scale),
                                      dev(d.B_scale), dev(d.C_scale), y_dtype="f32")
    torch.cuda.synchronize()
    h = codes.astype(np.float64) * scales.astype(np.float32).astype(np.float64)[:, :, None, None]
    yr, fr, _ = oracle.scan(d.x[0][:, None], d.B[0][:, None], d.C[0][:, None], d.dt[0][:, None],
                            d.A, d.D, d.x_scale, d.B_scale, d.C_scale, init_state=h)
    check_close(y.cpu().numpy(), yr[:, 0], "y")
    c2, s2 = oracle.quantize_state(fr)
    got = sq.cpu().numpy().astype(np.int32)
    dq = np.abs(got - c2.astype(np.int32))
    assert dq.max() <= 1 and (dq == 0).mean() >= 0.999
    assert np.allclose(ss.cpu().numpy(), s2, rtol=1e-5, atol=0)
