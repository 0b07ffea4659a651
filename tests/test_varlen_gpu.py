"""GPU parity of the variable-length / strided chunk scan (ssd_i8_chunk_scan_varlen).

Sequences packed back to back are independent scans: the oracle runs each one on its own slice
(with its own initial state) and the kernel's packed output must match it sequence by sequence.
Strided inputs are column slices of one wider projection buffer, as a model's in_proj output
would hand them over.
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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    qbuild.build()
    ssd_i8.library()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def packed_case(lengths, H, G, N, law="laplace_outliers_all", seed=0):
    """One packed problem: a single row of sum(lengths) tokens drawn by the workload generator,
    cut into sequences of the given lengths, with a seeded initial state per sequence."""
    T = int(sum(lengths))
    case = W.make_prefill(1, max(T, 1), H, 64, N, G, 256, law=law, seed=seed)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    rng = np.random.default_rng(seed + 7)
    init = rng.normal(0.0, 0.5, size=(len(lengths), H, 64, N)).astype(np.float32)
    return case, cu, init


def oracle_varlen(case, cu, init, with_init=True):
    """Per-sequence oracle: y [T, H, P] and final states [nseq, H, P, N]."""
    T = int(cu[-1])
    H, P, N = case.nheads, case.headdim, case.dstate
    y = np.zeros((T, H, P))
    fin = np.zeros((len(cu) - 1, H, P, N))
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        st = init[s][None] if with_init else None
        if b == a:
            fin[s] = init[s] if with_init else 0.0
            continue
        ys, fs = oracle.scan(case.x[:, a:b], case.B[:, a:b], case.C[:, a:b], case.dt[:, a:b],
                             case.A, case.D, case.x_scale, case.B_scale, case.C_scale,
                             init_state=st)[:2]
        y[a:b] = ys[0]
        fin[s] = fs[0]
    return y, fin


def gpu_varlen(case, cu, init, y_dtype="f32", y_scale=1.0, with_init=True, strided=False):
    T = int(cu[-1])
    H, P, N, G = case.nheads, case.headdim, case.dstate, case.ngroups
    if strided:
        # x | B | C | pad as columns of one [T, d] int8 buffer; dt inside a wider f32 buffer
        d = H * P + 2 * G * N + 48
        proj = torch.zeros((T, d), dtype=torch.int8, device=DEV)
        proj[:, :H * P] = dev(case.x[0, :T].reshape(T, H * P))
        proj[:, H * P:H * P + G * N] = dev(case.B[0, :T].reshape(T, G * N))
        proj[:, H * P + G * N:H * P + 2 * G * N] = dev(case.C[0, :T].reshape(T, G * N))
        x = proj[:, :H * P].view(T, H, P)
        B = proj[:, H * P:H * P + G * N].view(T, G, N)
        C = proj[:, H * P + G * N:H * P + 2 * G * N].view(T, G, N)
        dtb = torch.zeros((T, H + 5), dtype=torch.float32, device=DEV)
        dtb[:, 2:2 + H] = dev(case.dt[0, :T])
        dt = dtb[:, 2:2 + H]
    else:
        x, B, C, dt = (dev(a[0, :T]) for a in (case.x, case.B, case.C, case.dt))
    fs = torch.full((len(cu) - 1, H, P, N), float("nan"), dtype=torch.float32, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan_varlen(
        x, B, C, dt, dev(case.A), dev(case.D), dev(case.x_scale), dev(case.B_scale),
        dev(case.C_scale), cu, 256, init_state=dev(init) if with_init else None, final_state=fs,
        y_dtype=y_dtype, y_scale=y_scale)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), fs.cpu().numpy()


RAGGED = [300, 1, 128, 129, 0, 57, 1000, 256, 2]


@pytest.mark.parametrize("y_dtype", ["f32", "f16"])
def test_ragged_sequences_match_per_sequence_oracle(y_dtype):
    case, cu, init = packed_case(RAGGED, H=8, G=2, N=128, seed=11)
    yr, fr = oracle_varlen(case, cu, init)
    y, f = gpu_varlen(case, cu, init, y_dtype=y_dtype)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b > a:
            check_close(y[a:b], yr[a:b], f"y of sequence {s}")
        check_close(f[s], fr[s], f"final state of sequence {s}")


def test_ragged_sequences_int8_output():
    case, cu, init = packed_case(RAGGED, H=4, G=2, N=64, seed=12)
    yr, _ = oracle_varlen(case, cu, init)
    s_y = float(np.abs(yr).max() / 127.0)
    yq = gpu_varlen(case, cu, init, y_dtype="i8", y_scale=s_y)[0]
    check_i8(yq, oracle.requant(yr, s_y))


def test_many_short_sequences_without_initial_state():
    rng = np.random.default_rng(3)
    lengths = rng.integers(0, 41, size=150)
    case, cu, init = packed_case(lengths, H=4, G=1, N=32, law="laplace_spread", seed=13)
    yr, fr = oracle_varlen(case, cu, init, with_init=False)
    y, f = gpu_varlen(case, cu, init, with_init=False)
    check_close(y, yr, "y")
    check_close(f, fr, "final states")


def test_strided_projection_views():
    case, cu, init = packed_case([700, 33, 512, 1], H=8, G=2, N=128, seed=14)
    yr, fr = oracle_varlen(case, cu, init)
    y, f = gpu_varlen(case, cu, init, strided=True)
    check_close(y, yr, "y")
    check_close(f, fr, "final states")
    y2, f2 = gpu_varlen(case, cu, init, strided=False)
    assert np.array_equal(y, y2) and np.array_equal(f, f2), "strided and packed inputs disagree"


def test_long_sequences_split_across_ctas():
    # few heads and long sequences: ranges cut sequences, so states hand over between CTAs
    case, cu, init = packed_case([9000, 12000], H=2, G=1, N=128, seed=15)
    yr, fr = oracle_varlen(case, cu, init)
    y, f = gpu_varlen(case, cu, init)
    check_close(y, yr, "y")
    check_close(f, fr, "final states")


def test_uniform_varlen_equals_batched_call():
    case = W.make_prefill(3, 400, 8, 64, 128, 2, 256, law="laplace_outliers_all", seed=16,
                          with_init_state=True)
    yb = ssd_i8.ssd_i8_chunk_scan(dev(case.x), dev(case.B), dev(case.C), dev(case.dt),
                                  dev(case.A), dev(case.D), dev(case.x_scale),
                                  dev(case.B_scale), dev(case.C_scale), 256,
                                  init_state=dev(case.init_state), y_dtype="f32")
    T = 3 * 400
    flat = lambda a: dev(np.ascontiguousarray(a).reshape((T,) + a.shape[2:]))
    yv = ssd_i8.ssd_i8_chunk_scan_varlen(flat(case.x), flat(case.B), flat(case.C),
                                         flat(case.dt), dev(case.A), dev(case.D),
                                         dev(case.x_scale), dev(case.B_scale),
                                         dev(case.C_scale), [0, 400, 800, 1200], 256,
                                         init_state=dev(case.init_state), y_dtype="f32")
    torch.cuda.synchronize()
    assert torch.equal(yb.reshape(T, 8, 64), yv), "uniform varlen differs from the batched call"


def test_tokens_outside_sequences_are_untouched():
    case, _, _ = packed_case([600], H=4, G=1, N=64, seed=17)
    cu = np.array([100, 250, 250, 500], dtype=np.int32)  # tokens [0,100) and [500,600) unused
    init = np.random.default_rng(5).normal(0.0, 0.5, size=(3, 4, 64, 64)).astype(np.float32)
    T = 600
    x, B, C, dt = (dev(a[0, :T]) for a in (case.x, case.B, case.C, case.dt))
    y = torch.full((T, 4, 64), 7.0, dtype=torch.float32, device=DEV)
    ssd_i8.ssd_i8_chunk_scan_varlen(x, B, C, dt, dev(case.A), dev(case.D), dev(case.x_scale),
                                    dev(case.B_scale), dev(case.C_scale), cu, 256,
                                    init_state=dev(init[:3]), y=y, y_dtype="f32")
    torch.cuda.synchronize()
    yy = y.cpu().numpy()
    assert (yy[:100] == 7.0).all() and (yy[500:] == 7.0).all()
    ref = oracle.scan(case.x[:, 100:250], case.B[:, 100:250], case.C[:, 100:250],
                      case.dt[:, 100:250], case.A, case.D, case.x_scale, case.B_scale,
                      case.C_scale, init_state=init[0][None])[0][0]
    check_close(yy[100:250], ref, "y of the first sequence")


def test_malformed_sequences_are_rejected():
    case, cu, init = packed_case([64, 64], H=2, G=1, N=16, seed=18)
    args = [dev(a[0]) for a in (case.x, case.B, case.C, case.dt)]
    rest = [dev(case.A), dev(case.D), dev(case.x_scale), dev(case.B_scale), dev(case.C_scale)]
    with pytest.raises(ssd_i8.SSDError):
        ssd_i8.ssd_i8_chunk_scan_varlen(*args, *rest, [0, 100, 50], 256)  # decreasing
    with pytest.raises(ssd_i8.SSDError):
        ssd_i8.ssd_i8_chunk_scan_varlen(*args, *rest, [0, 64, 129], 256)  # past the tokens


def test_packed_serving_workload_sampled():
    """The packed serving prefill the benchmark times, at full size and in its launch
    configuration: 32768 tokens of the Mamba-2-8B layer as 22 prompts of mixed length, read as
    strided column slices of one projection buffer, int8 output.  Sampled (sequence, head)
    pairs (the shortest, the longest and the middle sequence of the list) are checked against the
    per-sequence oracle: the int8 output within one step, the f32 output of the same call and
    the final states within the tolerances."""
    case, cu = W.make_varlen_config()
    T, H, P, N, G = int(cu[-1]), case.nheads, case.headdim, case.dstate, case.ngroups
    lens = cu[1:] - cu[:-1]
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), len(lens) // 2})
    heads = [0, 77, 127]
    refs = {}
    for s in seqs:
        a, b = int(cu[s]), int(cu[s + 1])
        for h in heads:
            g = h // (H // G)
            yr, fr, _ = oracle.scan(case.x[:, a:b, h:h + 1], case.B[:, a:b, g:g + 1],
                                    case.C[:, a:b, g:g + 1], case.dt[:, a:b, h:h + 1],
                                    case.A[h:h + 1], case.D[h:h + 1], case.x_scale[h:h + 1],
                                    case.B_scale[g:g + 1], case.C_scale[g:g + 1])
            refs[(s, h)] = (yr[0, :, 0, :], fr[0, 0])
    s_y = float(max(np.abs(r[0]).max() for r in refs.values()) / 127.0)
    xw = H * P + 2 * G * N
    proj = torch.empty((T, xw), dtype=torch.int8, device=DEV)
    proj[:, :H * P] = dev(case.x.reshape(T, H * P))
    proj[:, H * P:H * P + G * N] = dev(case.B.reshape(T, G * N))
    proj[:, H * P + G * N:] = dev(case.C.reshape(T, G * N))
    args = [proj[:, :H * P].view(T, H, P), proj[:, H * P:H * P + G * N].view(T, G, N),
            proj[:, H * P + G * N:].view(T, G, N), dev(case.dt.reshape(T, H)), dev(case.A),
            dev(case.D), dev(case.x_scale), dev(case.B_scale), dev(case.C_scale), cu, 256]
    fs = torch.full((len(lens), H, P, N), float("nan"), dtype=torch.float32, device=DEV)
    yq = ssd_i8.ssd_i8_chunk_scan_varlen(*args, final_state=fs, y_dtype="i8", y_scale=s_y)
    y32 = ssd_i8.ssd_i8_chunk_scan_varlen(*args, y_dtype="f32")
    torch.cuda.synchronize()
    yq, y32, fs = yq.cpu().numpy(), y32.cpu().numpy(), fs.cpu().numpy()
    for (s, h), (yr, fr) in refs.items():
        a, b = int(cu[s]), int(cu[s + 1])
        check_i8(yq[a:b, h, :], oracle.requant(yr, s_y))
        check_close(y32[a:b, h, :], yr, f"y of sequence {s}, head {h}")
        check_close(fs[s, h], fr, f"final state of sequence {s}, head {h}")
