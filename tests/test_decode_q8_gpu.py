"""GPU parity of the int8 cached decode state (ssd_i8_state_quantize, ssd_i8_state_update_q8).

The quantisation rule is scale = max|h| / 127 per (batch, head) and code = clamp(rne(h /
scale), -127, 127).  Codes are integers decided by floating point, so the kernel's quantiser is
checked bit for bit against the same rule evaluated in the kernel's precision (fp32, numpy),
and against the fp64 oracle within one code.  The decode step is compared with the oracle from
the same cached state (y, codes, scales), and over a run of steps in which each side keeps its
own cache.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8
from quantized_mamba_ssd_b200 import workloads as W
from parity_util import check_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
CODE_FRACTION = 0.999  # codes equal to the oracle's (the rest within one step)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    qbuild.build()
    ssd_i8.library()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def fp32_rule(state):
    """The quantisation rule in fp32, the order the kernel evaluates it in."""
    st = np.asarray(state, dtype=np.float32)
    bsz, H = st.shape[:2]
    amax = np.abs(st).reshape(bsz, H, -1).max(axis=2).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(127.0) / amax, np.float32(0.0)).astype(np.float32)
    q = np.rint((st * inv[:, :, None, None]).astype(np.float32))
    q = np.clip(q, -127, 127).astype(np.int8)
    return q, (amax / np.float32(127.0)).astype(np.float32)


def codes_close(got, ref):
    """Every code within one step of the oracle's (a tie decided in another precision)."""
    d = np.abs(got.astype(np.int32) - ref.astype(np.int32))
    assert d.max() <= 1, f"a code differs by {d.max()}"
    assert (d == 0).mean() >= CODE_FRACTION, f"only {(d == 0).mean():.6f} of the codes agree"


@pytest.mark.parametrize("N", [16, 64, 128, 256])
def test_quantize_matches_rule_bit_exact(N):
    rng = np.random.default_rng(N)
    st = rng.laplace(0.0, 0.3, size=(3, 5, 64, N)).astype(np.float32)
    st[0, 1] = 0.0  # an all-zero (batch, head)
    q, s = ssd_i8.ssd_i8_state_quantize(dev(st))
    torch.cuda.synchronize()
    qr, sr = fp32_rule(st)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(s.cpu().numpy(), sr)
    qo, so = oracle.quantize_state(st)
    codes_close(q.cpu().numpy(), qo)
    assert np.allclose(s.cpu().numpy(), so, rtol=1e-6, atol=0)


def decode_inputs(bsz, H, G, N, seed):
    case = W.make_decode(bsz, 1, H, 64, N, G, seed=seed)
    t = 0
    return case, dict(x=case.x[t], B=case.B[t], C=case.C[t], dt=case.dt[t])


@pytest.mark.parametrize("N,G", [(128, 8), (64, 2), (256, 4), (16, 1)])
def test_one_step_from_the_same_cache(N, G):
    bsz, H = 4, 16
    case, tok = decode_inputs(bsz, H, G, N, seed=40 + N)
    codes, scales = oracle.quantize_state(case.state)
    scales32 = scales.astype(np.float32)
    q = dev(codes)
    s = dev(scales32)
    y = ssd_i8.ssd_i8_state_update_q8(q, s, dev(tok["x"]), dev(tok["B"]), dev(tok["C"]),
                                      dev(tok["dt"]), dev(case.A), dev(case.D),
                                      dev(case.x_scale), dev(case.B_scale), dev(case.C_scale),
                                      y_dtype="f32")
    torch.cuda.synchronize()
    yr, cr, sr = oracle.step_q8(codes, scales32, tok["x"], tok["B"], tok["C"], tok["dt"],
                                case.A, case.D, case.x_scale, case.B_scale, case.C_scale)
    check_close(y.cpu().numpy(), yr, "y")
    codes_close(q.cpu().numpy(), cr)
    assert np.allclose(s.cpu().numpy(), sr, rtol=1e-5, atol=0)


def test_run_of_steps_each_side_with_its_own_cache():
    bsz, H, G, N, steps = 8, 16, 4, 128, 16
    case = W.make_decode(bsz, steps, H, 64, N, G, seed=77)
    codes, scales = oracle.quantize_state(case.state)
    q, s = dev(codes), dev(scales.astype(np.float32))
    oc, osc = codes, scales.astype(np.float64)
    for t in range(steps):
        y = ssd_i8.ssd_i8_state_update_q8(q, s, dev(case.x[t]), dev(case.B[t]), dev(case.C[t]),
                                          dev(case.dt[t]), dev(case.A), dev(case.D),
                                          dev(case.x_scale), dev(case.B_scale),
                                          dev(case.C_scale), y_dtype="f32")
        yr, oc, osc = oracle.step_q8(oc, osc, case.x[t], case.B[t], case.C[t], case.dt[t],
                                     case.A, case.D, case.x_scale, case.B_scale, case.C_scale)
        torch.cuda.synchronize()
        check_close(y.cpu().numpy(), yr, f"y at step {t}")


def test_prefill_state_hands_over_to_the_int8_cache():
    # the final fp32 state of a prefill, quantised, then decoded: the same as the oracle run
    case = W.make_prefill(2, 300, 8, 64, 128, 2, 256, law="laplace_outliers_all", seed=91)
    fs = torch.empty((2, 8, 64, 128), dtype=torch.float32, device=DEV)
    ssd_i8.ssd_i8_chunk_scan(dev(case.x), dev(case.B), dev(case.C), dev(case.dt), dev(case.A),
                             dev(case.D), dev(case.x_scale), dev(case.B_scale),
                             dev(case.C_scale), 256, final_state=fs, y_dtype="f32")
    q, s = ssd_i8.ssd_i8_state_quantize(fs)
    torch.cuda.synchronize()
    fr = oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                     case.B_scale, case.C_scale)[1]
    deq = q.cpu().numpy().astype(np.float64) * s.cpu().numpy()[:, :, None, None]
    # the cache holds the oracle's final state to within half a step (+ the scan's tolerance)
    step = s.cpu().numpy()[:, :, None, None]
    assert (np.abs(deq - fr) <= 0.5 * step + 2e-3 * np.abs(fr).max()).all()


def test_int8_state_workload_sampled():
    """The batch-128, Mamba-2-8B-shaped decode at full size on the int8 cached state, in the
    launch configuration the benchmark times: 64 steps, sampled (batch, head) pairs followed
    through every step by the oracle with its own cache."""
    d = W.make_decode_config()
    steps = 64
    q, s = ssd_i8.ssd_i8_state_quantize(dev(d.state))
    codes0, scales0 = q.cpu().numpy(), s.cpu().numpy()
    pairs = [(0, 0), (127, 127), (64, 3), (5, 90)]
    ys = {pr: [] for pr in pairs}
    args = [dev(d.A), dev(d.D), dev(d.x_scale), dev(d.B_scale), dev(d.C_scale)]
    xs, Bs, Cs, dts = dev(d.x), dev(d.B), dev(d.C), dev(d.dt)
    for t in range(steps):
        y = ssd_i8.ssd_i8_state_update_q8(q, s, xs[t], Bs[t], Cs[t], dts[t], *args, y_dtype="f32")
        for (b, h) in pairs:
            ys[(b, h)].append(y[b, h].clone())
    torch.cuda.synchronize()
    H, G = d.nheads, d.ngroups
    for (b, h) in pairs:
        g = h // (H // G)
        oc = codes0[b:b + 1, h:h + 1]
        osc = scales0[b:b + 1, h:h + 1].astype(np.float64)
        refs = []
        for t in range(steps):
            yr, oc, osc = oracle.step_q8(oc, osc, d.x[t][b:b + 1, h:h + 1],
                                         d.B[t][b:b + 1, g:g + 1], d.C[t][b:b + 1, g:g + 1],
                                         d.dt[t][b:b + 1, h:h + 1], d.A[h:h + 1], d.D[h:h + 1],
                                         d.x_scale[h:h + 1], d.B_scale[g:g + 1],
                                         d.C_scale[g:g + 1])
            refs.append(yr[0, 0])
        got = torch.stack(ys[(b, h)]).cpu().numpy()
        check_close(got, np.stack(refs), f"int8-state decode y (b={b}, h={h})")
